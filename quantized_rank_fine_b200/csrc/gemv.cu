// Small-M forward: Y = X deq(Wq) + V B for M <= 16 tokens (NF4 dequant-GEMV).
//
// At a few tokens the forward is bound by reading the 4-bit codes once from HBM
// (0.516 B per weight), so the kernel is organised around that stream:
//
//   * Work unit: a 64-column panel of W (one absmax block per row) times a
//     K-range; grid = panels x K-splits, about two CTAs per SM.  Warp w of a
//     CTA takes every 8th 16-row step of the CTA's K-range, so consecutive warps
//     read consecutive rows.
//   * Tensor cores, swap-AB: mma.sync m16n8k16 with the weight as the 16 x 16
//     A operand (rows = 16 output columns, cols = 16 k) and the tokens as the
//     8-wide B operand.  A lane (g, t) loads one 32-bit word (8 codes) from each
//     of the rows k0+2t, k0+2t+1, k0+2t+8, k0+2t+9 of its panel; byte j of the
//     words fills tile j (output columns 8g+2j, 8g+2j+1).  A 256-entry table in
//     shared memory maps a code byte to the bf16 pair of its two levels (one copy
//     per lane, so lookups never conflict), and one byte-permute pairs two rows
//     into an A register.  Each warp issues the code loads of up to 8 of its
//     steps before the shared-memory set-up, and keeps 8 steps in flight after.
//   * The block scale is folded into the activations: sum_k x_k (a'_k l_k) =
//     sum_k (x_k a'_k) l_k.  Per CTA, x'[m][k] = bf16(x[m][k] * a'(k, panel)) is
//     computed once into shared memory (M/64 multiplies per weight instead of
//     one per weight), and the weight operand is the bf16 NF4 level itself.
//   * Each CTA sums its 8 warps in shared memory and writes one fp32 partial;
//     the last CTA of a panel (atomic ticket in the workspace, reset after use)
//     adds the K-split partials in order, adds V B, and writes bf16 Y.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kGvThreads = 256;
constexpr int kGvWarps = 8;
constexpr int kPanel = 64;
constexpr int kDepth = 8;                       // code-load steps in flight per warp
constexpr int kLutBytes = 256 * 32 * 4;         // 32 copies of the 256-entry table

struct GemvArgs {
  const uint8_t* codes;
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t K, N;          // weight (K = in, N = out)
  int M;                 // tokens, 1..16
  const uint16_t* X;     // (M, K) bf16
  const uint16_t* V;     // (M, r) bf16
  const uint16_t* B;     // (r, N) bf16
  int r;
  uint16_t* Y;           // (M, N) bf16
  float* part;           // [S][M][N] fp32
  uint32_t* tickets;     // [N / 64], zero between calls
  int S;                 // K-splits
  int Kc;                // rows per split (multiple of 16)
};

__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MT>   // token tiles of 8: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kGvThreads)
nf4_gemv_kernel(const GemvArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);                   // [256][32]: entry b, copy lane
  float* ascale = reinterpret_cast<float*>(smem + kLutBytes);          // Kc floats
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + kLutBytes + 4 * p.Kc);  // [MT*8][Kc] bf16
  float* red = reinterpret_cast<float*>(xs);                           // [8][MT*8][64] after the loop
  __shared__ int last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int panel = blockIdx.x, split = blockIdx.y;
  const int64_t k_begin = static_cast<int64_t>(split) * p.Kc;
  const int rows = static_cast<int>(p.K - k_begin < p.Kc ? p.K - k_begin : p.Kc);
  const int64_t blocks_per_row = p.N / kPanel;
  constexpr int TM = MT * 8;

  const int nsteps = rows / 16;
  const uint8_t* cbase = p.codes + (k_begin * p.N + static_cast<int64_t>(panel) * kPanel) / 2 + 4 * g;
  const int64_t row_bytes = p.N / 2;
  const int r0 = 2 * t, r1 = 2 * t + 1, r2 = 2 * t + 8, r3 = 2 * t + 9;
  // this warp's steps are warp, warp + 8, ...; the codes of the first kDepth of
  // them are requested before anything else
  uint32_t wq[kDepth][4];
#pragma unroll
  for (int i = 0; i < kDepth; ++i) {
    const int st = warp + i * kGvWarps;
    if (st < nsteps) {
      const uint8_t* c = cbase + static_cast<int64_t>(st * 16) * row_bytes;
      wq[i][0] = __ldcs(reinterpret_cast<const unsigned int*>(c + r0 * row_bytes));
      wq[i][1] = __ldcs(reinterpret_cast<const unsigned int*>(c + r1 * row_bytes));
      wq[i][2] = __ldcs(reinterpret_cast<const unsigned int*>(c + r2 * row_bytes));
      wq[i][3] = __ldcs(reinterpret_cast<const unsigned int*>(c + r3 * row_bytes));
    }
  }

  // level pairs of every code byte, one copy per lane
  {
    const uint32_t v = pack_bf16x2(nf4_level(tid & 15), nf4_level(tid >> 4));
    uint4* dst = reinterpret_cast<uint4*>(lut + tid * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(v, v, v, v);
  }
  // absmax' of this panel's block in each row of the range
  for (int kk = tid; kk < rows; kk += kGvThreads) {
    const int64_t b = (k_begin + kk) * blocks_per_row + panel;
    ascale[kk] = absmax_deq(p.dq_codes[b], p.dq_scales[b / kGroup]);
  }
  __syncthreads();
  // x' = bf16(x * a') for the real tokens, two k at a time (padded tokens are
  // never read: their B operand is zero in registers)
  for (int m = 0; m < p.M; ++m) {
    const uint32_t* xrow = reinterpret_cast<const uint32_t*>(p.X + static_cast<int64_t>(m) * p.K + k_begin);
    uint32_t* xsrow = reinterpret_cast<uint32_t*>(xs + m * p.Kc);
    for (int kk2 = tid; kk2 < rows / 2; kk2 += kGvThreads) {
      const uint32_t x2 = __ldg(xrow + kk2);
      xsrow[kk2] = pack_bf16x2(mul_rn(bf16_lo(x2), ascale[2 * kk2]), mul_rn(bf16_hi(x2), ascale[2 * kk2 + 1]));
    }
  }
  __syncthreads();

  float acc[MT][4][4];
#pragma unroll
  for (int a = 0; a < MT; ++a)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][j][c] = 0.0f;

  const uint32_t* mylut = lut + lane;
#pragma unroll 1
  for (int base = 0; base * kGvWarps + warp < nsteps; base += kDepth) {
#pragma unroll
   for (int i = 0; i < kDepth; ++i) {
    const int st = warp + (base + i) * kGvWarps;
    if (st >= nsteps) break;
    const uint32_t c0 = wq[i][0], c1 = wq[i][1], c2 = wq[i][2], c3 = wq[i][3];
    const int kk0 = st * 16;
    const int nst = st + kDepth * kGvWarps;      // refill this slot kDepth steps ahead
    if (nst < nsteps) {
      const uint8_t* c = cbase + static_cast<int64_t>(nst * 16) * row_bytes;
      wq[i][0] = __ldcs(reinterpret_cast<const unsigned int*>(c + r0 * row_bytes));
      wq[i][1] = __ldcs(reinterpret_cast<const unsigned int*>(c + r1 * row_bytes));
      wq[i][2] = __ldcs(reinterpret_cast<const unsigned int*>(c + r2 * row_bytes));
      wq[i][3] = __ldcs(reinterpret_cast<const unsigned int*>(c + r3 * row_bytes));
    }
    uint32_t bx[MT][2];
#pragma unroll
    for (int a = 0; a < MT; ++a) {
      const uint16_t* xr = xs + (a * 8 + g) * p.Kc + kk0;
      const bool real = (a * 8 + g) < p.M;
      bx[a][0] = real ? *reinterpret_cast<const uint32_t*>(xr + r0) : 0u;
      bx[a][1] = real ? *reinterpret_cast<const uint32_t*>(xr + r2) : 0u;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t la = mylut[((c0 >> (8 * j)) & 0xFFu) * 32];
      const uint32_t lb = mylut[((c1 >> (8 * j)) & 0xFFu) * 32];
      const uint32_t lc = mylut[((c2 >> (8 * j)) & 0xFFu) * 32];
      const uint32_t ld = mylut[((c3 >> (8 * j)) & 0xFFu) * 32];
      const uint32_t a0 = __byte_perm(la, lb, 0x5410);   // even column, rows 2t, 2t+1
      const uint32_t a1 = __byte_perm(la, lb, 0x7632);   // odd column
      const uint32_t a2 = __byte_perm(lc, ld, 0x5410);   // even column, rows 2t+8, 2t+9
      const uint32_t a3 = __byte_perm(lc, ld, 0x7632);
#pragma unroll
      for (int a = 0; a < MT; ++a) mma_bf16_16816(acc[a][j], a0, a1, a2, a3, bx[a][0], bx[a][1]);
    }
   }
  }
  __syncthreads();   // x' no longer read; its space becomes the reduction buffer

  // D fragment of tile j: (column 8g+2j, tokens 2t, 2t+1) and (column 8g+2j+1, same tokens).
#pragma unroll
  for (int a = 0; a < MT; ++a)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n0 = 8 * g + 2 * j;
      const int m0 = a * 8 + 2 * t;
      float* rw = red + warp * TM * kPanel;
      rw[m0 * kPanel + n0] = acc[a][j][0];
      rw[(m0 + 1) * kPanel + n0] = acc[a][j][1];
      rw[m0 * kPanel + n0 + 1] = acc[a][j][2];
      rw[(m0 + 1) * kPanel + n0 + 1] = acc[a][j][3];
    }
  __syncthreads();
  const int64_t col0 = static_cast<int64_t>(panel) * kPanel;
  for (int e = tid; e < p.M * kPanel; e += kGvThreads) {
    const int m = e / kPanel, n = e % kPanel;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kGvWarps; ++w) s += red[(w * TM + m) * kPanel + n];
    p.part[(static_cast<int64_t>(split) * p.M + m) * p.N + col0 + n] = s;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t ticket = atomicAdd(p.tickets + panel, 1u);
    last = (ticket == static_cast<uint32_t>(p.S - 1));
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int e = tid; e < p.M * kPanel; e += kGvThreads) {
    const int m = e / kPanel, n = e % kPanel;
    float y = 0.0f;
    for (int s = 0; s < p.S; ++s) y += __ldcg(p.part + (static_cast<int64_t>(s) * p.M + m) * p.N + col0 + n);
    float vb = 0.0f;
    for (int j = 0; j < p.r; ++j)
      vb = fmaf(__uint_as_float(static_cast<uint32_t>(p.V[m * p.r + j]) << 16),
                __uint_as_float(static_cast<uint32_t>(p.B[static_cast<int64_t>(j) * p.N + col0 + n]) << 16), vb);
    const uint32_t packed = pack_bf16x2(y + vb, 0.0f);
    p.Y[static_cast<int64_t>(m) * p.N + col0 + n] = static_cast<uint16_t>(packed & 0xFFFFu);
  }
  if (tid == 0) p.tickets[panel] = 0u;   // ready for the next call
}

constexpr int kMaxKc = 4096;

void gemv_plan(int64_t K, int64_t N, int& S, int& Kc) {
  const int64_t panels = N / kPanel;
  int64_t s = std::max<int64_t>(1, (2 * 148 + panels / 2) / panels);
  s = std::max<int64_t>(s, (K + kMaxKc - 1) / kMaxKc);
  int64_t kc = (K + s - 1) / s;
  kc = (kc + 127) / 128 * 128;
  s = (K + kc - 1) / kc;
  S = static_cast<int>(s);
  Kc = static_cast<int>(kc);
}

size_t gemv_smem_bytes(int Kc, int MT) {
  const size_t xs = static_cast<size_t>(MT) * 8 * Kc * 2;
  const size_t red = static_cast<size_t>(kGvWarps) * MT * 8 * kPanel * 4;
  return kLutBytes + 4 * static_cast<size_t>(Kc) + std::max(xs, red);
}

}  // namespace

size_t gemv_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  int S, Kc;
  gemv_plan(K, N, S, Kc);
  return static_cast<size_t>(S) * M * N * 4;
}

cudaError_t launch_gemv(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B, int64_t M,
                        int r, uint16_t* Y, float* part, uint32_t* tickets, cudaStream_t stream) {
  int S, Kc;
  gemv_plan(w.in, w.out, S, Kc);
  GemvArgs a{w.codes, w.dq_codes, w.dq_scales, w.in, w.out, static_cast<int>(M), X, V, B, r, Y, part, tickets, S, Kc};
  const int MT = M <= 8 ? 1 : 2;
  const size_t smem = gemv_smem_bytes(Kc, MT);
  dim3 grid(static_cast<unsigned>(w.out / kPanel), static_cast<unsigned>(S));
  // the largest dynamic shared memory any plan uses, set once per device
  static bool set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !set[dev]) {
    const int most = static_cast<int>(gemv_smem_bytes(kMaxKc, 2));
    cudaError_t e = cudaFuncSetAttribute(nf4_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(nf4_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  timing_before(QLORA_KERNEL_GEMV, stream);
  if (MT == 1)
    nf4_gemv_kernel<1><<<grid, kGvThreads, smem, stream>>>(a);
  else
    nf4_gemv_kernel<2><<<grid, kGvThreads, smem, stream>>>(a);
  timing_after(QLORA_KERNEL_GEMV, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
