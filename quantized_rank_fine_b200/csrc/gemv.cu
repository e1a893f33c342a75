// Small-M forward: Y = X deq(Wq) + V B for M <= 16 tokens (NF4 dequant-GEMV).
//
// At a few tokens the forward is bound by reading the 4-bit codes once from HBM
// (0.516 B per weight), so the kernel is organised around that stream:
//
//   * Work unit: a 64-column panel of W (one absmax block per row, 32 bytes of
//     codes per row) times a K-range; the grid (panels x K-splits) is sized to be
//     resident at once (two CTAs per SM).  A producer warp streams, with TMA, the
//     panel's codes (256 rows, 8 KB) and the matching 256 columns of X per stage
//     through a 4-stage shared-memory ring; 8 consumer warps each take 2 of the
//     16-row steps of every stage.  The absmax' of every row of the range is
//     computed once up front, so the loop touches no global memory.
//   * Tensor cores, swap-AB: mma.sync m16n8k16 with the weight as the 16 x 16 A
//     operand (rows = 16 output columns, cols = 16 k) and the tokens as the 8-wide
//     B operand.  Lane (g, t) reads one 32-bit word (8 codes) at byte 4g of four of
//     the step's rows; byte j of the words fills tile j (output columns 8g+2j,
//     8g+2j+1).  The k slots of a fragment may hold the step's rows in any order
//     as long as both operands agree, so slots (2t, 2t+1, 2t+8, 2t+9) take rows
//     (t, t+4, t+8, t+12): the four rows of each load are distinct mod 4 and the
//     32 lanes hit 32 banks.  A 256-entry shared table (16 copies, at most 2-way
//     conflicts) maps a code byte to the bf16 pair of its two levels; a
//     byte-permute pairs two rows into an A register.
//   * The block scale is folded into the activations: sum_k x_k (a'_k l_k) =
//     sum_k (x_k a'_k) l_k.  Each consumer warp computes x'[m][k] =
//     bf16(x[m][k] * a'(k, panel)) for its 32 rows of every stage (one row per
//     lane, M/64 multiplies per weight instead of one per weight) into its own
//     shared slice, in the same row order as the k slots; the weight operand is
//     the bf16 NF4 level itself.
//   * Each CTA sums its 8 warps in shared memory and writes one fp32 partial;
//     the last CTA of a panel (atomic ticket in the workspace, reset after use)
//     adds the K-split partials in order, adds V B, and writes bf16 Y.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace qlora {

namespace {

using namespace sm100;

constexpr int kGvConsumers = 8;
constexpr int kGvThreads = (kGvConsumers + 1) * 32;   // + 1 producer warp
constexpr int kPanel = 64;
constexpr int kStageRows = 256;
constexpr int kGvStages = 4;
constexpr uint32_t kCodeBytes = kStageRows * 32;      // codes of one panel
constexpr uint32_t kXBytes = 16 * kStageRows * 2;     // X of up to 16 tokens
constexpr uint32_t kStageBytes = kCodeBytes + kXBytes;
constexpr int kLutCopies = 16;
constexpr int kLutBytes = 256 * kLutCopies * 4;       // 16 copies of the 256-entry table
constexpr int kMaxKc = 4096;

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
  int Kc;                // rows per split (multiple of 256)
  uint32_t* status;
};

__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Position of row rho (0..15) of a 16-row step in the k-slot order.
__device__ __forceinline__ int slot_of_row(int rho) {
  const int a = rho & 3, b = rho >> 2;
  return 2 * a + (b & 1) + 8 * (b >> 1);
}

template <int MT>   // token tiles of 8: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kGvThreads)
nf4_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                const GemvArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;                                                   // kGvStages x (codes, X)
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + kGvStages * kStageBytes);   // [256][16]
  uint16_t* xs_all = reinterpret_cast<uint16_t*>(smem + kGvStages * kStageBytes + kLutBytes);  // [8][16][32]
  float* ascale = reinterpret_cast<float*>(smem + kGvStages * kStageBytes + kLutBytes +
                                           kGvConsumers * 16 * 32 * 2);  // [Kc]
  float* red = reinterpret_cast<float*>(ring);                            // [8][MT*8][64] after the loop
  __shared__ __align__(8) uint64_t bars[2 * kGvStages];
  __shared__ int last;
  constexpr int TM = MT * 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int panel = blockIdx.x, split = blockIdx.y;
  const int64_t k_begin = static_cast<int64_t>(split) * p.Kc;
  const int rows = static_cast<int>(p.K - k_begin < p.Kc ? p.K - k_begin : p.Kc);
  const int nstage = (rows + kStageRows - 1) / kStageRows;
  const int64_t blocks_per_row = p.N / kPanel;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kGvStages);

  if (tid == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kGvConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kGvConsumers) {
    // ------------------------------------------------------------ producer: first ring-full
    // of loads (fresh buffers, no waits), issued before the set-up below
    if (lane == 0) {
      tma_prefetch_desc(&tm_codes);
      tma_prefetch_desc(&tm_x);
      for (int i = 0; i < nstage && i < kGvStages; ++i) {
        const uint32_t dst = smem_addr(ring + i * kStageBytes);
        mbar_arrive_expect_tx(full0 + 8 * i, kCodeBytes + p.M * kStageRows * 2);
        tma_load_2d(dst, &tm_codes, full0 + 8 * i, panel * 32, static_cast<int32_t>(k_begin + i * kStageRows));
        tma_load_2d(dst + kCodeBytes, &tm_x, full0 + 8 * i, static_cast<int32_t>(k_begin + i * kStageRows), 0);
      }
    }
  } else {
    // level pairs of every code byte, 16 copies
    {
      const uint32_t v = pack_bf16x2(c_nf4_level[tid & 15], c_nf4_level[tid >> 4]);
      uint4* dst = reinterpret_cast<uint4*>(lut + tid * kLutCopies);
#pragma unroll
      for (int i = 0; i < kLutCopies / 4; ++i) dst[i] = make_uint4(v, v, v, v);
    }
  }
  // absmax' of this panel's block in every row of the range: every load of a
  // thread is issued before any result is used (rows <= 4096 = 288 x 15 rows)
  {
    constexpr int kPer = (kMaxKc + kGvThreads - 1) / kGvThreads;
    uint8_t qc[kPer];
    float qs[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int kk = tid + u * kGvThreads;
      if (kk < rows) {
        const int64_t b = (k_begin + kk) * blocks_per_row + panel;
        qc[u] = __ldg(p.dq_codes + b);
        qs[u] = __ldg(p.dq_scales + b / kGroup);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int kk = tid + u * kGvThreads;
      if (kk < rows) ascale[kk] = absmax_deq(qc[u], qs[u]);
    }
  }
  __syncthreads();   // level table ready

  float acc[MT][4][4];
#pragma unroll
  for (int a = 0; a < MT; ++a)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][j][c] = 0.0f;

  if (warp == kGvConsumers) {
    // ------------------------------------------------------------ producer: the rest, each
    // stage after the consumers have released its buffer
    if (lane == 0) {
      int issued = nstage < kGvStages ? nstage : kGvStages;
      for (int i = kGvStages; i < nstage; ++i) {
        const int s = i % kGvStages;
        const uint32_t ph = (i / kGvStages) & 1;
        if (!mbar_wait(empty0 + 8 * s, ph ^ 1, p.status, kFlagTimeoutProducer)) break;
        const uint32_t dst = smem_addr(ring + s * kStageBytes);
        mbar_arrive_expect_tx(full0 + 8 * s, kCodeBytes + p.M * kStageRows * 2);
        tma_load_2d(dst, &tm_codes, full0 + 8 * s, panel * 32, static_cast<int32_t>(k_begin + i * kStageRows));
        tma_load_2d(dst + kCodeBytes, &tm_x, full0 + 8 * s, static_cast<int32_t>(k_begin + i * kStageRows), 0);
        issued = i + 1;
      }
      // The ring becomes the reduction buffer below: make sure none of the copies
      // issued last is still in flight (immediate unless a consumer gave up).
      for (int i = issued > kGvStages ? issued - kGvStages : 0; i < issued; ++i)
        mbar_wait(full0 + 8 * (i % kGvStages), (i / kGvStages) & 1, p.status, kFlagTimeoutProducer);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const uint32_t* mylut = lut + (lane & (kLutCopies - 1));
    uint16_t* xs = xs_all + warp * (16 * 32);                // this warp's [token][32 rows] slice
    const int rho = 32 * warp + lane;                        // this lane's row within a stage
    const int pos = (rho & 16) + slot_of_row(rho & 15);      // its place in the warp's slot order
    for (int i = 0; i < nstage; ++i) {
      const int s = i % kGvStages;
      const uint32_t ph = (i / kGvStages) & 1;
      const bool got = mbar_wait(full0 + 8 * s, ph, p.status, kFlagTimeoutMma);
      if (!__all_sync(0xffffffffu, got)) break;
      // x' of this warp's 32 rows of the stage (zero past the end of the range)
      {
        const int kk = i * kStageRows + rho;
        const float a = kk < rows ? ascale[kk] : 0.0f;
        const uint16_t* xt = reinterpret_cast<const uint16_t*>(ring + s * kStageBytes + kCodeBytes);
        for (int m = 0; m < p.M; ++m) {
          const float x = __uint_as_float(static_cast<uint32_t>(xt[m * kStageRows + rho]) << 16);
          xs[m * 32 + pos] = static_cast<uint16_t>(pack_bf16x2(mul_rn(x, a), 0.0f));
        }
      }
      __syncwarp();
      const uint8_t* tile = ring + s * kStageBytes + 4 * g;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int step_row = (2 * warp + h) * 16;          // within the stage
        const int kk0 = i * kStageRows + step_row;         // within the split
        if (kk0 >= rows) break;
        const uint32_t c0 = *reinterpret_cast<const uint32_t*>(tile + (step_row + t) * 32);
        const uint32_t c1 = *reinterpret_cast<const uint32_t*>(tile + (step_row + t + 4) * 32);
        const uint32_t c2 = *reinterpret_cast<const uint32_t*>(tile + (step_row + t + 8) * 32);
        const uint32_t c3 = *reinterpret_cast<const uint32_t*>(tile + (step_row + t + 12) * 32);
        uint32_t bx[MT][2];
#pragma unroll
        for (int a = 0; a < MT; ++a) {
          const bool real = (a * 8 + g) < p.M;
          const uint16_t* xr = xs + (real ? (a * 8 + g) : 0) * 32 + h * 16;
          bx[a][0] = real ? *reinterpret_cast<const uint32_t*>(xr + 2 * t) : 0u;
          bx[a][1] = real ? *reinterpret_cast<const uint32_t*>(xr + 2 * t + 8) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t la = mylut[((c0 >> (8 * j)) & 0xFFu) * kLutCopies];
          const uint32_t lb = mylut[((c1 >> (8 * j)) & 0xFFu) * kLutCopies];
          const uint32_t lc = mylut[((c2 >> (8 * j)) & 0xFFu) * kLutCopies];
          const uint32_t ld = mylut[((c3 >> (8 * j)) & 0xFFu) * kLutCopies];
          const uint32_t a0 = __byte_perm(la, lb, 0x5410);   // even column, slots 2t, 2t+1
          const uint32_t a1 = __byte_perm(la, lb, 0x7632);   // odd column
          const uint32_t a2 = __byte_perm(lc, ld, 0x5410);   // even column, slots 2t+8, 2t+9
          const uint32_t a3 = __byte_perm(lc, ld, 0x7632);
#pragma unroll
          for (int a = 0; a < MT; ++a) mma_bf16_16816(acc[a][j], a0, a1, a2, a3, bx[a][0], bx[a][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
  }
  __syncthreads();   // ring no longer read (every stage issued was consumed); it becomes the reduction buffer

  // D fragment of tile j: (column 8g+2j, tokens 2t, 2t+1) and (column 8g+2j+1, same tokens).
  if (warp < kGvConsumers) {
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
  }
  __syncthreads();
  const int64_t col0 = static_cast<int64_t>(panel) * kPanel;
  if (p.S == 1) {
    for (int e = tid; e < p.M * kPanel; e += kGvThreads) {
      const int m = e / kPanel, n = e % kPanel;
      float y = 0.0f;
#pragma unroll
      for (int w = 0; w < kGvConsumers; ++w) y += red[(w * TM + m) * kPanel + n];
      float vb = 0.0f;
      for (int j = 0; j < p.r; ++j)
        vb = fmaf(__uint_as_float(static_cast<uint32_t>(p.V[m * p.r + j]) << 16),
                  __uint_as_float(static_cast<uint32_t>(p.B[static_cast<int64_t>(j) * p.N + col0 + n]) << 16), vb);
      p.Y[static_cast<int64_t>(m) * p.N + col0 + n] = static_cast<uint16_t>(pack_bf16x2(y + vb, 0.0f));
    }
    return;
  }
  for (int e = tid; e < p.M * kPanel; e += kGvThreads) {
    const int m = e / kPanel, n = e % kPanel;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kGvConsumers; ++w) sum += red[(w * TM + m) * kPanel + n];
    p.part[(static_cast<int64_t>(split) * p.M + m) * p.N + col0 + n] = sum;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last = (atomicAdd(p.tickets + panel, 1u) == static_cast<uint32_t>(p.S - 1));
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
    p.Y[static_cast<int64_t>(m) * p.N + col0 + n] = static_cast<uint16_t>(pack_bf16x2(y + vb, 0.0f));
  }
  if (tid == 0) p.tickets[panel] = 0u;   // ready for the next call
}

// Resident CTAs: each uses at most 112 KB of shared memory, two per SM.
constexpr int kGvResident = 2 * 148;

void gemv_plan(int64_t K, int64_t N, int& S, int& Kc) {
  const int64_t panels = N / kPanel;
  int64_t s = std::max<int64_t>(1, kGvResident / panels);
  s = std::max<int64_t>(s, (K + kMaxKc - 1) / kMaxKc);
  int64_t kc = (K + s - 1) / s;
  kc = (kc + kStageRows - 1) / kStageRows * kStageRows;
  s = (K + kc - 1) / kc;
  S = static_cast<int>(s);
  Kc = static_cast<int>(kc);
}

size_t gemv_smem_bytes(int Kc) {
  return kGvStages * kStageBytes + kLutBytes + static_cast<size_t>(kGvConsumers) * 16 * 32 * 2 +
         4 * static_cast<size_t>(Kc);
}

PFN_cuTensorMapEncodeTiled_v12000 gemv_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

size_t gemv_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  int S, Kc;
  gemv_plan(K, N, S, Kc);
  return S > 1 ? static_cast<size_t>(S) * M * N * 4 : 0;
}

cudaError_t launch_gemv(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B, int64_t M,
                        int r, uint16_t* Y, float* part, uint32_t* tickets, uint32_t* status, cudaStream_t stream) {
  int S, Kc;
  gemv_plan(w.in, w.out, S, Kc);
  // codes as an (in x out/2) byte matrix; box = one 64-column panel (32 bytes) x 256 rows
  CUtensorMap tm;
  auto enc = gemv_encoder();
  if (!enc) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(w.out / 2), static_cast<cuuint64_t>(w.in)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(w.out / 2)};
  cuuint32_t box[2] = {32, kStageRows};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(w.codes), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // X (M x in) bf16: box = 256 columns x M rows
  CUtensorMap tx;
  cuuint64_t xdims[2] = {static_cast<cuuint64_t>(w.in), static_cast<cuuint64_t>(M)};
  cuuint64_t xstrides[1] = {static_cast<cuuint64_t>(w.in * 2)};
  cuuint32_t xbox[2] = {kStageRows, static_cast<cuuint32_t>(M)};
  if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), xdims, xstrides, xbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  GemvArgs a{w.codes, w.dq_codes, w.dq_scales, w.in, w.out, static_cast<int>(M), X, V, B, r, Y, part, tickets,
             S, Kc, status};
  const int MT = M <= 8 ? 1 : 2;
  const size_t smem = gemv_smem_bytes(Kc);
  // the largest dynamic shared memory any plan uses, set once per device
  static bool set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !set[dev]) {
    const int most = static_cast<int>(gemv_smem_bytes(kMaxKc));
    cudaError_t e = cudaFuncSetAttribute(nf4_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(nf4_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  dim3 grid(static_cast<unsigned>(w.out / kPanel), static_cast<unsigned>(S));
  timing_before(QLORA_KERNEL_GEMV, stream);
  if (MT == 1)
    nf4_gemv_kernel<1><<<grid, kGvThreads, smem, stream>>>(tm, tx, a);
  else
    nf4_gemv_kernel<2><<<grid, kGvThreads, smem, stream>>>(tm, tx, a);
  timing_after(QLORA_KERNEL_GEMV, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
