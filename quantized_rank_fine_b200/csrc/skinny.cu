// Rank-r side products of the adapted layer.
//
//   V  = X A        (M x r)   forward intermediate ("How it works" step 2, (X A) B)
//   U  = dY B^T     (M x r)   backward intermediate
//   dA = X^T U      (in x r)  ("How it works" step 4, dA = dW B^T with dW = X^T dY)
//   dB = V^T dY     (r x out) (dB = A^T dW)
//
// Each is a contraction with one side only r (<= 64 per pass) wide, so the
// kernels are bound by reading the big operand (X or dY) once from HBM; the
// reduction dimension (in/out for V/U, the M tokens for dA/dB) is split across
// CTAs so that even small M fills the 148 SMs, with fp32 partial sums written to
// the workspace and a second kernel adding the splits in a fixed order
// (deterministic results).  Tiles are 64 x 64 bf16 staged by cp.async into
// 128-byte-swizzled shared memory and consumed with ldmatrix + mma.sync
// m16n8k16 (bf16 in, fp32 accumulate).
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kSkThreads = 128;    // 4 warps, 16 output rows each
constexpr int kTile = 64;          // rows/cols of a staged tile
constexpr int kTileBytes = kTile * kTile * 2;

// One operand of the contraction as it sits in global memory: element
// (row, col) at base[row * ld + col]; rows >= nrows or cols >= ncols read as 0.
// The reduction index k runs along rows when k_on_rows, else along columns.
struct Operand {
  const uint16_t* base;
  int64_t ld;
  int64_t nrows, ncols;
  bool k_on_rows;
  int64_t fixed0;   // origin of the non-k dimension for this CTA
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Stage the 64x64 tile of `op` whose k-origin is k0 into swizzled smem.
__device__ __forceinline__ void load_tile(const Operand& op, int64_t k0, uint8_t* smem) {
  const int64_t r0 = op.k_on_rows ? k0 : op.fixed0;
  const int64_t c0 = op.k_on_rows ? op.fixed0 : k0;
  const uint32_t s = smem_u32(smem);
#pragma unroll
  for (int i = 0; i < (kTile * 8) / kSkThreads; ++i) {
    const int e = threadIdx.x + i * kSkThreads;
    const int row = e >> 3, chunk = e & 7;
    const int64_t gr = r0 + row, gc = c0 + chunk * 8;
    const bool valid = (gr < op.nrows) && (gc < op.ncols);
    const uint16_t* src = valid ? op.base + gr * op.ld + gc : op.base;
    cp_async16(s + swz(row, chunk), src, valid);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C (64 x RC) += Aop (64 x K) * Bop (K x RC) over this CTA's k-range.
//   Aop stored [m][k] (a_trans = false) or [k][m] (a_trans = true).
//   Bop stored [n][k] (b_trans = false) or [k][n] (b_trans = true).
// Output: fp32 partial at part[(split * out_rows + row) * out_ld + col], or,
// with a single split, the final value (bf16 or fp32, optionally transposed).
struct SkinnyArgs {
  Operand a, b;
  int64_t k_begin, k_per_split, k_total;
  int64_t out_rows;       // rows of C (M, or in/out for the weight gradients)
  int r;                  // columns of C
  float* part;            // fp32 partials [splits][out_rows][r] (splits > 1)
  void* out;              // final output when splits == 1
  int out_kind;           // 0 = bf16 [row][r], 1 = fp32 [row][r], 2 = fp32 transposed [r][row]
  int splits;
};

template <bool kATrans, bool kBTrans>
__global__ void __launch_bounds__(kSkThreads)
skinny_mma_kernel(SkinnyArgs p) {
  __shared__ __align__(128) uint8_t smem[2][2][kTileBytes];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.y;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int j0 = blockIdx.z * kTile;

  Operand A = p.a, B = p.b;
  A.fixed0 = m0;
  B.fixed0 = j0;
  const int64_t kb = p.k_begin + split * p.k_per_split;
  const int64_t ke = min(p.k_total, kb + p.k_per_split);
  const int nk = ke > kb ? static_cast<int>((ke - kb + kTile - 1) / kTile) : 0;

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  const int ntile = min(8, (p.r - j0 + 7) / 8);   // n8 tiles that hold real columns

  if (nk > 0) {
    load_tile(A, kb, smem[0][0]);
    load_tile(B, kb, smem[0][1]);
    cp_async_commit();
  }
  for (int t = 0; t < nk; ++t) {
    const int cur = t & 1;
    if (t + 1 < nk) {
      load_tile(A, kb + (t + 1) * kTile, smem[cur ^ 1][0]);
      load_tile(B, kb + (t + 1) * kTile, smem[cur ^ 1][1]);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sa = smem_u32(smem[cur][0]);
    const uint32_t sb = smem_u32(smem[cur][1]);
#pragma unroll
    for (int ks = 0; ks < kTile; ks += 16) {
      uint32_t af[4];
      const int mi = warp * 16;
      if (!kATrans) {
        const int row = mi + (lane & 15), chunk = (ks >> 3) + (lane >> 4);
        ldsm_x4(sa + swz(row, chunk), af[0], af[1], af[2], af[3]);
      } else {
        const int q = lane >> 3;
        const int row = ks + (lane & 7) + ((q >> 1) << 3), chunk = (mi >> 3) + (q & 1);
        ldsm_x4_t(sa + swz(row, chunk), af[0], af[1], af[2], af[3]);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {          // pairs of n8 tiles
        if (2 * np >= ntile) break;
        uint32_t b0, b1, b2, b3;
        const int q = lane >> 3;
        if (!kBTrans) {
          // matrices: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
          const int row = np * 16 + (lane & 7) + ((q >> 1) << 3), chunk = (ks >> 3) + (q & 1);
          ldsm_x4(sb + swz(row, chunk), b0, b1, b2, b3);
        } else {
          // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
          const int row = ks + (lane & 7) + ((q & 1) << 3), chunk = np * 2 + (q >> 1);
          ldsm_x4_t(sb + swz(row, chunk), b0, b1, b2, b3);
        }
        mma_bf16(acc[2 * np], af, b0, b1);
        if (2 * np + 1 < ntile) mma_bf16(acc[2 * np + 1], af, b2, b3);
      }
    }
    __syncthreads();
  }

  // Epilogue: c0,c1 -> (row g, cols 2t, 2t+1); c2,c3 -> (row g+8, same cols).
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    if (nt >= ntile) break;
    const int col = j0 + nt * 8 + 2 * tq;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = m0 + warp * 16 + g + 8 * h;
      if (row >= p.out_rows) continue;
      const float v0 = acc[nt][2 * h], v1 = acc[nt][2 * h + 1];
      if (p.splits > 1) {
        float* d = p.part + (static_cast<int64_t>(split) * p.out_rows + row) * p.r + col;
        *reinterpret_cast<float2*>(d) = make_float2(v0, v1);
      } else if (p.out_kind == 0) {
        uint16_t* d = reinterpret_cast<uint16_t*>(p.out) + row * p.r + col;
        *reinterpret_cast<uint32_t*>(d) = pack_bf16x2(v0, v1);
      } else if (p.out_kind == 1) {
        float* d = reinterpret_cast<float*>(p.out) + row * p.r + col;
        *reinterpret_cast<float2*>(d) = make_float2(v0, v1);
      } else {
        float* d = reinterpret_cast<float*>(p.out);
        d[static_cast<int64_t>(col) * p.out_rows + row] = v0;
        d[static_cast<int64_t>(col + 1) * p.out_rows + row] = v1;
      }
    }
  }
}

// Sum the split partials in split order and write the final layout.
__global__ void reduce_splits_kernel(const float* __restrict__ part, int splits, int64_t rows, int r,
                                     void* __restrict__ out, int out_kind) {
  const int64_t n = rows * r;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int k = 0; k < splits; ++k) s += part[k * n + i];
    if (out_kind == 0) {
      reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(s);
    } else if (out_kind == 1) {
      reinterpret_cast<float*>(out)[i] = s;
    } else {
      const int64_t row = i / r, col = i % r;
      reinterpret_cast<float*>(out)[col * rows + row] = s;
    }
  }
}

constexpr int kTargetCtas = 2 * 148;

int choose_splits(int64_t base_ctas, int64_t k_total) {
  const int64_t ktiles = (k_total + kTile - 1) / kTile;
  int64_t s = (kTargetCtas + base_ctas - 1) / base_ctas;
  s = std::min<int64_t>(s, std::max<int64_t>(1, ktiles / 2));
  s = std::min<int64_t>(s, kMaxSplits);
  return static_cast<int>(std::max<int64_t>(1, s));
}

cudaError_t run_skinny(bool a_trans, bool b_trans, const Operand& a, const Operand& b,
                       int64_t k_total, int64_t out_rows, int r, void* out, int out_kind,
                       float* part, cudaStream_t stream) {
  const int64_t mt = (out_rows + kTile - 1) / kTile;
  const int rt = (r + kTile - 1) / kTile;
  const int splits = choose_splits(mt * rt, k_total);
  int64_t kps = (k_total + splits - 1) / splits;
  kps = (kps + kTile - 1) / kTile * kTile;
  SkinnyArgs p{a, b, 0, kps, k_total, out_rows, r, part, out, out_kind, splits};
  dim3 grid(static_cast<unsigned>(mt), splits, rt);
  timing_before(QLORA_KERNEL_RANK_R, stream);
  if (!a_trans && b_trans) skinny_mma_kernel<false, true><<<grid, kSkThreads, 0, stream>>>(p);
  else if (!a_trans && !b_trans) skinny_mma_kernel<false, false><<<grid, kSkThreads, 0, stream>>>(p);
  else if (a_trans && b_trans) skinny_mma_kernel<true, true><<<grid, kSkThreads, 0, stream>>>(p);
  else skinny_mma_kernel<true, false><<<grid, kSkThreads, 0, stream>>>(p);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && splits > 1) {
    const int64_t n = out_rows * r;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 4 * 148));
    reduce_splits_kernel<<<blocks, 256, 0, stream>>>(part, splits, out_rows, r, out, out_kind);
    count_launch();
    e = cudaGetLastError();
  }
  timing_after(QLORA_KERNEL_RANK_R, stream);
  return e;
}

}  // namespace

size_t skinny_partial_floats(int64_t out_rows, int r, int64_t k_total) {
  const int64_t mt = (out_rows + kTile - 1) / kTile;
  const int rt = (r + kTile - 1) / kTile;
  const int splits = choose_splits(mt * rt, k_total);
  return splits > 1 ? static_cast<size_t>(splits) * out_rows * r : 0;
}

// V = X A: X (M, in) row-major [m][k]; A (in, r) row-major [k][j].
cudaError_t launch_xa(const uint16_t* X, const uint16_t* A, int64_t M, int64_t n_in, int r,
                      uint16_t* V, float* part, cudaStream_t stream) {
  Operand a{X, n_in, M, n_in, false, 0};
  Operand b{A, r, n_in, r, true, 0};
  return run_skinny(false, true, a, b, n_in, M, r, V, 0, part, stream);
}

// U = dY B^T: dY (M, out) [m][k]; B (r, out) row-major = [j][k].
cudaError_t launch_dybt(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t n_out, int r,
                        uint16_t* U, float* part, cudaStream_t stream) {
  Operand a{dY, n_out, M, n_out, false, 0};
  Operand b{B, n_out, r, n_out, false, 0};
  return run_skinny(false, false, a, b, n_out, M, r, U, 0, part, stream);
}

// dA = X^T U (in, r): A-operand X stored [k = token][m = in]; U stored [k][j].
cudaError_t launch_xtu(const uint16_t* X, const uint16_t* U, int64_t M, int64_t n_in, int r,
                       float* dA, float* part, cudaStream_t stream) {
  Operand a{X, n_in, M, n_in, true, 0};
  Operand b{U, r, M, r, true, 0};
  return run_skinny(true, true, a, b, M, n_in, r, dA, 1, part, stream);
}

// dB = V^T dY (r, out), computed as dB^T = dY^T V (out, r) and stored transposed.
cudaError_t launch_vtdy(const uint16_t* V, const uint16_t* dY, int64_t M, int64_t n_out, int r,
                        float* dB, float* part, cudaStream_t stream) {
  Operand a{dY, n_out, M, n_out, true, 0};
  Operand b{V, r, M, r, true, 0};
  return run_skinny(true, true, a, b, M, n_out, r, dB, 2, part, stream);
}

}  // namespace qlora
