// Rank-r side products of the adapted layer on the tcgen05 tensor cores.
//
//   V  = X A        (M x r)   forward intermediate ("How it works" step 2, (X A) B)
//   U  = dY B^T     (M x r)   backward intermediate
//   dA = X^T U      (in x r)  ("How it works" step 4, dA = dW B^T with dW = X^T dY)
//   dB = V^T dY     (r x out) (dB = A^T dW), computed as dB^T = dY^T V and stored transposed
//
// Each is D (rows x r) = sum_k Aop(rows, k) Bop(r, k) with r <= 64 per pass, bound
// by streaming the big operand (X or dY) from HBM once.  A CTA owns 128 output
// rows and one slice of the reduction: TMA brings 128 x 64 (Aop) and 64 x 64
// (Bop) bf16 tiles into a 3-stage shared-memory ring (128-byte swizzle, K- or
// MN-major as the operand sits in memory; two fit on an SM), one thread issues
// tcgen05.mma into a 128 x r fp32 TMEM accumulator, and four warps move the
// result out.  The reduction is split across CTAs so that the grid holds about
// one CTA per SM; the splits of a row tile form one thread-block cluster.
// Each split stores its TMEM rows straight into the shared memory of the CTA
// that owns those rows (distributed shared memory); after one cluster barrier
// the owners add the splits in order (deterministic, no workspace, no atomics).
// One launch may carry two independent products of the same operand layouts
// (dA and dB, which both reduce over the tokens): the row tiles of the second
// follow those of the first in the grid, and both use the same split count.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace qlora {

namespace {

using namespace sm100;

constexpr int kSkThreads = 192;    // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kSkStages = 3;       // 72 KB ring + 36 KB receive buffer: two CTAs per SM
constexpr int kRowsT = 128;        // output rows per CTA (UMMA M)
constexpr int kKT = 64;            // reduction step
constexpr int kColsT = 64;         // output columns per CTA
constexpr uint32_t kATile = kRowsT * kKT * 2;    // 16 KB
constexpr uint32_t kBTile = kColsT * kKT * 2;    // 8 KB
constexpr uint32_t kSkStage = kATile + kBTile;
constexpr int kRecvRows = kRowsT + kMaxSplits;   // S * ceil(128 / S) rows at most
constexpr uint32_t kRecvBytes = kRecvRows * kColsT * 4;
constexpr uint32_t kSkSmem = kSkStages * kSkStage + kRecvBytes + 1024 + 256;

struct SkArgs {
  int64_t rows;          // output rows
  int r;                 // output columns
  int64_t k_total;       // reduction length
  int64_t k_per_split;   // multiple of 64
  void* out;
  int out_kind;          // 0 = bf16 [row][r], 1 = fp32 [row][r], 2 = fp32 transposed [r][row]
  uint32_t* status;
  int adam;              // out_kind 1 or 2: apply the Adam step instead of storing
  AdamParams ap;
  float scale;           // every value is multiplied by it before the store
  int accumulate;        // out_kind 1 or 2: add to the stored values instead of overwriting
  const uint8_t* keep;   // out_kind 0: dropout keep mask [row][r] (1 = keep), or nullptr
  float keep_scale;      // factor of the kept values (1 / (1 - p))
};

// One Adam / AdamW step of parameter element i with gradient g (fp32, IEEE
// division and square root; see qlora_linear_bwd_adam for the rule).
__device__ __forceinline__ void adam_element(const AdamParams& a, int64_t i, float g) {
  const float th = a.theta[i] * a.decay;
  const float m = fmaf(a.b1, a.m[i], a.omb1 * g);
  const float v = fmaf(a.b2, a.v[i], a.omb2 * (g * g));
  const float den = sqrtf(__fdiv_rn(v, a.bc2)) + a.eps;
  const float th1 = th - a.lr * __fdiv_rn(__fdiv_rn(m, a.bc1), den);
  a.theta[i] = th1;
  a.m[i] = m;
  a.v[i] = v;
  a.p16[i] = static_cast<uint16_t>(pack_bf16x2(th1, 0.0f));
}

__device__ __forceinline__ void store_pair(const SkArgs& p, int64_t row, int col, float v0, float v1) {
  v0 *= p.scale;
  v1 *= p.scale;
  if (p.adam) {
    // dA (in, r): element (row, col); dB (r, out) from dB^T: element (col, row)
    if (p.out_kind == 1) {
      adam_element(p.ap, row * p.r + col, v0);
      adam_element(p.ap, row * p.r + col + 1, v1);
    } else {
      adam_element(p.ap, static_cast<int64_t>(col) * p.rows + row, v0);
      adam_element(p.ap, static_cast<int64_t>(col + 1) * p.rows + row, v1);
    }
    return;
  }
  if (p.out_kind == 0) {
    if (p.keep) {
      const uint8_t* k = p.keep + row * p.r + col;
      v0 *= k[0] ? p.keep_scale : 0.0f;
      v1 *= k[1] ? p.keep_scale : 0.0f;
    }
    *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.out) + row * p.r + col) = pack_bf16x2(v0, v1);
  } else if (p.out_kind == 1) {
    float2* d = reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + row * p.r + col);
    if (p.accumulate) {
      const float2 o = *d;
      v0 += o.x;
      v1 += o.y;
    }
    *d = make_float2(v0, v1);
  } else {
    float* d = reinterpret_cast<float*>(p.out);
    float* d0 = d + static_cast<int64_t>(col) * p.rows + row;
    float* d1 = d + static_cast<int64_t>(col + 1) * p.rows + row;
    if (p.accumulate) {
      v0 += *d0;
      v1 += *d1;
    }
    *d0 = v0;
    *d1 = v1;
  }
}

// A_MN: Aop stored with the row index contiguous (MN-major), else k contiguous.
// B_MN: Bop stored with the column index contiguous (MN-major), else k contiguous.
// Row tiles [0, rt0) compute product 0 (tm_a0, tm_b0, p0), the rest product 1.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kSkThreads, 2)
skinny_tc_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
                 const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
                 const __grid_constant__ SkArgs p0, const __grid_constant__ SkArgs p1, const int rt0) {
  const bool second = static_cast<int>(blockIdx.x) >= rt0;
  const SkArgs& p = second ? p1 : p0;
  const CUtensorMap* tm_a = second ? &tm_a1 : &tm_a0;
  const CUtensorMap* tm_b = second ? &tm_b1 : &tm_b0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* recv = reinterpret_cast<float*>(smem + kSkStages * kSkStage);       // [S][cap][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSkStages * kSkStage + kRecvBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kSkStages + 1);
  const uint32_t full0 = smem_addr(bars), free0 = smem_addr(bars + kSkStages);
  const uint32_t tmem_full = smem_addr(bars + 2 * kSkStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(second ? static_cast<int>(blockIdx.x) - rt0 : blockIdx.x) * kRowsT;
  const int split = blockIdx.y;
  const int col0 = blockIdx.z * kColsT;
  const int cols = min(kColsT, p.r - col0);
  const int n_mma = (cols + 15) / 16 * 16;
  const int64_t kbeg = split * p.k_per_split;
  const int64_t kend = min(p.k_total, kbeg + p.k_per_split);
  const int nkb = kend > kbeg ? static_cast<int>((kend - kbeg + kKT - 1) / kKT) : 0;
  // the splits of this row tile are the CTAs of the cluster (rank = split)
  const int S = static_cast<int>(gridDim.y);
  const int cap = (kRowsT + S - 1) / S;   // rows owned by each split

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(free0 + 8 * s, 1);
    }
    mbar_init(tmem_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 64);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tm_a);
    tma_prefetch_desc(tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent: the set-up above overlaps the kernel
  // before; nothing in global memory is touched until that kernel has finished.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kSkStages;
        const uint32_t ph = (kb / kSkStages) & 1;
        if (!mbar_wait(free0 + 8 * s, ph ^ 1, p.status, kFlagTimeoutProducer)) break;
        const uint32_t a_dst = smem_addr(smem + s * kSkStage), b_dst = a_dst + kATile;
        const uint32_t bar = full0 + 8 * s;
        const int32_t k0 = static_cast<int32_t>(kbeg + kb * kKT);
        mbar_arrive_expect_tx(bar, kSkStage);
        if (!A_MN) {
          tma_load_2d(a_dst, tm_a, bar, k0, static_cast<int32_t>(row0));
        } else {
          tma_load_2d(a_dst, tm_a, bar, static_cast<int32_t>(row0), k0);
          tma_load_2d(a_dst + 8192, tm_a, bar, static_cast<int32_t>(row0 + 64), k0);
        }
        if (!B_MN) tma_load_2d(b_dst, tm_b, bar, k0, col0);
        else tma_load_2d(b_dst, tm_b, bar, col0, k0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, n_mma, A_MN, B_MN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kSkStages;
        const uint32_t ph = (kb / kSkStages) & 1;
        if (!mbar_wait(full0 + 8 * s, ph, p.status, kFlagTimeoutMma)) break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + s * kSkStage), b_base = a_base + kATile;
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b_base + kk * 32, 16, 1024);
          umma_bf16(tmem_base, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(free0 + 8 * s);
      }
      umma_commit(tmem_full);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const bool ok =
        __all_sync(0xffffffffu, nkb == 0 || mbar_wait(tmem_full, 0, p.status, kFlagTimeoutEpilogue));
    tc_fence_after();
    const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
    const int rl = quarter * 32 + lane;            // row within the tile
    const int64_t row = row0 + rl;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    // the owner of this row and this split's slot in the owner's receive buffer
    const int owner = rl / cap;
    const uint32_t dst =
        S > 1 ? mapa_shared(smem_addr(recv) + static_cast<uint32_t>(((split * cap + rl - owner * cap) * kColsT) * 4),
                            static_cast<uint32_t>(owner))
              : 0u;
#pragma unroll 1
    for (int c = 0; c < n_mma; c += 16) {
      uint32_t v[16];
      if (ok && nkb > 0) {
        // load and wait in one statement: the registers are valid only after the wait
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
            "tcgen05.wait::ld.sync.aligned;"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15])
            : "r"(taddr + c)
            : "memory");
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0u;   // an empty slice contributes zeros
      }
      if (S == 1) {
        if (row < p.rows) {
#pragma unroll
          for (int i = 0; i < 16; i += 2)
            if (c + i < cols) store_pair(p, row, col0 + c + i, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; i += 4)   // cols is a multiple of 8
          if (c + i < cols)
            st_shared_cluster_v4(dst + static_cast<uint32_t>((c + i) * 4),
                                 make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                             __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 64);
  }
  if (S == 1) return;

  // ------------------------------------------------------------ split reduction
  cluster_sync();   // every split's rows have landed in their owners' buffers
  const int r_begin = split * cap, r_end = min(kRowsT, r_begin + cap);
  const int pairs = cols / 2;
  for (int e = threadIdx.x; e < (r_end - r_begin) * pairs; e += kSkThreads) {
    const int slot = e / pairs, cc = 2 * (e - slot * pairs);
    const int64_t row = row0 + r_begin + slot;
    if (row >= p.rows) continue;
    float v0 = 0.0f, v1 = 0.0f;
    for (int sp = 0; sp < S; ++sp) {
      const float2 x = *reinterpret_cast<const float2*>(recv + (sp * cap + slot) * kColsT + cc);
      v0 += x.x;
      v1 += x.y;
    }
    store_pair(p, row, col0 + cc, v0, v1);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// bf16 row-major (rows x cols) -> tensor map with a (box_cols x box_rows) box, 128B swizzle.
bool bf16_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTAs of one launch: one per SM.  Two fit on an SM, so the next rank-r launch
// (a programmatic dependent) is resident and waiting while this one drains.  The
// launch of dA with dB, which a GEMM or the next call follows, takes two per SM
// (twice the splits): one linear's forward + backward at M = 2048 ran 1.2% faster
// (4096 x 4096: 130.2 against 131.9 us; 4096 x 11008: 311.8 against 315.5 us).
constexpr int kResident = 148;

struct Plan {
  int splits;
  int64_t kps;
  dim3 grid;
};

// Split count for one product (rows x r, reduction k_total) or two of the same
// rank and reduction length (rows1 > 0): as many reduction slices as give one
// CTA per SM (kResident), each slice at least two K-steps long.
Plan plan(int64_t rows, int r, int64_t k_total, int64_t rows1 = 0, int resident = kResident) {
  const int64_t rt = (rows + kRowsT - 1) / kRowsT + (rows1 + kRowsT - 1) / kRowsT;
  const int ct = (r + kColsT - 1) / kColsT;
  const int64_t ktiles = (k_total + kKT - 1) / kKT;
  int64_t s = resident / (rt * ct);
  s = std::min<int64_t>(s, std::max<int64_t>(1, ktiles / 2));
  s = std::max<int64_t>(1, std::min<int64_t>(s, kMaxSplits));
  const int64_t kps = (ktiles + s - 1) / s * kKT;
  s = (k_total + kps - 1) / kps;
  return Plan{static_cast<int>(s), kps, dim3(static_cast<unsigned>(rt), static_cast<unsigned>(s), ct)};
}

// One product of the launch: its operand maps and what is stored where.
struct Product {
  CUtensorMap ta, tb;
  int64_t rows;
  void* out;
  int out_kind;
  const AdamParams* adam;
  float scale;
  Dropout drop;
};

// Launch product x (and product y, if given: same rank r and reduction k_total).
template <bool A_MN, bool B_MN>
cudaError_t run(const Product& x, const Product* y, int r, int64_t k_total, uint32_t* status, cudaStream_t stream,
                bool accumulate, int resident = kResident) {
  static bool set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(skinny_tc_kernel<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSkSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(skinny_tc_kernel<A_MN, B_MN>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  const Plan pl = plan(x.rows, r, k_total, y ? y->rows : 0, resident);
  auto args = [&](const Product& q) {
    return SkArgs{q.rows, r, k_total, pl.kps, q.out, q.out_kind, status, q.adam ? 1 : 0,
                  q.adam ? *q.adam : AdamParams{}, q.scale, accumulate ? 1 : 0, q.drop.keep, q.drop.keep_scale};
  };
  const SkArgs a0 = args(x), a1 = y ? args(*y) : a0;
  const int rt0 = static_cast<int>((x.rows + kRowsT - 1) / kRowsT);
  const Product& yy = y ? *y : x;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = pl.grid;
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = kSkSmem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = static_cast<unsigned>(pl.splits);
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  timing_before(QLORA_KERNEL_RANK_R, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, skinny_tc_kernel<A_MN, B_MN>, x.ta, x.tb, yy.ta, yy.tb, a0, a1, rt0);
  timing_after(QLORA_KERNEL_RANK_R, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

// V = X A: Aop = X (M x in, k contiguous); Bop[j][k] = A[k][j] (j contiguous).
cudaError_t launch_xa(const uint16_t* X, const uint16_t* A, int64_t M, int64_t n_in, int r, uint16_t* V,
                      uint32_t* status, cudaStream_t stream, float scale, Dropout drop) {
  Product x{};
  if (!bf16_map(&x.ta, X, M, n_in, 64, 128) || !bf16_map(&x.tb, A, n_in, r, 64, 64)) return cudaErrorInvalidValue;
  x.rows = M;
  x.out = V;
  x.out_kind = 0;
  x.scale = scale;
  x.drop = drop;
  return run<false, true>(x, nullptr, r, n_in, status, stream, false);
}

// U = dY B^T: Aop = dY (M x out, k contiguous); Bop = B (r x out, k contiguous).
cudaError_t launch_dybt(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t n_out, int r, uint16_t* U,
                        uint32_t* status, cudaStream_t stream, float scale, Dropout drop) {
  Product x{};
  if (!bf16_map(&x.ta, dY, M, n_out, 64, 128) || !bf16_map(&x.tb, B, r, n_out, 64, 64)) return cudaErrorInvalidValue;
  x.rows = M;
  x.out = U;
  x.out_kind = 0;
  x.scale = scale;
  x.drop = drop;
  return run<false, false>(x, nullptr, r, n_out, status, stream, false);
}

// dB^T = dY^T V: Aop[o][m] = dY[m][o] (o contiguous); Bop[j][m] = V[m][j]; stored as dB (r x out).
// dA = X^T U: Aop[i][m] = X[m][i] (i contiguous); Bop[j][m] = U[m][j] (j contiguous).
// Both reduce over the M tokens, so they share one launch: dB's row tiles first.
cudaError_t launch_dbda(const uint16_t* V, const uint16_t* dY, const uint16_t* X, const uint16_t* U, int64_t M,
                        int64_t n_in, int64_t n_out, int r, float* dA, float* dB, uint32_t* status,
                        cudaStream_t stream, const AdamParams* adam_a, const AdamParams* adam_b, bool accumulate) {
  Product b{}, a{};
  if (!bf16_map(&b.ta, dY, M, n_out, 64, 64) || !bf16_map(&b.tb, V, M, r, 64, 64) ||
      !bf16_map(&a.ta, X, M, n_in, 64, 64) || !bf16_map(&a.tb, U, M, r, 64, 64))
    return cudaErrorInvalidValue;
  b.rows = n_out;
  b.out = dB;
  b.out_kind = 2;
  b.adam = adam_b;
  b.scale = 1.0f;
  a.rows = n_in;
  a.out = dA;
  a.out_kind = 1;
  a.adam = adam_a;
  a.scale = 1.0f;
  return run<true, true>(b, &a, r, M, status, stream, accumulate, 2 * kResident);
}

}  // namespace qlora
