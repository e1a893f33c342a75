// Fused NF4-dequant GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM).
//
//   forward  Y  = [X | V] . [deq(Wq) ; B]      (M x out, K = in + r)
//   dX       dX = [dY | U] . [deq(Wq)^T ; A^T] (M x in,  K = out + r)
//
// ("How it works" steps 2-4 and "What QLoRA adds over LoRA" of "QLoRA (low-rank
// adapters on a quantized model)": the frozen weight is dequantised to bf16 for
// each matmul; the adapter product (X A) B, and U A^T in the backward, is the
// same contraction extended by r along K, so it lands in the same accumulator.)
//
// CTA tile 256 (M) x 256 (N), K step 64, 3-stage shared-memory ring, one CTA per
// SM.  Two UMMA M=128 x N=256 accumulators fill the 512 TMEM columns; both use
// the same dequantised weight tile, so each weight is dequantised M/256 times.
// Warp roles (320 threads):
//   warp 0     TMA producer: per K-step the activation tile (256 x 64 bf16,
//              128B swizzle) and the packed codes of the weight tile (8 KB); for
//              the adapter K-steps the V/U tile and the B/A tile instead.
//   warp 1     TMEM allocation + the single thread that issues tcgen05.mma.
//   warps 2-9  dequant producers (one thread per 64-weight block per K-step):
//              codes from shared memory -> per-block 16-entry bf16 table ->
//              byte-permute lookup -> 16-byte stores in the UMMA canonical
//              layout; then the epilogue (TMEM -> registers -> bf16 -> global).
// Barriers per stage: `loaded` (TMA bytes), `ready` (8 dequant warps, after the
// weight tile is written) and `free` (tcgen05.commit once the MMAs have read it).
// The weight tile is written MN-major for the forward (N contiguous in W) and
// K-major for dX (K contiguous in W), so the dequant never transposes.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace qlora {

namespace {

using namespace sm100;

constexpr int kBM = 256, kBN = 256, kBK = 64, kStages = 3;
constexpr int kThreads = 320;
constexpr int kDeqWarps = 8;
constexpr uint32_t kABytes = kBM * kBK * 2;     // 32 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;     // 32 KB
constexpr uint32_t kCBytes = kBN * kBK / 2;     // 8 KB of packed codes
constexpr uint32_t kStageBytes = kABytes + kBBytes + kCBytes;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
  const uint8_t* codes;
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t w_out;      // columns of the stored weight (out)
  int64_t M, N, K;    // output M x N, weight reduction length K (multiple of 64)
  int r;
  uint16_t* D;        // bf16 (M, N)
  uint32_t* status;
};

// Per-block table: v_j = bf16(fl32(level_j * a)) for j = 0..15, split into the
// low bytes (lo[0..3]) and high bytes (hi[0..3]) of the 16 entries, 4 per word.
struct BlockLut {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ BlockLut make_lut(float a) {
  uint32_t pr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    pr[i] = pack_bf16x2(mul_rn(nf4_level(2 * i), a), mul_rn(nf4_level(2 * i + 1), a));
  BlockLut t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x6420);
    t.hi[q] = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x7531);
  }
  return t;
}

// Four 4-bit codes (nibbles of x, element order low to high) -> two bf16x2 words.
__device__ __forceinline__ void lut4(const BlockLut& t, uint32_t x, uint32_t& o01, uint32_t& o23) {
  const uint32_t s_lo = x & 0x7777u;                              // index within a half table
  const uint32_t s_pick = 0x3210u | ((x >> 1) & 0x4444u);         // +4 where the code is >= 8
  const uint32_t lo = __byte_perm(__byte_perm(t.lo[0], t.lo[1], s_lo),
                                  __byte_perm(t.lo[2], t.lo[3], s_lo), s_pick);
  const uint32_t hi = __byte_perm(__byte_perm(t.hi[0], t.hi[1], s_lo),
                                  __byte_perm(t.hi[2], t.hi[3], s_lo), s_pick);
  o01 = __byte_perm(lo, hi, 0x5140);
  o23 = __byte_perm(lo, hi, 0x7362);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

template <bool kDX>
__global__ void __launch_bounds__(kThreads, 1)
nf4_gemm_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_ext_a,
                const __grid_constant__ CUtensorMap tm_ext_b, const __grid_constant__ CUtensorMap tm_codes,
                const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 1);
  const uint32_t loaded0 = smem_addr(bars), ready0 = smem_addr(bars + kStages);
  const uint32_t free0 = smem_addr(bars + 2 * kStages), tmem_full = smem_addr(bars + 3 * kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
  const int nkb_w = static_cast<int>(p.K / kBK);
  const int n_ext = (p.r + kBK - 1) / kBK;
  const int nkb = nkb_w + n_ext;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(loaded0 + 8 * s, 1);
      mbar_init(ready0 + 8 * s, kDeqWarps);
      mbar_init(free0 + 8 * s, 1);
    }
    mbar_init(tmem_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_ext_a);
    tma_prefetch_desc(&tm_ext_b);
    tma_prefetch_desc(&tm_codes);
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
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        if (!mbar_wait(free0 + 8 * s, ph ^ 1, p.status, kFlagTimeoutProducer)) break;
        const uint32_t a_dst = smem_addr(smem + s * kStageBytes);
        const uint32_t b_dst = a_dst + kABytes;
        const uint32_t c_dst = b_dst + kBBytes;
        const uint32_t bar = loaded0 + 8 * s;
        if (kb < nkb_w) {
          mbar_arrive_expect_tx(bar, kABytes + kCBytes);
          tma_load_2d(a_dst, &tm_act, bar, kb * kBK, static_cast<int32_t>(m0));
          if (!kDX) tma_load_2d(c_dst, &tm_codes, bar, static_cast<int32_t>(n0 / 2), kb * kBK);
          else tma_load_2d(c_dst, &tm_codes, bar, kb * (kBK / 2), static_cast<int32_t>(n0));
        } else {
          const int j = kb - nkb_w;
          mbar_arrive_expect_tx(bar, kABytes + kBBytes);
          tma_load_2d(a_dst, &tm_ext_a, bar, j * kBK, static_cast<int32_t>(m0));
          if (!kDX) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              tma_load_2d(b_dst + i * 8192, &tm_ext_b, bar, static_cast<int32_t>(n0 + 64 * i), j * kBK);
          } else {
            tma_load_2d(b_dst, &tm_ext_b, bar, j * kBK, static_cast<int32_t>(n0));
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 256, false, !kDX);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        if (!mbar_wait(ready0 + 8 * s, ph, p.status, kFlagTimeoutMma)) break;
        if (!mbar_wait(loaded0 + 8 * s, ph, p.status, kFlagTimeoutMma)) break;
        tc_fence_after();
        int nk16 = 4;
        if (kb >= nkb_w) nk16 = min(4, (p.r - (kb - nkb_w) * kBK + 15) / 16);
        const uint32_t a_base = smem_addr(smem + s * kStageBytes);
        const uint32_t b_base = a_base + kABytes;
        for (int kk = 0; kk < nk16; ++kk) {
          const uint64_t bdesc = kDX ? smem_desc_sw128(b_base + kk * 32, 16, 1024)
                                     : smem_desc_sw128(b_base + kk * 2048, 8192, 1024);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t adesc = smem_desc_sw128(a_base + h * 16384 + kk * 32, 16, 1024);
            umma_bf16(tmem_base + h * 256, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit(free0 + 8 * s);
      }
      umma_commit(tmem_full);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant producers
    const int t = threadIdx.x - 64;                 // 0..255: one 64-weight block each
    const int64_t blocks_per_row = p.w_out / kBlock;
    int64_t blk;                                    // block index at kb = 0
    bool valid;
    uint32_t row_off;                               // byte offset of this thread's 8 chunks (weight tile)
    uint32_t code_off0, code_off1;                  // byte offsets of its two 16-byte code chunks
    int swz;
    if (!kDX) {
      // Quarter-warps (8 lanes) take 8 consecutive k rows of one 64-wide n block,
      // so their 16-byte stores fall in 8 distinct bank groups.
      const int kr = (t & 7) + ((t >> 5) << 3), j = (t >> 3) & 3;
      valid = (n0 + 64 * j) < p.N;
      blk = static_cast<int64_t>(kr) * blocks_per_row + (n0 >> 6) + j;
      row_off = j * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128;
      swz = kr & 7;
      // codes tile: 64 rows of 128 bytes, 128-byte swizzle
      code_off0 = kr * 128 + (((2 * j) ^ (kr & 7)) << 4);
      code_off1 = kr * 128 + (((2 * j + 1) ^ (kr & 7)) << 4);
    } else {
      const int nr = t;
      valid = (n0 + nr) < p.N;
      blk = (n0 + nr) * blocks_per_row;
      row_off = nr * 128;
      swz = nr & 7;
      // codes tile: 256 rows of 32 bytes, 32-byte swizzle
      const int x = (nr >> 2) & 1;
      code_off0 = nr * 32 + ((0 ^ x) << 4);
      code_off1 = nr * 32 + ((1 ^ x) << 4);
    }
    // K-step kb moves the block index by 64 rows (forward) or 1 block (dX).
    const int64_t blk_step = kDX ? 1 : 64 * blocks_per_row;

    // absmax codes and scales, two K-steps ahead
    uint8_t dqc0 = 0, dqc1 = 0;
    float dqs0 = 0.0f, dqs1 = 0.0f;
    if (valid && nkb_w > 0) {
      dqc0 = __ldg(p.dq_codes + blk);
      dqs0 = __ldg(p.dq_scales + blk / kGroup);
    }
    if (valid && nkb_w > 1) {
      dqc1 = __ldg(p.dq_codes + blk + blk_step);
      dqs1 = __ldg(p.dq_scales + (blk + blk_step) / kGroup);
    }
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (kb / kStages) & 1;
      // every lane waits; the warp leaves the loop together if the wait gave up
      const bool got = mbar_wait(loaded0 + 8 * s, ph, p.status, kFlagTimeoutProducer);
      if (!__all_sync(0xffffffffu, got)) break;
      if (kb < nkb_w) {
        const uint32_t stage = smem_addr(smem + s * kStageBytes);
        const uint32_t dst = stage + kABytes + row_off;
        const uint32_t csrc = stage + kABytes + kBBytes;
        uint32_t w[8];
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(csrc + code_off0));
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]) : "r"(csrc + code_off1));
        const BlockLut lut = make_lut(valid ? absmax_deq(dqc0, dqs0) : 0.0f);
        dqc0 = dqc1;
        dqs0 = dqs1;
        if (valid && kb + 2 < nkb_w) {
          const int64_t nb = blk + (kb + 2) * blk_step;
          dqc1 = __ldg(p.dq_codes + nb);
          dqs1 = __ldg(p.dq_scales + nb / kGroup);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o0, o1, o2, o3;
          lut4(lut, w[c] & 0xFFFFu, o0, o1);
          lut4(lut, w[c] >> 16, o2, o3);
          st_shared_v4(dst + ((c ^ swz) << 4), o0, o1, o2, o3);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(ready0 + 8 * s);
    }

    // ------------------------------------------------------------ epilogue
    const bool ok = __all_sync(0xffffffffu, mbar_wait(tmem_full, 0, p.status, kFlagTimeoutEpilogue));
    tc_fence_after();
    if (ok) {
      const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
      const int half = (warp - 2) >> 2;             // which M=128 accumulator
      const int64_t row = m0 + half * 128 + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 256;
#pragma unroll 1
      for (int cb = 0; cb < kBN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + cb * 32, v);
        tmem_ld_wait();
        const int64_t col = n0 + cb * 32;
        if (row < p.M && col < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(p.D + row * p.N + col);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
            dst[q] = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// Row-major matrix (rows x cols elements of `esize` bytes) -> 2-D tensor map with
// a (box_cols x box_rows) box; box_cols * esize must not exceed the swizzle span.
bool make_map_t(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows,
                CUtensorMapDataType dtype, int esize, CUtensorMapSwizzle swizzle) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult rc = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

// bf16 matrix, 128-byte swizzle (box_cols <= 64).
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  return make_map_t(m, base, rows, cols, box_cols, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool kDX>
cudaError_t launch_gemm(const CUtensorMap& act, const CUtensorMap& ea, const CUtensorMap& eb, const CUtensorMap& cm,
                        const GemmArgs& a, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nf4_gemm_kernel<kDX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((a.N + kBN - 1) / kBN), static_cast<unsigned>((a.M + kBM - 1) / kBM));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const int which = kDX ? QLORA_KERNEL_DX_GEMM : QLORA_KERNEL_FWD_GEMM;
  timing_before(which, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, nf4_gemm_kernel<kDX>, act, ea, eb, cm, a);
  timing_after(which, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

// Y = X deq(W) + V B.
cudaError_t launch_fwd_gemm(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B,
                            int64_t M, int r, uint16_t* Y, uint32_t* status, cudaStream_t stream) {
  CUtensorMap act, ea, eb, cm;
  // codes as a (in x out/2) byte matrix: 64 rows x 128 bytes per K-step, 128-byte swizzle
  if (!make_map(&act, X, M, w.in, 64, 256) || !make_map(&ea, V, M, r, 64, 256) ||
      !make_map(&eb, B, r, w.out, 64, 64) ||
      !make_map_t(&cm, w.codes, w.in, w.out / 2, 128, 64, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmArgs a{w.codes, w.dq_codes, w.dq_scales, w.out, M, w.out, w.in, r, Y, status};
  return launch_gemm<false>(act, ea, eb, cm, a, stream);
}

// dX = dY deq(W)^T + U A^T.
cudaError_t launch_dx_gemm(const WeightView& w, const uint16_t* dY, const uint16_t* U, const uint16_t* A,
                           int64_t M, int r, uint16_t* dX, uint32_t* status, cudaStream_t stream) {
  CUtensorMap act, ea, eb, cm;
  // codes as a (in x out/2) byte matrix: 256 rows x 32 bytes per K-step, 32-byte swizzle
  if (!make_map(&act, dY, M, w.out, 64, 256) || !make_map(&ea, U, M, r, 64, 256) ||
      !make_map(&eb, A, w.in, r, 64, 256) ||
      !make_map_t(&cm, w.codes, w.in, w.out / 2, 32, 256, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  GemmArgs a{w.codes, w.dq_codes, w.dq_scales, w.out, M, w.in, w.out, r, dX, status};
  return launch_gemm<true>(act, ea, eb, cm, a, stream);
}

}  // namespace qlora
