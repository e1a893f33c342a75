// NF4 blockwise quantisation with double-quantised absmax, one pass over W0.
//
// What it computes ("LLMs · QLoRA" blockwise quantiser; "What QLoRA adds over
// LoRA" NF4 + double quantisation; "LoRA & QLoRA" "Double Quantization"):
//   per block of 64 consecutive weights:  a = max |w|,  x = fl32(w / a),
//     code = index of the nearest NF4 level (ties to the lower level);
//   per group of 256 consecutive blocks:  s = fl32(max a / 448),
//     dq_code = E4M3_RNE_satfinite(fl32(a / s))   (0 when s = 0).
//
// Layout: a persistent grid, one 512-thread CTA per SM, walks the groups (16,384
// weights = 64 KB of fp32 each).  A bulk asynchronous copy streams each group
// into one of three 64 KB shared-memory buffers, two groups ahead of the one
// being encoded, so HBM is read continuously with no thread involvement.  Warp w
// owns blocks 16w .. 16w+15 of a group, 8 at a time; lane l serves a quarter (16
// consecutive weights) of block l/4, reading its four 16-byte chunks in a
// rotated order so that the 8 lanes of each quarter-warp hit 8 different bank
// groups.  The block absmax needs a 2-step shuffle and each lane stores its 16
// codes as one 8-byte word (a warp writes 256 contiguous bytes).  HBM traffic
// per weight: 4 B read + 0.5 B codes + 1/64 B dq code + 4/16384 B scale.
//
// Division.  x must be the correctly rounded quotient.  The fast path multiplies
// by the correctly rounded reciprocal of a (|q - x| <= 3 * 2^-24 for |x| <= 1)
// and only when q lies within 2^-20 of the decision threshold it is compared
// with does it fall back to the IEEE division __fdiv_rn.  Away from a threshold
// q and x select the same code, so the codes equal those of the exact division.
//
// Nearest level.  A 65-cell table over [-1, 1] holds, per cell, the one
// threshold inside it (thresholds are >= 0.08 apart; 2.0 when none) with the
// number of thresholds below the cell stored in its 4 low mantissa bits: one
// 32-bit shared-memory word per lookup.  Cell k = round(32 v + 32) is read off
// the bits of one fused multiply-add with a 1.5 * 2^23 offset; no threshold lies
// within 2.3e-4 of a cell edge.  The 4 borrowed bits move a threshold by at most
// 15 ulp (< 2^-20); together with |q - x| <= 3 * 2^-24, any q farther than 2^-19
// from the stored threshold is on the same side as the exact x of the exact
// threshold.  A lane whose 16 values include one closer than that (rare) redoes
// all 16 with IEEE division and a direct count over the 15 thresholds.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qlora {

namespace {

constexpr int kQThreads = 512;
constexpr int kQWarps = kQThreads / 32;
constexpr int kQBuf = 3;                              // groups in flight
constexpr uint32_t kGroupBytes = kGroup * kBlock * 4; // 64 KB of fp32
constexpr int kCells = 65;
constexpr float kRoundBase = 12582912.0f;            // 1.5 * 2^23: integers land in the low bits

// Fast code of q; sets `near` when q is within 2^-19 of the cell's threshold.
__device__ __forceinline__ uint32_t fast_code(float q, const uint32_t* __restrict__ lut, bool& near) {
  const float f = fmaf(q, 32.0f, 32.0f + kRoundBase);
  // q is in [-1, 1] up to rounding, so the cell is in [0, 64]; the clamp keeps the
  // table read in bounds for any input.
  const uint32_t k = min(static_cast<uint32_t>(__float_as_int(f) - __float_as_int(kRoundBase)),
                         static_cast<uint32_t>(kCells - 1));
  const uint32_t e = lut[k];
  const float thr = __uint_as_float(e);
  near |= fabsf(q - thr) < 0x1p-19f;
  return (e & 0xFu) + (q > thr ? 1u : 0u);
}

// Exact code of the correctly rounded quotient x: the number of thresholds below x.
__device__ __forceinline__ uint32_t exact_code(float w, float a) {
  const float x = (a > 0.0f) ? __fdiv_rn(w, a) : 0.0f;
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < 15; ++j) c += (x > nf4_threshold(j)) ? 1u : 0u;
  return c;
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return a | (b << 4) | (c << 8) | (d << 12);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__global__ void __launch_bounds__(kQThreads, 1)
quantize_nf4_kernel(const float* __restrict__ W0, int64_t nblocks, int64_t ngroups, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ dq_codes, float* __restrict__ dq_scales) {
  extern __shared__ __align__(128) uint8_t qsmem[];
  __shared__ uint32_t lut[kCells];
  __shared__ float amax[kGroup];
  __shared__ float red[8];
  __shared__ __align__(8) uint64_t bars[kQBuf];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t buf0 = sm100::smem_addr(qsmem), bar0 = sm100::smem_addr(bars);
  if (tid < kCells) {
    const float lo = -1.0f + (tid - 0.5f) * (1.0f / 32.0f);
    const float hi = lo + (1.0f / 32.0f);
    uint32_t base = 0;
    float thr = 2.0f;
#pragma unroll
    for (int j = 0; j < 15; ++j) {
      const float t = nf4_threshold(j);
      base += (t < lo) ? 1u : 0u;
      if (t >= lo && t < hi) thr = t;
    }
    lut[tid] = (__float_as_uint(thr) & ~0xFu) | base;
  }
  if (tid == 0) {
    for (int b = 0; b < kQBuf; ++b) sm100::mbar_init(bar0 + 8 * b, 1);
    sm100::fence_mbar_init();
    for (int b = 0; b < kQBuf; ++b) {
      const int64_t g = blockIdx.x + static_cast<int64_t>(b) * gridDim.x;
      if (g >= ngroups) break;
      const int64_t nb = min(static_cast<int64_t>(kGroup), nblocks - g * kGroup);
      const uint32_t bytes = static_cast<uint32_t>(nb * kBlock * 4);
      sm100::mbar_arrive_expect_tx(bar0 + 8 * b, bytes);
      bulk_load(buf0 + b * kGroupBytes, W0 + g * kGroup * kBlock, bytes, bar0 + 8 * b);
    }
  }
  __syncthreads();

  const int quarter = lane & 3;            // which 16 weights of its block
  const int bsub = lane >> 2;              // block among the 8 of an iteration
  // rotated chunk order: the 8 lanes of a quarter-warp read 8 different 16-byte bank groups
  const int rot = (quarter >> 1) + 2 * (bsub & 1);
  int64_t i = 0, failed_at = -1;
  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x, ++i) {
    const int b = static_cast<int>(i % kQBuf);
    const uint32_t ph = static_cast<uint32_t>((i / kQBuf) & 1);
    const bool got = sm100::mbar_wait(bar0 + 8 * b, ph, nullptr, 0);
    if (!__syncthreads_and(got)) {
      failed_at = i;
      break;
    }
    const int64_t blk0 = g * kGroup;
    const int nblk = static_cast<int>(nblocks - blk0 < kGroup ? nblocks - blk0 : kGroup);
    const float* gs = reinterpret_cast<const float*>(qsmem + b * kGroupBytes);

#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int lb = warp * 16 + it * 8 + bsub;
      float4 v[4];
      int ci[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        ci[c] = (c + rot) & 3;
        v[c] = (lb < nblk) ? *reinterpret_cast<const float4*>(gs + lb * kBlock + quarter * 16 + 4 * ci[c])
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float m = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v[c].x), fabsf(v[c].y)), fmaxf(fabsf(v[c].z), fabsf(v[c].w))));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (lb < nblk) {
        float rcp = (m > 0.0f) ? __frcp_rn(m) : 0.0f;
        bool near = !(rcp <= 3.0e38f);     // a subnormal absmax: exact path only
        if (near) rcp = 0.0f;
        uint32_t c4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          c4[c] = pack4(fast_code(__fmul_rn(v[c].x, rcp), lut, near), fast_code(__fmul_rn(v[c].y, rcp), lut, near),
                        fast_code(__fmul_rn(v[c].z, rcp), lut, near), fast_code(__fmul_rn(v[c].w, rcp), lut, near));
        if (near) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            c4[c] = pack4(exact_code(v[c].x, m), exact_code(v[c].y, m), exact_code(v[c].z, m), exact_code(v[c].w, m));
        }
        uint64_t word = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) word |= static_cast<uint64_t>(c4[c]) << (16 * ci[c]);
        *reinterpret_cast<uint2*>(codes + (blk0 + lb) * (kBlock / 2) + quarter * 8) =
            make_uint2(static_cast<uint32_t>(word), static_cast<uint32_t>(word >> 32));
        if (quarter == 0) amax[lb] = m;
      }
    }
    __syncthreads();   // buffer b fully read; absmax of the group in shared memory
    if (tid == 0) {
      const int64_t gn = g + static_cast<int64_t>(kQBuf) * gridDim.x;
      if (gn < ngroups) {
        const int64_t nb = min(static_cast<int64_t>(kGroup), nblocks - gn * kGroup);
        const uint32_t bytes = static_cast<uint32_t>(nb * kBlock * 4);
        sm100::mbar_arrive_expect_tx(bar0 + 8 * b, bytes);
        bulk_load(buf0 + b * kGroupBytes, W0 + gn * kGroup * kBlock, bytes, bar0 + 8 * b);
      }
    }

    // Group maximum of the block absmax values (threads 0..255).
    if (tid < kGroup) {
      float gm = (tid < nblk) ? amax[tid] : 0.0f;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
      if (lane == 0) red[warp] = gm;
    }
    __syncthreads();
    if (tid < kGroup) {
      float gm = red[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) gm = fmaxf(gm, red[w]);
      const float sc = __fdiv_rn(gm, 448.0f);
      if (tid < nblk) {
        uint8_t c = 0;
        if (sc > 0.0f) {
          const float y = __fdiv_rn(amax[tid], sc);
          c = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
        }
        dq_codes[blk0 + tid] = c;
      }
      if (tid == 0) dq_scales[g] = sc;
    }
    __syncthreads();   // amax and red reused by the next group
  }
  // A wait that gave up leaves up to kQBuf copies in flight into this CTA's
  // shared memory: wait for them (again bounded) before the CTA exits.
  if (failed_at >= 0 && tid == 0) {
    for (int64_t j = failed_at; j < failed_at + kQBuf; ++j) {
      if (blockIdx.x + j * gridDim.x >= ngroups) break;
      sm100::mbar_wait(bar0 + 8 * static_cast<int>(j % kQBuf), static_cast<uint32_t>((j / kQBuf) & 1), nullptr, 0);
    }
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_quantize_nf4(const float* W0, int64_t n, uint8_t* codes, uint8_t* dq_codes,
                                float* dq_scales, cudaStream_t stream) {
  const int64_t nblocks = n / kBlock;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  if (ngroups == 0) return cudaSuccess;
  static bool set[64] = {};
  static int sms[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(quantize_nf4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kQBuf * kGroupBytes));
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  const int64_t grid = std::min<int64_t>(ngroups, dev < 64 ? sms[dev] : 148);
  timing_before(QLORA_KERNEL_QUANTIZE, stream);
  quantize_nf4_kernel<<<static_cast<unsigned>(grid), kQThreads, kQBuf * kGroupBytes, stream>>>(
      W0, nblocks, ngroups, codes, dq_codes, dq_scales);
  timing_after(QLORA_KERNEL_QUANTIZE, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
