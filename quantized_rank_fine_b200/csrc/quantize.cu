// NF4 blockwise quantisation with double-quantised absmax, one pass over W0.
//
// What it computes ("LLMs · QLoRA" blockwise quantiser; "What QLoRA adds over
// LoRA" NF4 + double quantisation; "LoRA & QLoRA" "Double Quantization"):
//   per block of 64 consecutive weights:  a = max |w|,  x = fl32(w / a),
//     code = index of the nearest NF4 level (ties to the lower level);
//   per group of 256 consecutive blocks:  s = fl32(max a / 448),
//     dq_code = E4M3_RNE_satfinite(fl32(a / s))   (0 when s = 0).
//
// Layout: one CTA per group (16,384 weights = 64 KB of fp32), 8 warps, each warp
// owning 32 consecutive blocks handled 8 at a time: lane l serves a quarter (16
// consecutive weights) of block l/4, so the block absmax needs only a 2-step
// shuffle and each lane stores its 16 codes as one 8-byte word (a warp writes
// 256 contiguous bytes).  All 64 weights of a lane's four iterations are loaded
// before any is used.  HBM traffic per weight: 4 B read + 0.5 B codes + 1/64 B dq
// code + 4/16384 B scale.
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

namespace qlora {

namespace {

constexpr int kQThreads = 256;
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

__global__ void __launch_bounds__(kQThreads, 3)
quantize_nf4_kernel(const float* __restrict__ W0, int64_t nblocks, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ dq_codes, float* __restrict__ dq_scales) {
  __shared__ uint32_t lut[kCells];
  __shared__ float amax[kGroup];
  __shared__ float red[kQThreads / 32];

  const int tid = threadIdx.x;
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

  const int64_t g = blockIdx.x;
  const int64_t blk0 = g * kGroup;
  const int nblk = static_cast<int>(nblocks - blk0 < kGroup ? nblocks - blk0 : kGroup);
  const int warp = tid >> 5, lane = tid & 31;
  const int quarter = lane & 3;           // which 16 weights of the block
  __syncthreads();                         // cell table ready

#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float4 v[2][4];
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int lb = warp * 32 + (2 * half + it) * 8 + (lane >> 2);
      const float4* src = reinterpret_cast<const float4*>(W0 + (blk0 + lb) * kBlock + quarter * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v[it][i] = (lb < nblk) ? __ldcs(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int lb = warp * 32 + (2 * half + it) * 8 + (lane >> 2);
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v[it][i].x), fabsf(v[it][i].y)), fmaxf(fabsf(v[it][i].z), fabsf(v[it][i].w))));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (lb < nblk) {
        float rcp = (m > 0.0f) ? __frcp_rn(m) : 0.0f;
        bool near = !(rcp <= 3.0e38f);     // a subnormal absmax: exact path only
        if (near) rcp = 0.0f;
        uint32_t c[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          c[4 * i + 0] = fast_code(__fmul_rn(v[it][i].x, rcp), lut, near);
          c[4 * i + 1] = fast_code(__fmul_rn(v[it][i].y, rcp), lut, near);
          c[4 * i + 2] = fast_code(__fmul_rn(v[it][i].z, rcp), lut, near);
          c[4 * i + 3] = fast_code(__fmul_rn(v[it][i].w, rcp), lut, near);
        }
        if (near) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            c[4 * i + 0] = exact_code(v[it][i].x, m);
            c[4 * i + 1] = exact_code(v[it][i].y, m);
            c[4 * i + 2] = exact_code(v[it][i].z, m);
            c[4 * i + 3] = exact_code(v[it][i].w, m);
          }
        }
        const uint32_t lo = pack4(c[0], c[1], c[2], c[3]) | (pack4(c[4], c[5], c[6], c[7]) << 16);
        const uint32_t hi = pack4(c[8], c[9], c[10], c[11]) | (pack4(c[12], c[13], c[14], c[15]) << 16);
        *reinterpret_cast<uint2*>(codes + (blk0 + lb) * (kBlock / 2) + quarter * 8) = make_uint2(lo, hi);
        if (quarter == 0) amax[lb] = m;
      }
    }
  }
  __syncthreads();

  // Group maximum of the block absmax values.
  float gm = (tid < nblk) ? amax[tid] : 0.0f;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
  if (lane == 0) red[warp] = gm;
  __syncthreads();
  gm = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) gm = fmaxf(gm, red[w]);

  const float s = __fdiv_rn(gm, 448.0f);
  if (tid < nblk) {
    uint8_t c = 0;
    if (s > 0.0f) {
      const float y = __fdiv_rn(amax[tid], s);
      c = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
    }
    dq_codes[blk0 + tid] = c;
  }
  if (tid == 0) dq_scales[g] = s;
}

}  // namespace

cudaError_t launch_quantize_nf4(const float* W0, int64_t n, uint8_t* codes, uint8_t* dq_codes,
                                float* dq_scales, cudaStream_t stream) {
  const int64_t nblocks = n / kBlock;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  if (ngroups == 0) return cudaSuccess;
  timing_before(QLORA_KERNEL_QUANTIZE, stream);
  quantize_nf4_kernel<<<static_cast<unsigned>(ngroups), kQThreads, 0, stream>>>(
      W0, nblocks, codes, dq_codes, dq_scales);
  timing_after(QLORA_KERNEL_QUANTIZE, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
