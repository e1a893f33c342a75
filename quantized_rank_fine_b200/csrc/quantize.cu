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
// owning 32 consecutive blocks handled 8 at a time.  A warp-wide 128-bit load
// covers 512 contiguous bytes (two blocks, one per half-warp), so every load
// instruction is fully coalesced; the block absmax is a 4-step shuffle reduction
// inside each half-warp.  HBM traffic per weight: 4 B read + 0.5 B codes +
// 1/64 B dq code + 4/16384 B scale.
//
// Division.  x must be the correctly rounded quotient.  The fast path multiplies
// by the correctly rounded reciprocal of a (|q - x| <= 3 * 2^-24 for |x| <= 1)
// and only when q lies within 2^-20 of the decision threshold it is compared
// with does it fall back to the IEEE division __fdiv_rn.  Away from a threshold
// q and x select the same code, so the codes equal those of the exact division.
//
// Nearest level.  A 65-cell table over [-1, 1] (cells of width 1/32) holds, per
// cell, the number of thresholds below the cell and the one threshold inside it
// (at most one: thresholds are >= 0.08 apart); no threshold lies within 0.0016 of
// a cell edge, so rounding in the cell index never changes the count.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kQThreads = 256;
constexpr int kCells = 65;

struct CellEntry {
  float thr;   // threshold inside the cell, or 2 (none)
  int base;    // thresholds strictly below the cell's lower edge
};

__device__ __forceinline__ int nf4_code_from(float v, const CellEntry* __restrict__ lut,
                                             float& dist) {
  int k = __float2int_rd(fmaf(v, 32.0f, 32.0f));
  k = min(max(k, 0), kCells - 1);
  CellEntry e = lut[k];
  dist = fabsf(v - e.thr);
  return e.base + (v > e.thr ? 1 : 0);
}

__device__ __forceinline__ int encode_one(float w, float a, float rcp, bool fast_ok,
                                          const CellEntry* __restrict__ lut) {
  float dist;
  int code = nf4_code_from(__fmul_rn(w, rcp), lut, dist);
  if (!fast_ok || dist < 0x1p-20f) {
    float x = (a > 0.0f) ? __fdiv_rn(w, a) : 0.0f;
    code = nf4_code_from(x, lut, dist);
  }
  return code;
}

__global__ void __launch_bounds__(kQThreads)
quantize_nf4_kernel(const float* __restrict__ W0, int64_t nblocks, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ dq_codes, float* __restrict__ dq_scales) {
  __shared__ CellEntry lut[kCells];
  __shared__ float amax[kGroup];
  __shared__ float red[kQThreads / 32];

  const int tid = threadIdx.x;
  if (tid < kCells) {
    const float lo = -1.0f + tid * (1.0f / 32.0f);
    const float hi = lo + (1.0f / 32.0f);
    int base = 0;
    float thr = 2.0f;
#pragma unroll
    for (int j = 0; j < 15; ++j) {
      const float t = nf4_threshold(j);
      base += (t < lo) ? 1 : 0;
      if (t >= lo && t < hi) thr = t;
    }
    lut[tid] = CellEntry{thr, base};
  }
  __syncthreads();

  const int64_t g = blockIdx.x;
  const int64_t blk0 = g * kGroup;
  const int nblk = static_cast<int>(nblocks - blk0 < kGroup ? nblocks - blk0 : kGroup);
  const int warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4;            // which block of a pair this lane serves

  // Each warp: blocks [warp*32, warp*32+32) of the group, 8 per iteration.
  float4 v[4][4];
#pragma unroll
  for (int it = 0; it < 4; ++it) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int lb = warp * 32 + it * 8 + 2 * i + half;   // block within the group
      if (lb < nblk) {
        const int64_t off = (blk0 + lb) * kBlock + (lane & 15) * 4;
        v[it][i] = __ldcs(reinterpret_cast<const float4*>(W0 + off));
      } else {
        v[it][i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }

#pragma unroll
  for (int it = 0; it < 4; ++it) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int lb = warp * 32 + it * 8 + 2 * i + half;
      const float4 q = v[it][i];
      float m = fmaxf(fmaxf(fabsf(q.x), fabsf(q.y)), fmaxf(fabsf(q.z), fabsf(q.w)));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lb < nblk) {
        const float rcp = (m > 0.0f) ? __frcp_rn(m) : 0.0f;
        const bool fast_ok = (rcp <= 3.0e38f);            // false for a subnormal absmax
        const uint32_t c0 = encode_one(q.x, m, rcp, fast_ok, lut);
        const uint32_t c1 = encode_one(q.y, m, rcp, fast_ok, lut);
        const uint32_t c2 = encode_one(q.z, m, rcp, fast_ok, lut);
        const uint32_t c3 = encode_one(q.w, m, rcp, fast_ok, lut);
        const uint16_t packed = static_cast<uint16_t>(c0 | (c1 << 4) | (c2 << 8) | (c3 << 12));
        const int64_t byte = ((blk0 + lb) * kBlock + (lane & 15) * 4) >> 1;
        *reinterpret_cast<uint16_t*>(codes + byte) = packed;
        if ((lane & 15) == 0) amax[lb] = m;
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
