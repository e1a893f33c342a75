// Symmetric uniform integer quantisation with one scale per 16 weights, the
// base quantiser of the pages' own simulation ("QLoRA (low-rank adapters on a
// quantized model)", "The code, line by line": symmetric uniform integers, one
// scale per 16 consecutive entries of the flattened (in, out) matrix;
// "Simplifications": no NF4, no double quantisation; "What the simulations
// show": 2, 3 and 4 bits, "2-bit" being ternary {-s, 0, s}).
//
//   per group of 16:  s = fl32(max |w| / Q),  Q = 2^(b-1) - 1,
//                     q = clamp(rint(fl32(w / s)), -Q, Q)  (ties to even; 0 when s = 0),
//   stored as the nibble q + 8 (element 2k in the low nibble of byte k), s as fp32;
//   w' = fl32(q s).
//
// Both kernels stream: one thread per group (64 bytes of fp32 in, 8 bytes of
// codes and 4 bytes of scale out, or the reverse), so a warp reads 2 KB and writes
// 256 + 128 contiguous bytes.  IEEE division (__fdiv_rn) decides each code, as the
// reading fixes; the quantiser is a one-time pass over the weight.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kIqThreads = 256;

__global__ void __launch_bounds__(kIqThreads)
int_quantize_kernel(const float4* __restrict__ W0, int64_t ngroups, float qmax, uint2* __restrict__ codes,
                    float* __restrict__ scales) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * kIqThreads + threadIdx.x;
  if (g >= ngroups) return;
  float w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = W0[g * 4 + i];
    w[4 * i] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
  const float s = __fdiv_rn(a, qmax);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float q = 0.0f;
    if (s > 0.0f) q = fminf(fmaxf(rintf(__fdiv_rn(w[i], s)), -qmax), qmax);
    const uint32_t c = static_cast<uint32_t>(static_cast<int>(q) + 8);
    if (i < 8) lo |= c << (4 * i);
    else hi |= c << (4 * (i - 8));
  }
  codes[g] = make_uint2(lo, hi);
  scales[g] = s;
}

template <bool kBf16>
__global__ void __launch_bounds__(kIqThreads)
int_dequantize_kernel(const uint2* __restrict__ codes, const float* __restrict__ scales, int64_t ngroups,
                      void* __restrict__ out) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * kIqThreads + threadIdx.x;
  if (g >= ngroups) return;
  const uint2 c = codes[g];
  const float s = scales[g];
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t word = i < 8 ? c.x : c.y;
    const int q = static_cast<int>((word >> (4 * (i & 7))) & 0xFu) - 8;
    v[i] = mul_rn(static_cast<float>(q), s);
  }
  if (kBf16) {
    uint4* o = reinterpret_cast<uint4*>(out) + g * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      o[h] = make_uint4(pack_bf16x2(v[8 * h], v[8 * h + 1]), pack_bf16x2(v[8 * h + 2], v[8 * h + 3]),
                        pack_bf16x2(v[8 * h + 4], v[8 * h + 5]), pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
  } else {
    float4* o = reinterpret_cast<float4*>(out) + g * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

}  // namespace

cudaError_t launch_int_quantize(const float* W0, int64_t n, int bits, uint8_t* codes, float* scales,
                                cudaStream_t stream) {
  const int64_t ngroups = n / 16;
  if (ngroups == 0) return cudaSuccess;
  const float qmax = static_cast<float>((1 << (bits - 1)) - 1);
  const unsigned grid = static_cast<unsigned>((ngroups + kIqThreads - 1) / kIqThreads);
  timing_before(QLORA_KERNEL_QUANTIZE, stream);
  int_quantize_kernel<<<grid, kIqThreads, 0, stream>>>(reinterpret_cast<const float4*>(W0), ngroups, qmax,
                                                       reinterpret_cast<uint2*>(codes), scales);
  timing_after(QLORA_KERNEL_QUANTIZE, stream);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_int_dequantize(const uint8_t* codes, const float* scales, int64_t n, bool bf16, void* out,
                                  cudaStream_t stream) {
  const int64_t ngroups = n / 16;
  if (ngroups == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((ngroups + kIqThreads - 1) / kIqThreads);
  timing_before(QLORA_KERNEL_DEQUANTIZE, stream);
  if (bf16)
    int_dequantize_kernel<true><<<grid, kIqThreads, 0, stream>>>(reinterpret_cast<const uint2*>(codes), scales,
                                                                 ngroups, out);
  else
    int_dequantize_kernel<false><<<grid, kIqThreads, 0, stream>>>(reinterpret_cast<const uint2*>(codes), scales,
                                                                  ngroups, out);
  timing_after(QLORA_KERNEL_DEQUANTIZE, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
