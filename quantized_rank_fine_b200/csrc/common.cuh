// Shared device helpers and format constants of libqlora (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/qlora.h"

namespace qlora {

constexpr int kBlock = QLORA_BLOCK;   // weights per absmax block
constexpr int kGroup = QLORA_GROUP;   // absmax values per fp32 scale

// The 16 NF4 levels as binary32, ascending (code = index).  They are the normal
// quantiles of the QLoRA construction ("What QLoRA adds over LoRA": 16 levels at
// quantiles of a standard normal; "LoRA & QLoRA", NF4 value table): 8 positive
// quantiles at evenly spaced probabilities from (31/32 + 29/30)/2 down to 1/2
// (exclusive), 7 negated ones at 7 such probabilities, and 0, all divided by the
// largest quantile, each rounded once to binary32.
__host__ __device__ constexpr float nf4_level(int i) {
  constexpr float kLevels[16] = {
      -0x1.000000p+0f, -0x1.647362p-1f, -0x1.0cd65cp-1f, -0x1.94653cp-2f,
      -0x1.234496p-2f, -0x1.7a6a7ap-3f, -0x1.74f0d2p-4f, 0.0f,
      0x1.45f602p-4f,  0x1.4995bep-3f,  0x1.f809b4p-3f,  0x1.5a066cp-2f,
      0x1.c3496ap-2f,  0x1.200f52p-1f,  0x1.722760p-1f,  0x1.000000p+0f};
  return kLevels[i];
}

// Decision thresholds of the nearest-level search: t_j is the midpoint
// (l_j + l_{j+1}) / 2 rounded DOWN to binary32.  For any binary32 x,
// x > t_j  <=>  x > the exact midpoint, so code = #{j : x > t_j} is the exact
// argmin with ties to the lower level.
__host__ __device__ constexpr float nf4_threshold(int j) {
  constexpr float kThr[15] = {
      -0x1.b239b2p-1f, -0x1.38a4e0p-1f, -0x1.d708fap-2f, -0x1.5bd4eap-2f,
      -0x1.e079d4p-3f, -0x1.1a7172p-3f, -0x1.74f0d2p-5f, 0x1.45f602p-5f,
      0x1.ec90bep-4f,  0x1.a0cfb8p-3f,  0x1.2b05a2p-2f,  0x1.8ea7eap-2f,
      0x1.00da02p-1f,  0x1.491b58p-1f,  0x1.b913b0p-1f};
  return kThr[j];
}

// Copies of the two tables for run-time indices in device code: indexing the
// constexpr arrays above with a run-time value makes every thread build its own
// copy in local memory.
static __constant__ float c_nf4_level[16] = {
    nf4_level(0), nf4_level(1), nf4_level(2),  nf4_level(3),  nf4_level(4),  nf4_level(5),
    nf4_level(6), nf4_level(7), nf4_level(8),  nf4_level(9),  nf4_level(10), nf4_level(11),
    nf4_level(12), nf4_level(13), nf4_level(14), nf4_level(15)};
static __constant__ float c_nf4_threshold[15] = {
    nf4_threshold(0), nf4_threshold(1), nf4_threshold(2),  nf4_threshold(3),  nf4_threshold(4),
    nf4_threshold(5), nf4_threshold(6), nf4_threshold(7),  nf4_threshold(8),  nf4_threshold(9),
    nf4_threshold(10), nf4_threshold(11), nf4_threshold(12), nf4_threshold(13), nf4_threshold(14)};

// ---------------------------------------------------------------- numerics

// IEEE binary32 product with no contraction into an FMA.
__device__ __forceinline__ float mul_rn(float a, float b) { return __fmul_rn(a, b); }

// E4M3 byte -> float (exact: every E4M3 value is a half-precision normal).
__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}

// Dequantised block absmax: fl32(e4m3(c) * s), or fl32(c * s) when the absmax
// codes are linear uint8 (u8; the same for every thread of a launch).
__device__ __forceinline__ float absmax_deq(uint8_t c, float s, bool u8) {
  return mul_rn(u8 ? static_cast<float>(c) : e4m3_to_float(c), s);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // RNE each
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ---------------------------------------------------------------- error flag

// Bits of the status word at the start of a workspace.
enum : uint32_t {
  kFlagTimeoutProducer = 1u << 0,
  kFlagTimeoutMma = 1u << 1,
  kFlagTimeoutEpilogue = 1u << 2,
  kFlagTimeoutSelftest = 1u << 3,
};

__device__ __forceinline__ void raise_flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

}  // namespace qlora
