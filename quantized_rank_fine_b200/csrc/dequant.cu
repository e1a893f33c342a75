// Dense dequantisation and adapter merge of the frozen NF4 weight.
//
// dequantize ("LLMs · QLoRA": levels[idx] * scale; "What QLoRA adds over LoRA":
// absmax quantised to 8 bits, weights dequantised to bf16):
//   a'_b = fl32(e4m3(dq_code_b) * s_g) (or fl32(dq_code_b * s_g) for linear
//   uint8 absmax codes),  w' = fl32(level[code] * a'_b); for the INT16 format
//   (qlora_quantize_int) w' = fl32((code - 8) * s) with one scale per 16 weights,
//   written as fp32 or as bf16(w').  Plain binary32 products, no FMA contraction,
//   so the result is bit-exact.
// merge ("QLoRA (low-rank adapters on a quantized model)", "How it works" step 5):
//   W = w' + A B with fp32 accumulation over the rank.
// LoftQ-style initialisation (same page, "Going further": start A and B from an
// SVD of W0 - Q(W0)): the quantisation residual R = fl32(W0 - w'), one mode of
// the dequantisation kernel; and the symmetric split of a caller's rank-r SVD
// U diag(S) Vh into the adapters, A = bf16(fl32(U fl32(sqrt S))) and
// B = bf16(fl32(fl32(sqrt S) Vh)).
//
// Both are HBM-bound streaming kernels: each thread handles 16 consecutive
// weights (8 code bytes, one 64-byte fp32 or 32-byte bf16 output run), so every
// warp reads 256 contiguous code bytes and writes 2 KB (fp32) contiguously.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kDqThreads = 256;

// Output of the dequantisation kernel: fp32 w', bf16(w'), or the residual
// fl32(W0 - w') of the weight W0 the codes were quantised from.
enum DqMode { kDqF32 = 0, kDqBf16 = 1, kDqResidual = 2 };

template <int kMode>
__global__ void __launch_bounds__(kDqThreads)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ dq_codes,
                  const float* __restrict__ dq_scales, int64_t n16, void* __restrict__ out, int fmt,
                  const float* __restrict__ W0) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = fmt == kFmtInt16 ? static_cast<float>(static_cast<int>(threadIdx.x) - 8)
                                                           : nf4_level(threadIdx.x);
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDqThreads + threadIdx.x;
  if (t >= n16) return;
  const int64_t blk = t >> 2;                       // 4 threads per 64-weight block
  const float a = fmt == kFmtInt16 ? dq_scales[t]   // one scale per 16 weights
                                   : absmax_deq(dq_codes[blk], dq_scales[blk / kGroup], fmt == kFmtU8);
  const uint2 c = __ldcs(reinterpret_cast<const uint2*>(codes) + t);
  float w[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t word = (i < 4) ? c.x : c.y;
    const uint32_t byte = (word >> (8 * (i & 3))) & 0xFFu;
    w[2 * i] = mul_rn(lv[byte & 0xF], a);
    w[2 * i + 1] = mul_rn(lv[byte >> 4], a);
  }
  if constexpr (kMode == kDqResidual) {
    const float4* w0 = reinterpret_cast<const float4*>(W0) + 4 * t;
    float4* o = reinterpret_cast<float4*>(out) + 4 * t;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcs(w0 + i);
      __stcs(o + i, make_float4(__fsub_rn(v.x, w[4 * i]), __fsub_rn(v.y, w[4 * i + 1]),
                                __fsub_rn(v.z, w[4 * i + 2]), __fsub_rn(v.w, w[4 * i + 3])));
    }
  } else if constexpr (kMode == kDqBf16) {
    uint4* o = reinterpret_cast<uint4*>(out) + 2 * t;
    uint4 p0, p1;
    p0.x = pack_bf16x2(w[0], w[1]);   p0.y = pack_bf16x2(w[2], w[3]);
    p0.z = pack_bf16x2(w[4], w[5]);   p0.w = pack_bf16x2(w[6], w[7]);
    p1.x = pack_bf16x2(w[8], w[9]);   p1.y = pack_bf16x2(w[10], w[11]);
    p1.z = pack_bf16x2(w[12], w[13]); p1.w = pack_bf16x2(w[14], w[15]);
    __stcs(o, p0);
    __stcs(o + 1, p1);
  } else {
    float4* o = reinterpret_cast<float4*>(out) + 4 * t;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      __stcs(o + i, make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
  }
}

// Merge: CTA tile of 32 rows x 256 columns; thread (ty, tx) owns columns
// 8tx .. 8tx+7 of rows ty, ty+8, ty+16, ty+24.  The rank is consumed in slices
// of 32 staged in shared memory as fp32.
constexpr int kMgRows = 32, kMgCols = 256, kMgR = 32;

template <bool kBf16>
__global__ void __launch_bounds__(256)
merge_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ dq_codes,
             const float* __restrict__ dq_scales, const __nv_bfloat16* __restrict__ A,
             const __nv_bfloat16* __restrict__ B, int r, int64_t n_in, int64_t n_out,
             void* __restrict__ out, int fmt) {
  __shared__ float sA[kMgRows][kMgR + 1];
  __shared__ __align__(16) float sB[kMgR][kMgCols];
  __shared__ float lv[16];
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  if (tid < 16) lv[tid] = fmt == kFmtInt16 ? static_cast<float>(tid - 8) : nf4_level(tid);
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * kMgRows;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kMgCols;

  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int j0 = 0; j0 < r; j0 += kMgR) {
    __syncthreads();
    for (int e = tid; e < kMgRows * kMgR; e += 256) {
      const int rr = e / kMgR, jj = e % kMgR;
      const int64_t row = row0 + rr;
      sA[rr][jj] = (row < n_in && j0 + jj < r) ? __bfloat162float(A[row * r + j0 + jj]) : 0.0f;
    }
    for (int e = tid; e < kMgR * kMgCols; e += 256) {
      const int jj = e / kMgCols, cc = e % kMgCols;
      const int64_t col = col0 + cc;
      sB[jj][cc] = (col < n_out && j0 + jj < r) ? __bfloat162float(B[(j0 + jj) * n_out + col]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kMgR; ++jj) {
      float b[8];
      const float4 b0 = *reinterpret_cast<const float4*>(&sB[jj][8 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sB[jj][8 * tx + 4]);
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = sA[ty + 8 * i][jj];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a, b[j], acc[i][j]);
      }
    }
  }

  const int64_t col = col0 + 8 * tx;
  if (col >= n_out) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = row0 + ty + 8 * i;
    if (row >= n_in) continue;
    const int64_t e0 = row * n_out + col;                 // multiple of 8
    const int64_t blk = e0 / kBlock;
    const float a = fmt == kFmtInt16 ? dq_scales[e0 / 16]
                                     : absmax_deq(dq_codes[blk], dq_scales[blk / kGroup], fmt == kFmtU8);
    const uint32_t c = *reinterpret_cast<const uint32_t*>(codes + e0 / 2);
    float w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = __fadd_rn(mul_rn(lv[(c >> (4 * j)) & 0xF], a), acc[i][j]);
    if constexpr (kBf16) {
      uint4 p;
      p.x = pack_bf16x2(w[0], w[1]); p.y = pack_bf16x2(w[2], w[3]);
      p.z = pack_bf16x2(w[4], w[5]); p.w = pack_bf16x2(w[6], w[7]);
      *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + e0) = p;
    } else {
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e0);
      o[0] = make_float4(w[0], w[1], w[2], w[3]);
      o[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
  }
}

// A (in x r) and B (r x out) from the leading r singular triplets: thread e
// writes element e of A (e < in r) or element e - in r of B.
__global__ void __launch_bounds__(256)
loftq_split_kernel(const float* __restrict__ U, int64_t ldu, const float* __restrict__ S,
                   const float* __restrict__ Vh, int64_t ldv, int64_t n_in, int64_t n_out, int r,
                   uint16_t* __restrict__ A, uint16_t* __restrict__ B) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t na = n_in * r;
  if (e < na) {
    const int64_t i = e / r;
    const int j = static_cast<int>(e - i * r);
    A[e] = static_cast<uint16_t>(pack_bf16x2(mul_rn(U[i * ldu + j], __fsqrt_rn(S[j])), 0.0f));
  } else if (e < na + static_cast<int64_t>(r) * n_out) {
    const int64_t f = e - na;
    const int j = static_cast<int>(f / n_out);
    const int64_t o = f - static_cast<int64_t>(j) * n_out;
    B[f] = static_cast<uint16_t>(pack_bf16x2(mul_rn(__fsqrt_rn(S[j]), Vh[j * ldv + o]), 0.0f));
  }
}

}  // namespace

cudaError_t launch_loftq_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldv,
                               int64_t n_in, int64_t n_out, int r, uint16_t* A, uint16_t* B, cudaStream_t stream) {
  const int64_t n = (n_in + n_out) * r;
  loftq_split_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(U, ldu, S, Vh, ldv, n_in, n_out,
                                                                                 r, A, B);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* dq_codes,
                              const float* dq_scales, int64_t n, bool bf16, void* out,
                              cudaStream_t stream, int fmt, const float* W0) {
  const int64_t n16 = n / 16;
  if (n16 == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((n16 + kDqThreads - 1) / kDqThreads);
  timing_before(QLORA_KERNEL_DEQUANTIZE, stream);
  if (W0)
    dequantize_kernel<kDqResidual><<<grid, kDqThreads, 0, stream>>>(codes, dq_codes, dq_scales, n16, out, fmt, W0);
  else if (bf16)
    dequantize_kernel<kDqBf16><<<grid, kDqThreads, 0, stream>>>(codes, dq_codes, dq_scales, n16, out, fmt, nullptr);
  else
    dequantize_kernel<kDqF32><<<grid, kDqThreads, 0, stream>>>(codes, dq_codes, dq_scales, n16, out, fmt, nullptr);
  timing_after(QLORA_KERNEL_DEQUANTIZE, stream);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_merge(const uint8_t* codes, const uint8_t* dq_codes, const float* dq_scales,
                         const uint16_t* A, const uint16_t* B, int r, int64_t n_in,
                         int64_t n_out, bool bf16, void* out, cudaStream_t stream, int fmt) {
  dim3 grid(static_cast<unsigned>((n_out + kMgCols - 1) / kMgCols),
            static_cast<unsigned>((n_in + kMgRows - 1) / kMgRows));
  const auto* a = reinterpret_cast<const __nv_bfloat16*>(A);
  const auto* b = reinterpret_cast<const __nv_bfloat16*>(B);
  timing_before(QLORA_KERNEL_MERGE, stream);
  if (bf16)
    merge_kernel<true><<<grid, 256, 0, stream>>>(codes, dq_codes, dq_scales, a, b, r, n_in, n_out, out, fmt);
  else
    merge_kernel<false><<<grid, 256, 0, stream>>>(codes, dq_codes, dq_scales, a, b, r, n_in, n_out, out, fmt);
  timing_after(QLORA_KERNEL_MERGE, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
