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

// Chunks of 16 weights per thread: chunk u of thread t is t + u * (grid threads),
// so each of a thread's loads is coalesced across the warp and all of them are
// in flight before any arithmetic.
constexpr int kDqUnroll = 4;

template <int kMode>
__device__ __forceinline__ void dequant_store(const float (&w)[16], int64_t t, void* __restrict__ out,
                                              const float* __restrict__ W0) {
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

template <int kMode>
__global__ void __launch_bounds__(kDqThreads)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ dq_codes,
                  const float* __restrict__ dq_scales, int64_t n16, void* __restrict__ out, int fmt,
                  const float* __restrict__ W0) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = fmt == kFmtInt16 ? static_cast<float>(static_cast<int>(threadIdx.x) - 8)
                                                           : nf4_level(threadIdx.x);
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDqThreads;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kDqThreads + threadIdx.x;
  uint2 c[kDqUnroll];
  float a[kDqUnroll];
#pragma unroll
  for (int u = 0; u < kDqUnroll; ++u) {
    const int64_t t = t0 + u * stride;
    c[u] = make_uint2(0u, 0u);
    a[u] = 0.0f;
    if (t < n16) {
      const int64_t blk = t >> 2;                       // 4 chunks per 64-weight block
      c[u] = __ldcs(reinterpret_cast<const uint2*>(codes) + t);
      a[u] = fmt == kFmtInt16 ? dq_scales[t]          // one scale per 16 weights
                              : absmax_deq(dq_codes[blk], dq_scales[blk / kGroup], fmt == kFmtU8);
    }
  }
#pragma unroll
  for (int u = 0; u < kDqUnroll; ++u) {
    const int64_t t = t0 + u * stride;
    if (t >= n16) break;
    float w[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t word = (i < 4) ? c[u].x : c[u].y;
      const uint32_t byte = (word >> (8 * (i & 3))) & 0xFFu;
      w[2 * i] = mul_rn(lv[byte & 0xF], a[u]);
      w[2 * i + 1] = mul_rn(lv[byte >> 4], a[u]);
    }
    dequant_store<kMode>(w, t, out, W0);
  }
}

// Merge: W = w' + A B.  The rank-r product runs on the tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate); the epilogue adds the dequantised weight
// and stores.  CTA tile: 128 rows x 64 columns, 8 warps of 16 rows each.  The
// CTA's 64 columns of B (r x 64 bf16, zero-padded to a multiple of 16 rows) sit
// row-major in shared memory with a 144-byte row pitch, read as transposed 8 x 8
// blocks (ldmatrix .trans) that are exactly the MMA's B fragments, without bank
// conflicts; A fragments are 32-bit loads of A's rows.  Lane (g, t) ends with
// rows g and g + 8 of its warp and columns 8j + 2t, 8j + 2t + 1 of every 8-column
// tile j: one code byte per (row, tile), and each warp store of 4 lanes writes
// 32 contiguous bytes.
constexpr int kMgRows = 128, kMgCols = 64;
constexpr int kMgPitch = kMgCols + 8;          // bf16 per shared row of B (144 bytes)

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool kBf16>
__global__ void __launch_bounds__(256)
merge_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ dq_codes,
             const float* __restrict__ dq_scales, const uint16_t* __restrict__ A,
             const uint16_t* __restrict__ B, int r, int64_t n_in, int64_t n_out,
             void* __restrict__ out, int fmt) {
  extern __shared__ __align__(16) uint16_t sB[];   // [r16][kMgPitch]
  __shared__ float lv[16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int r16 = (r + 15) & ~15;
  if (tid < 16) lv[tid] = fmt == kFmtInt16 ? static_cast<float>(tid - 8) : nf4_level(tid);
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * kMgRows;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kMgCols;
  // B's rows 0..r-1, columns n0..n0+63, as 16-byte chunks; rows r..r16-1 zero
  for (int e = tid; e < r16 * (kMgCols / 8); e += 256) {
    const int k = e >> 3, c = e & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < r) v = *reinterpret_cast<const uint4*>(B + static_cast<int64_t>(k) * n_out + n0 + 8 * c);
    *reinterpret_cast<uint4*>(sB + k * kMgPitch + 8 * c) = v;
  }
  __syncthreads();

  const int64_t rg = row0 + warp * 16 + g;         // rows rg and rg + 8
  const bool ok0 = rg < n_in, ok1 = rg + 8 < n_in;
  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.0f;
  const uint32_t sb = static_cast<uint32_t>(__cvta_generic_to_shared(sB));
  for (int k0 = 0; k0 < r16; k0 += 16) {
    const int ka = k0 + 2 * t, kb = ka + 8;
    auto ld_a = [&](int64_t row, bool ok, int k) -> uint32_t {
      return (ok && k < r) ? *reinterpret_cast<const uint32_t*>(A + row * r + k) : 0u;
    };
    const uint32_t a0 = ld_a(rg, ok0, ka), a1 = ld_a(rg + 8, ok1, ka);
    const uint32_t a2 = ld_a(rg, ok0, kb), a3 = ld_a(rg + 8, ok1, kb);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      // matrices: (k0..7, tile j), (k8..15, tile j), (k0..7, tile j+1), (k8..15, tile j+1);
      // lane 8q + i gives row i of matrix q
      const int q = lane >> 3, i = lane & 7;
      const uint32_t addr = sb + static_cast<uint32_t>(((k0 + (q & 1) * 8 + i) * kMgPitch + (j + (q >> 1)) * 8) * 2);
      uint32_t b0, b1, b2, b3;
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                   : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                   : "r"(addr));
      mma_16816(acc[j], a0, a1, a2, a3, b0, b1);
      mma_16816(acc[j + 1], a0, a1, a2, a3, b2, b3);
    }
  }

  // epilogue: w' + the product, row rg (c[0], c[1]) and rg + 8 (c[2], c[3])
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t row = rg + 8 * h;
    if (row >= n_in) continue;
    const int64_t e0 = row * n_out + n0;          // a multiple of 64
    const uint4 cw0 = *reinterpret_cast<const uint4*>(codes + e0 / 2);
    const uint4 cw1 = *reinterpret_cast<const uint4*>(codes + e0 / 2 + 16);
    const uint32_t cw[8] = {cw0.x, cw0.y, cw0.z, cw0.w, cw1.x, cw1.y, cw1.z, cw1.w};
    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float a = 0.0f;
    if (fmt == kFmtInt16) s4 = *reinterpret_cast<const float4*>(dq_scales + e0 / 16);   // one per 16 columns
    else a = absmax_deq(dq_codes[e0 / kBlock], dq_scales[e0 / kBlock / kGroup], fmt == kFmtU8);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t byte = (cw[j] >> (8 * t)) & 0xFFu;      // columns 8j + 2t, 8j + 2t + 1
      const float sc = fmt == kFmtInt16 ? (j < 2 ? s4.x : j < 4 ? s4.y : j < 6 ? s4.z : s4.w) : a;
      const float w0 = __fadd_rn(mul_rn(lv[byte & 0xF], sc), acc[j][2 * h]);
      const float w1 = __fadd_rn(mul_rn(lv[byte >> 4], sc), acc[j][2 * h + 1]);
      const int64_t at = e0 + 8 * j + 2 * t;
      if constexpr (kBf16)
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(out) + at) = pack_bf16x2(w0, w1);
      else
        *reinterpret_cast<float2*>(reinterpret_cast<float*>(out) + at) = make_float2(w0, w1);
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
  const unsigned grid = static_cast<unsigned>((n16 + kDqThreads * kDqUnroll - 1) / (kDqThreads * kDqUnroll));
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
  dim3 grid(static_cast<unsigned>(n_out / kMgCols), static_cast<unsigned>((n_in + kMgRows - 1) / kMgRows));
  const size_t smem = static_cast<size_t>((r + 15) & ~15) * kMgPitch * 2;
  timing_before(QLORA_KERNEL_MERGE, stream);
  if (bf16)
    merge_kernel<true><<<grid, 256, smem, stream>>>(codes, dq_codes, dq_scales, A, B, r, n_in, n_out, out, fmt);
  else
    merge_kernel<false><<<grid, 256, smem, stream>>>(codes, dq_codes, dq_scales, A, B, r, n_in, n_out, out, fmt);
  timing_after(QLORA_KERNEL_MERGE, stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qlora
