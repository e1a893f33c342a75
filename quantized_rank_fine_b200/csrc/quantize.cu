// NF4 blockwise quantisation with double-quantised absmax, one pass over W0.
//
// What it computes ("LLMs · QLoRA" blockwise quantiser; "What QLoRA adds over
// LoRA" NF4 + double quantisation; "LoRA & QLoRA" "Double Quantization"):
//   per block of 64 consecutive weights:  a = max |w|,  x = fl32(w / a),
//     code = index of the nearest NF4 level (ties to the lower level);
//   per group of 256 consecutive blocks:  s = fl32(max a / 448),
//     dq_code = E4M3_RNE_satfinite(fl32(a / s))   (0 when s = 0);
//   or, with linear uint8 absmax codes, s = fl32(max a / 255) and
//     dq_code = min(255, rint(fl32(a / s)))  (ties to even; 0 when s = 0).
//
// Layout: a persistent grid of two 256-thread CTAs per SM walks the groups
// (16,384 weights = 64 KB of fp32 each), every group as two halves of 128 blocks.
// One launch can take several weights (a batch of up to kQMaxJobs): their groups
// are numbered one after the other, so the CTAs run through all of them without a
// tail per weight.
// A bulk asynchronous copy streams each half-group into one of three 32 KB
// shared-memory buffers, two halves ahead of the one being encoded, so HBM is
// read continuously with no thread involvement.  Warp w owns blocks 16w .. 16w+15
// of a half, 8 at a time; lane l serves a quarter (16 consecutive weights) of
// block l/4, reading its four 16-byte chunks in a rotated order so that the 8
// lanes of each quarter-warp hit 8 different bank groups.  The block absmax needs
// a 2-step shuffle and each lane stores its 16 codes as one 8-byte word (a warp
// writes 256 contiguous bytes).  HBM traffic per weight: 4 B read + 0.5 B codes +
// 1/64 B dq code + 4/16384 B scale.
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
// threshold.  The (rare) weights closer than that are redone one by one with
// IEEE division against the exact threshold of their cell.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qlora {

namespace {

constexpr int kQThreads = 256;
constexpr int kHalfBlocks = kGroup / 2;                // blocks per half-group
constexpr int kQBuf = 3;                               // half-groups in flight
constexpr uint32_t kHalfBytes = kHalfBlocks * kBlock * 4;   // 32 KB of fp32
constexpr int kCells = 65;
constexpr float kRoundBase = 12582912.0f;            // 1.5 * 2^23: integers land in the low bits

// Status word of the quantiser (it takes no workspace): a bounded wait for a
// bulk copy that gives up raises a bit here; qlora_quantize_status reads and
// clears it.  One per device (a __device__ variable of the module).
__device__ uint32_t g_quantize_status;

// Fast code of q; `near` accumulates whether q is within 2^-19 of the cell's threshold.
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

// Exact code of the correctly rounded quotient x = w / a: the thresholds below x.
__device__ __forceinline__ uint32_t exact_code(float w, float a, const float* __restrict__ thr) {
  const float x = (a > 0.0f) ? __fdiv_rn(w, a) : 0.0f;
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < 15; ++j) c += (x > thr[j]) ? 1u : 0u;
  return c;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// The weights of one launch.  Group gg of the launch is group gg - group0[j] of
// weight j, for the j with group0[j] <= gg < group0[j + 1].
// NJ is the capacity: 1 for a single weight (a small parameter block, so that a
// launch per weight costs no more than before), kQMaxJobs for a batch.
template <int NJ>
struct QJobs {
  int n;
  int64_t group0[NJ + 1];
  int64_t nblocks[NJ];
  const float* W0[NJ];
  uint8_t* codes[NJ];
  uint8_t* dq_codes[NJ];
  float* dq_scales[NJ];
};

// The weight of group gg, searched upward from `j` (a CTA's groups only increase,
// so each search starts where the previous one ended).
template <int NJ>
__device__ __forceinline__ int job_of(const QJobs<NJ>& q, int64_t gg, int j = 0) {
  if constexpr (NJ == 1) return 0;
  while (j + 1 < q.n && q.group0[j + 1] <= gg) ++j;
  return j;
}

// Work item i of this CTA: half (i & 1) of its group number i >> 1.  `jc` is the
// weight of the item issued before (items are issued in increasing order).
template <int NJ>
__device__ __forceinline__ void issue_half(int64_t i, const QJobs<NJ>& q, uint32_t buf0, uint32_t bar0, int& jc) {
  const int64_t gg = blockIdx.x + (i >> 1) * gridDim.x;
  if (gg >= q.group0[q.n]) return;
  const int j = jc = job_of(q, gg, jc);
  const int64_t blk = (gg - q.group0[j]) * kGroup + (i & 1) * kHalfBlocks;
  const int b = static_cast<int>(i % kQBuf);
  if (blk >= q.nblocks[j]) {   // the empty second half of a short group: complete the phase
    sm100::mbar_arrive(bar0 + 8 * b);
    return;
  }
  const int64_t nb = min(static_cast<int64_t>(kHalfBlocks), q.nblocks[j] - blk);
  const uint32_t bytes = static_cast<uint32_t>(nb * kBlock * 4);
  sm100::mbar_arrive_expect_tx(bar0 + 8 * b, bytes);
  bulk_load(buf0 + b * kHalfBytes, q.W0[j] + blk * kBlock, bytes, bar0 + 8 * b);
}

template <int NJ>
__global__ void __launch_bounds__(kQThreads, 2)
quantize_nf4_kernel(const __grid_constant__ QJobs<NJ> q, bool dq_u8) {
  extern __shared__ __align__(128) uint8_t qsmem[];
  __shared__ uint32_t lut[kCells];
  __shared__ float thr_exact[16];
  __shared__ float amax[kGroup];
  __shared__ float red[kQThreads / 32];
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
  if (tid < 16) thr_exact[tid] = tid < 15 ? c_nf4_threshold[tid] : 2.0f;
  int jissue = 0, jgroup = 0;   // the weights of the last copy issued (thread 0) and of the current group
  if (tid == 0) {
    for (int b = 0; b < kQBuf; ++b) sm100::mbar_init(bar0 + 8 * b, 1);
    sm100::fence_mbar_init();
    // W0 may be written by the kernel this one follows (programmatic dependent
    // launch): the set-up above overlaps its tail, the copies wait for it
    sm100::grid_dependency_wait();
    for (int j = 0; j < kQBuf; ++j) issue_half(j, q, buf0, bar0, jissue);
  }
  __syncthreads();
  // the outputs are written only after the kernel before has completed
  sm100::grid_dependency_wait();

  const int quarter = lane & 3;            // which 16 weights of its block
  const int bsub = lane >> 2;              // block among the 8 of an iteration
  // rotated chunk order: the 8 lanes of a quarter-warp read 8 different 16-byte bank groups
  const int rot = (quarter >> 1) + 2 * (bsub & 1);
  int64_t j = 0, failed_at = -1;
  const int64_t ngroups = q.group0[q.n];
  for (int64_t gg = blockIdx.x; gg < ngroups; gg += gridDim.x) {
    // group g of weight jb
    const int jb = jgroup = job_of(q, gg, jgroup);
    const int64_t g = gg - q.group0[jb];
    const int64_t blk0 = g * kGroup;
    const int nblk = static_cast<int>(q.nblocks[jb] - blk0 < kGroup ? q.nblocks[jb] - blk0 : kGroup);
    uint8_t* __restrict__ codes = q.codes[jb];
    uint8_t* __restrict__ dq_codes = q.dq_codes[jb];
    float* __restrict__ dq_scales = q.dq_scales[jb];
    // Every group is two work items.  The second half of a short group (a weight's
    // last) is empty: its barrier phase completes without a copy and nothing is
    // encoded, so the item numbering of the copies and of this loop stay in step
    // across the weights of the launch.
    for (int h = 0; h < 2; ++h, ++j) {
      const bool empty = h * kHalfBlocks >= nblk;
      // one weight: its short group is this CTA's last, nothing follows the empty half
      if constexpr (NJ == 1) {
        if (empty) break;
      }
      const int b = static_cast<int>(j % kQBuf);
      const uint32_t ph = static_cast<uint32_t>((j / kQBuf) & 1);
      const bool got = sm100::mbar_wait(bar0 + 8 * b, ph, &g_quantize_status, kFlagTimeoutProducer);
      if (!__syncthreads_and(got)) {
        failed_at = j;
        break;
      }
      const float* gs = reinterpret_cast<const float*>(qsmem + b * kHalfBytes);
      if (!empty) {
#pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int hb = warp * 16 + it * 8 + bsub;     // block within the half
          const int lb = h * kHalfBlocks + hb;          // block within the group
          float4 v[4];
          int ci[4];
  #pragma unroll
          for (int c = 0; c < 4; ++c) {
            ci[c] = (c + rot) & 3;
            v[c] = (lb < nblk) ? *reinterpret_cast<const float4*>(gs + hb * kBlock + quarter * 16 + 4 * ci[c])
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
            const bool exact_all = !(rcp <= 3.0e38f);   // a subnormal absmax: exact path only
            if (exact_all) rcp = 0.0f;
            uint64_t word = 0;
            uint32_t near_chunks = 0;                   // bit ci: that chunk may sit across a threshold
  #pragma unroll
            for (int c = 0; c < 4; ++c) {
              bool nr = exact_all;
              const uint32_t c4 = fast_code(__fmul_rn(v[c].x, rcp), lut, nr) |
                                  (fast_code(__fmul_rn(v[c].y, rcp), lut, nr) << 4) |
                                  (fast_code(__fmul_rn(v[c].z, rcp), lut, nr) << 8) |
                                  (fast_code(__fmul_rn(v[c].w, rcp), lut, nr) << 12);
              word |= static_cast<uint64_t>(c4) << (16 * ci[c]);
              near_chunks |= (nr ? 1u : 0u) << ci[c];
            }
            // redo (rarely) the chunks with a quotient that may sit across its threshold
            while (near_chunks) {
              const int cc = __ffs(near_chunks) - 1;
              near_chunks &= near_chunks - 1;
              const float4 w4 = *reinterpret_cast<const float4*>(gs + hb * kBlock + quarter * 16 + 4 * cc);
              const uint32_t c4 = exact_code(w4.x, m, thr_exact) | (exact_code(w4.y, m, thr_exact) << 4) |
                                  (exact_code(w4.z, m, thr_exact) << 8) | (exact_code(w4.w, m, thr_exact) << 12);
              word = (word & ~(0xFFFFull << (16 * cc))) | (static_cast<uint64_t>(c4) << (16 * cc));
            }
            *reinterpret_cast<uint2*>(codes + (blk0 + lb) * (kBlock / 2) + quarter * 8) =
                make_uint2(static_cast<uint32_t>(word), static_cast<uint32_t>(word >> 32));
            if (quarter == 0) amax[lb] = m;
          }
        }
      }
      __syncthreads();   // buffer b fully read
      if (tid == 0) issue_half(j + kQBuf, q, buf0, bar0, jissue);
    }
    if (failed_at >= 0) break;

    // Group maximum of the block absmax values.
    float gm = (tid < nblk) ? amax[tid] : 0.0f;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    if (lane == 0) red[warp] = gm;
    __syncthreads();
    gm = red[0];
#pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w) gm = fmaxf(gm, red[w]);
    const float sc = __fdiv_rn(gm, dq_u8 ? 255.0f : 448.0f);
    if (tid < nblk) {
      uint8_t c = 0;
      if (sc > 0.0f) {
        const float y = __fdiv_rn(amax[tid], sc);
        c = dq_u8 ? static_cast<uint8_t>(fminf(rintf(y), 255.0f))
                  : static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
      }
      dq_codes[blk0 + tid] = c;
    }
    if (tid == 0) dq_scales[g] = sc;
    __syncthreads();   // amax and red reused by the next group
  }
  // A wait that gave up leaves up to kQBuf copies in flight into this CTA's
  // shared memory: wait for them (again bounded) before the CTA exits.
  if (failed_at >= 0 && tid == 0) {
    for (int64_t k = failed_at; k < failed_at + kQBuf; ++k) {
      const int64_t gk = blockIdx.x + (k >> 1) * gridDim.x;
      if (gk >= ngroups) continue;
      const int jk = job_of(q, gk);
      if ((gk - q.group0[jk]) * kGroup + (k & 1) * kHalfBlocks >= q.nblocks[jk]) continue;
      sm100::mbar_wait(bar0 + 8 * static_cast<int>(k % kQBuf), static_cast<uint32_t>((k / kQBuf) & 1),
                       &g_quantize_status, kFlagTimeoutProducer);
    }
  }
  __syncthreads();
}

}  // namespace

namespace {

// One launch over jobs [0, n) (n <= NJ).
template <int NJ>
cudaError_t launch_jobs(const QuantizeJob* jobs, int n, cudaStream_t stream, bool dq_u8) {
  QJobs<NJ> q{};
  q.n = 0;
  q.group0[0] = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t nblocks = jobs[i].n / kBlock;
    if (nblocks == 0) continue;
    const int k = q.n++;
    q.nblocks[k] = nblocks;
    q.W0[k] = jobs[i].W0;
    q.codes[k] = jobs[i].codes;
    q.dq_codes[k] = jobs[i].dq_codes;
    q.dq_scales[k] = jobs[i].dq_scales;
    q.group0[k + 1] = q.group0[k] + (nblocks + kGroup - 1) / kGroup;
  }
  const int64_t ngroups = q.group0[q.n];
  if (ngroups == 0) return cudaSuccess;
  static bool set[64] = {};
  static int sms[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(quantize_nf4_kernel<NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kQBuf * kHalfBytes));
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  const int64_t grid = std::min<int64_t>(ngroups, 2 * (dev < 64 ? sms[dev] : 148));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = kQBuf * kHalfBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  timing_before(QLORA_KERNEL_QUANTIZE, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_nf4_kernel<NJ>, q, dq_u8);
  timing_after(QLORA_KERNEL_QUANTIZE, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_nf4(const float* W0, int64_t n, uint8_t* codes, uint8_t* dq_codes,
                                float* dq_scales, cudaStream_t stream, bool dq_u8) {
  const QuantizeJob job{W0, n, codes, dq_codes, dq_scales};
  return launch_jobs<1>(&job, 1, stream, dq_u8);
}

cudaError_t launch_quantize_nf4_batch(const QuantizeJob* jobs, int n, cudaStream_t stream, bool dq_u8) {
  for (int i = 0; i < n; i += kQMaxJobs) {
    const cudaError_t e = launch_jobs<kQMaxJobs>(jobs + i, std::min(kQMaxJobs, n - i), stream, dq_u8);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Synchronise `stream`, then report (and clear) the quantiser's status word.
cudaError_t quantize_status_take(cudaStream_t stream, uint32_t* flags) {
  *flags = 0;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(flags, g_quantize_status, sizeof(uint32_t));
  if (e == cudaSuccess && *flags != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_quantize_status, &zero, sizeof(uint32_t));
  }
  return e;
}

}  // namespace qlora
