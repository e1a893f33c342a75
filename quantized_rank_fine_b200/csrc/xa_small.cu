// Adapter down-projection V = X A for a few tokens (M <= 16), the first step of
// the small-M forward ("LoRA & QLoRA": the low-rank path X A B beside the frozen
// base; V = X A is the r-wide intermediate).
//
// At M <= 16 the product is M*K*r multiply-adds over K*r adapter weights: far
// too little for tensor-core tiles of 128 rows, so it runs on CUDA cores and is
// organised for latency instead:
//   * Grid (adapter-column tiles of 64) x (K-splits); the K-splits of a column
//     tile form one thread-block cluster.  A CTA copies its rows of X and of A
//     into shared memory with 16-byte loads (all of a thread's loads in flight
//     at once), 256 rows at a time, and forms its fp32 partial: a thread
//     accumulates one (column, token) pair over the rows kl, kl + nkl, ... of
//     its row lane kl (up to four pairs over all rows when the pairs outnumber
//     the threads); the row lanes are summed in shared memory.
//   * Each CTA stores every element of its partial into the receive buffer of
//     the CTA that owns the element (distributed shared memory); after one
//     cluster barrier the owners add the splits in order and write bf16 V.
//   * Launched as a programmatic dependent of the kernel before it, so that its
//     CTAs are resident when that kernel ends; it reads nothing in global memory
//     before that kernel has finished.  It then lets the dependent small-M forward
//     start at once: that kernel streams the 4-bit weights meanwhile and waits
//     for V only when it reaches the adapter rows.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qlora {

namespace {

using namespace sm100;

constexpr int kXaThreads = 256;
constexpr int kXaCols = 64;        // adapter columns per CTA
constexpr int kXaChunk = 256;      // rows of X and A in shared memory at a time
constexpr int kXaMaxCluster = 16;
constexpr int kXPitch = kXaChunk + 8;   // padded row of X in shared memory (bank spread)
constexpr int kXaMaxPer = 4;            // (column, token) pairs per thread: 64 x 16 / 256

struct XaArgs {
  const uint16_t* X;   // (M, K) bf16
  const uint16_t* A;   // (K, r) bf16
  int M;
  int64_t K;
  int r;
  int Kc;              // rows per split (multiple of 64)
  uint16_t* V;         // (M, r) bf16
  float scale;         // V = bf16(scale * X A)
  const uint8_t* keep; // dropout keep mask (M, r), 1 = keep, or nullptr
  float keep_scale;    // factor of the kept values (1 / (1 - p))
};

__global__ void __launch_bounds__(kXaThreads) xa_small_kernel(const XaArgs p) {
  // Everything before this kernel has finished once the wait returns, so the
  // dependent launched right after (which reads its own inputs at once) sees
  // them complete.
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);                       // [M][kXPitch]
  uint16_t* as = xs + kGemvMaxTokens * kXPitch;                           // [kXaChunk][kXaCols]
  float* red = reinterpret_cast<float*>(as + kXaChunk * kXaCols);         // [nkl][P] row lanes
  float* part = red + kXaThreads;                                         // [M x cols]
  float* recv = part + kGemvMaxTokens * kXaCols;                          // [S][cap]

  const int tid = threadIdx.x;
  const int jt = blockIdx.x, split = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(split) * p.Kc;
  const int rows = static_cast<int>(p.K - k0 < p.Kc ? p.K - k0 : p.Kc);   // multiple of 64
  const int c0 = jt * kXaCols;
  const int cols = p.r - c0 < kXaCols ? p.r - c0 : kXaCols;               // multiple of 8
  const int cw = cols > 32 ? 64 : (cols > 16 ? 32 : (cols > 8 ? 16 : 8));
  // (column, token) pairs: column j < cw, token m < mw (powers of two >= cols, M);
  // with P = cw * mw <= 256 thread t takes pair t % P and row lane t / P of
  // nkl = 256 / P, else pairs t + 256 u (u < P / 256) over all rows
  const int mw = p.M > 8 ? 16 : (p.M > 4 ? 8 : (p.M > 2 ? 4 : (p.M > 1 ? 2 : 1)));
  const int P = cw * mw;
  const int per = P > kXaThreads ? P / kXaThreads : 1;
  const int nkl = P >= kXaThreads ? 1 : kXaThreads / P;
  const int kl = P >= kXaThreads ? 0 : tid / P;
  float acc[kXaMaxPer];
#pragma unroll
  for (int u = 0; u < kXaMaxPer; ++u) acc[u] = 0.0f;

  for (int r0 = 0; r0 < rows; r0 += kXaChunk) {
    const int n = rows - r0 < kXaChunk ? rows - r0 : kXaChunk;   // multiple of 64
    // X rows: M x n bf16, 8 per 16-byte load (row pitch padded by 8 elements)
    const int xq = n / 8;
    for (int i = tid; i < p.M * xq; i += kXaThreads) {
      const int mm = i / xq, q = i % xq;
      reinterpret_cast<uint4*>(xs + mm * kXPitch)[q] =
          reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(mm) * p.K + k0 + r0)[q];
    }
    // A rows: n x cols bf16 of this column tile
    const int aq = cols / 8;
    for (int i = tid; i < n * aq; i += kXaThreads) {
      const int k = i / aq, q = i % aq;
      reinterpret_cast<uint4*>(as + k * kXaCols)[q] =
          reinterpret_cast<const uint4*>(p.A + (k0 + r0 + k) * p.r + c0)[q];
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kXaMaxPer; ++u) {
      const int pair = P >= kXaThreads ? tid + kXaThreads * u : tid % P;
      const int j = pair % cw, m = pair / cw;
      if (u < per && j < cols && m < p.M) {
        const uint16_t* xr = xs + m * kXPitch;
        float s = acc[u];
#pragma unroll 4
        for (int k = kl; k < n; k += nkl)
          s = fmaf(__uint_as_float(static_cast<uint32_t>(xr[k]) << 16),
                   __uint_as_float(static_cast<uint32_t>(as[k * kXaCols + j]) << 16), s);
        acc[u] = s;
      }
    }
    __syncthreads();   // the chunk buffers are refilled next
  }

  // this CTA's partial, part[m * cols + j]: the row lanes summed in order
  if (nkl > 1) {
    red[tid] = acc[0];   // red[kl * P + pair]
    __syncthreads();
    for (int e = tid; e < p.M * cols; e += kXaThreads) {
      const int mm = e / cols, jj = e % cols;
      float s = 0.0f;
      for (int l = 0; l < nkl; ++l) s += red[l * P + mm * cw + jj];
      part[e] = s;
    }
  } else {
#pragma unroll
    for (int u = 0; u < kXaMaxPer; ++u) {
      const int pair = tid + kXaThreads * u;
      const int j = pair % cw, m = pair / cw;
      if (u < per && j < cols && m < p.M) part[m * cols + j] = acc[u];
    }
  }
  __syncthreads();

  // split-K across the cluster: element e of the M x cols partial belongs to CTA
  // e / cap; each CTA stores its value into the owner's receive slot (its rank),
  // and after one cluster barrier the owner adds the slots in split order
  const int S = static_cast<int>(cluster_nctarank()), rank = static_cast<int>(cluster_ctarank());
  const int E = p.M * cols;
  const int cap = (E + S - 1) / S;
  const uint32_t recv_addr = smem_addr(recv);
  for (int e = tid; e < E; e += kXaThreads) {
    const int o = e / cap, slot = e - o * cap;
    st_shared_cluster_f32(mapa_shared(recv_addr + static_cast<uint32_t>((rank * cap + slot) * 4), o), part[e]);
  }
  cluster_sync();   // every push has landed
  for (int slot = tid; slot < cap && rank * cap + slot < E; slot += kXaThreads) {
    const int e = rank * cap + slot;
    float y = 0.0f;
    for (int sp = 0; sp < S; ++sp) y += recv[sp * cap + slot];
    const int mm = e / cols, jj = e % cols;
    const int64_t at = static_cast<int64_t>(mm) * p.r + c0 + jj;
    float v = y * p.scale;
    if (p.keep) v *= p.keep[at] ? p.keep_scale : 0.0f;
    p.V[at] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f));
  }
}

constexpr size_t kXaSmemBytes = (kGemvMaxTokens * kXPitch + kXaChunk * kXaCols) * 2 +
                                (kXaThreads + kGemvMaxTokens * kXaCols + kGemvMaxTokens * kXaCols + kXaMaxCluster) * 4;

// K-splits (the cluster size): about 256 rows each, at most kXaMaxCluster.
void xa_plan(int64_t K, int& S, int& Kc) {
  int64_t s = K / 256;
  s = s < 1 ? 1 : (s > kXaMaxCluster ? kXaMaxCluster : s);
  int64_t kc = ((K + s - 1) / s + 63) / 64 * 64;
  S = static_cast<int>((K + kc - 1) / kc);
  Kc = static_cast<int>(kc);
}

}  // namespace

cudaError_t launch_xa_small(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, uint16_t* V,
                            cudaStream_t stream, float scale, Dropout drop) {
  if (M < 1 || M > kGemvMaxTokens) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(xa_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kXaSmemBytes));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(xa_small_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int S, Kc;
  xa_plan(K, S, Kc);
  XaArgs a{X, A, static_cast<int>(M), K, r, Kc, V, scale, drop.keep, drop.keep_scale};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((r + kXaCols - 1) / kXaCols), static_cast<unsigned>(S));
  cfg.blockDim = dim3(kXaThreads);
  cfg.dynamicSmemBytes = kXaSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = static_cast<unsigned>(S);
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  timing_before(QLORA_KERNEL_RANK_R, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, xa_small_kernel, a);
  timing_after(QLORA_KERNEL_RANK_R, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace qlora
