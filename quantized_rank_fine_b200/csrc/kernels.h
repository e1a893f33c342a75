// Internal launch functions of libqlora (host side).  Every function enqueues
// on `stream` and returns the launch status; arguments are already validated.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

namespace qlora {

constexpr int kMaxSplits = 16;   // most K/M splits of the rank-r kernels

// Workspace prefix shared by every call, which must start at zero (the only
// part of a workspace that needs initialising): the status word(s), then the
// counters of the fused GEMM's split tiles (one per CTA, left zero by every
// launch).  The prefix has the same layout for every call, so calls of
// different kinds can share a workspace.
constexpr size_t kWsStatusBytes = 256;
constexpr int kMaxGemmCtas = 256;
constexpr size_t kWsCounterBytes = kMaxGemmCtas * sizeof(uint32_t);
constexpr size_t kWsFixedBytes = kWsStatusBytes + kWsCounterBytes;

// Bookkeeping of the measurement helpers (defined in api.cu): every kernel
// launch is counted; an armed timing hook brackets launches of one kernel kind.
void count_launch();
void timing_before(int which, cudaStream_t stream);
void timing_after(int which, cudaStream_t stream);

struct WeightView {
  const uint8_t* codes;
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t in, out;
  int fmt;            // kFmtE4M3, kFmtU8 or kFmtInt16
};

// Weight formats (the values of qlora_nf4_weight.dq_format): NF4 with E4M3 or
// linear uint8 absmax codes, or symmetric integers (level = code - 8) with one
// fp32 scale per 16 weights in dq_scales.
constexpr int kFmtE4M3 = 0, kFmtU8 = 1, kFmtInt16 = 2;

// dq_u8 / u8: the absmax codes are linear uint8 (s = max / 255) instead of E4M3.
cudaError_t launch_quantize_nf4(const float* W0, int64_t n, uint8_t* codes, uint8_t* dq_codes,
                                float* dq_scales, cudaStream_t stream, bool dq_u8 = false);
// Several weights (n weights each, a multiple of 64): up to kQMaxJobs per launch,
// whose groups the persistent grid walks as one sequence.
constexpr int kQMaxJobs = 32;
struct QuantizeJob {
  const float* W0;
  int64_t n;
  uint8_t* codes;
  uint8_t* dq_codes;
  float* dq_scales;
};
cudaError_t launch_quantize_nf4_batch(const QuantizeJob* jobs, int n, cudaStream_t stream, bool dq_u8 = false);
// With W0 != nullptr the output is the fp32 residual fl32(W0 - w') instead (bf16 ignored).
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* dq_codes, const float* dq_scales,
                              int64_t n, bool bf16, void* out, cudaStream_t stream, int fmt = kFmtE4M3,
                              const float* W0 = nullptr);
// A = bf16(U[:, :r] fl32(sqrt S)), B = bf16(fl32(sqrt S) Vh[:r, :]); row strides ldu, ldv (elements).
cudaError_t launch_loftq_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldv,
                               int64_t n_in, int64_t n_out, int r, uint16_t* A, uint16_t* B, cudaStream_t stream);
cudaError_t launch_merge(const uint8_t* codes, const uint8_t* dq_codes, const float* dq_scales,
                         const uint16_t* A, const uint16_t* B, int r, int64_t n_in, int64_t n_out,
                         bool bf16, void* out, cudaStream_t stream, int fmt = kFmtE4M3);

// Symmetric uniform INT quantisation, one scale per 16 weights (bits 2..4),
// and its dense dequantisation.  n is a multiple of 16; W0, codes, scales and
// out 16-byte aligned (8-byte for codes).
cudaError_t launch_int_quantize(const float* W0, int64_t n, int bits, uint8_t* codes, float* scales,
                                cudaStream_t stream);
cudaError_t launch_int_dequantize(const uint8_t* codes, const float* scales, int64_t n, bool bf16, void* out,
                                  cudaStream_t stream);

// One Adam step fused into a gradient's final store (see qlora_linear_bwd_adam):
// the element g of parameter index i updates theta[i], m[i], v[i] and p16[i].
struct AdamParams {
  float* theta;
  float* m;
  float* v;
  uint16_t* p16;
  float lr, b1, b2, omb1, omb2, eps, decay, bc1, bc2;   // omb = 1 - b, decay = 1 - lr wd, bc = 1 - b^t
};

// Rank-r products (tcgen05), split-K reduced inside a thread-block cluster;
// `status` is the workspace status word.  V and U are scaled by `scale` (the
// adapter scale) as they are formed.  dA and dB take an optional Adam step
// (adam != nullptr): the gradient then updates the optimizer state instead of
// being stored; `accumulate` adds them to the stored values instead.
//
// Dropout on the low-rank intermediate: with keep != nullptr (device, M x r,
// 1 = keep) every stored element of V and U is also multiplied by keep_scale
// (1 / (1 - p)) where it is kept and by 0 where it is dropped.
struct Dropout {
  const uint8_t* keep = nullptr;
  float keep_scale = 1.0f;
};
cudaError_t launch_xa(const uint16_t* X, const uint16_t* A, int64_t M, int64_t n_in, int r, uint16_t* V,
                      uint32_t* status, cudaStream_t stream, float scale = 1.0f, Dropout drop = {});
cudaError_t launch_dybt(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t n_out, int r,
                        uint16_t* U, uint32_t* status, cudaStream_t stream, float scale = 1.0f,
                        Dropout drop = {});
// dB (r x out, fp32, stored from dB^T = dY^T V) and dA = X^T U (in x r, fp32) in
// one launch; with adam_a / adam_b the Adam step replaces the stores.
cudaError_t launch_dbda(const uint16_t* V, const uint16_t* dY, const uint16_t* X, const uint16_t* U, int64_t M,
                        int64_t n_in, int64_t n_out, int r, float* dA, float* dB, uint32_t* status,
                        cudaStream_t stream, const AdamParams* adam_a = nullptr, const AdamParams* adam_b = nullptr,
                        bool accumulate = false);

// Small-M forward (M <= kGemvMaxTokens): base + adapter in one kernel, the
// K-splits of a column tile reduced inside a thread-block cluster; no workspace.
// Launched as a programmatic dependent of the kernel before it (which writes V).
constexpr int64_t kGemvMaxTokens = 16;
bool gemv_supported(int64_t M, int64_t K, int64_t N);
// V = X A for M <= kGemvMaxTokens on CUDA cores (K split over a cluster); lets
// the small-M forward launched after it start early.
cudaError_t launch_xa_small(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, uint16_t* V,
                            cudaStream_t stream, float scale = 1.0f, Dropout drop = {});
cudaError_t launch_gemv(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B, int64_t M,
                        int r, uint16_t* Y, uint32_t* status, cudaStream_t stream);

// Fused dequant GEMMs (tcgen05, persistent grid); `status` is the workspace
// status word.  When the tile count does not divide evenly over the CTAs the
// K-steps of the last tiles are shared between CTAs: `counters` (the
// workspace's kMaxGemmCtas counters, zero) and `partials` (one 256 x 256 fp32
// tile per CTA, *_gemm_split_bytes) hold their hand-over.  With partials ==
// nullptr, or fewer bytes, every tile stays whole.  Launch them only right after
// the rank-r kernel that writes V or U (launch_xa, launch_dybt, launch_dbda):
// they read their other inputs before that kernel has finished, which is safe
// because it starts them only once the kernels before it have finished.
cudaError_t launch_fwd_gemm(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B,
                            int64_t M, int r, uint16_t* Y, uint32_t* status, uint32_t* counters,
                            void* partials, size_t partial_bytes, cudaStream_t stream);
cudaError_t launch_dx_gemm(const WeightView& w, const uint16_t* dY, const uint16_t* U, const uint16_t* A,
                           int64_t M, int r, uint16_t* dX, uint32_t* status, uint32_t* counters,
                           void* partials, size_t partial_bytes, cudaStream_t stream);
size_t fwd_gemm_split_bytes(int64_t M, int64_t n_in, int64_t n_out, int r);
size_t dx_gemm_split_bytes(int64_t M, int64_t n_in, int64_t n_out, int r);
// Most CTAs the GEMMs use (0: one per SM); a testing and tuning knob.
void set_gemm_ctas(int ctas);

// Synchronise `stream` and read (then clear) the quantiser's device status word.
cudaError_t quantize_status_take(cudaStream_t stream, uint32_t* flags);

// One bounded wait that nothing completes (kind 0: an mbarrier without
// arrivals; kind 1: `counter`, left at 0, awaited to reach 1), giving up after
// limit_ns and raising kFlagTimeoutSelftest in `status`.
cudaError_t launch_selftest_wait(uint32_t* status, const uint32_t* counter, int kind, uint64_t limit_ns,
                                 cudaStream_t stream);

// Smallest workspace a forward/backward call accepts (no split tiles); the
// size qlora_workspace_bytes returns also holds the split region.
size_t ws_min_bytes(int op, int64_t M, int64_t in, int64_t out, int r);

}  // namespace qlora
