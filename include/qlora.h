/*
 * libqlora -- the QLoRA adapted linear layer on NVIDIA B200 (sm_100a).
 *
 * A linear layer whose frozen weight W0 (in x out, stored row-major as (in, out))
 * is kept as 4-bit NormalFloat (NF4) codes with one absmax per 64 consecutive
 * weights, the absmax values themselves double-quantised to 8-bit codes (E4M3, or
 * linear uint8) with one fp32 scale per 256 absmax values -- or, the pages' second
 * base quantiser, as symmetric 2-4 bit integers with one fp32 scale per 16
 * weights -- plus trainable low-rank adapters A (in x r) and B (r x out):
 *
 *     forward   Y  = X deq(Wq) + (X A) B
 *     backward  dX = dY deq(Wq)^T + (dY B^T) A^T
 *               dA = X^T (dY B^T)            dB = (X A)^T dY
 *
 * Sources (pages of the method, cited by title and section):
 *   "QLoRA (low-rank adapters on a quantized model)" -- "How it works" steps 1-5
 *     (quantize once and freeze; W = Wq + A B with B = 0 at the start; dA = dW B^T,
 *     dB = A^T dW; optional merge), "What QLoRA adds over LoRA" (NF4 levels at
 *     normal quantiles, one absmax per block of 64, absmax quantised to 8 bits,
 *     weights dequantised to bf16 for each matmul and never updated).
 *   "LLMs · QLoRA" -- the blockwise quantiser: reshape to rows of 64, absmax per
 *     row, nearest level by argmin, reconstruction level[idx] * scale.
 *   "LoRA & QLoRA" -- "Mathematical Formulation" (h = W0 x + B(A x)),
 *     "Double Quantization" (absmax constants to an 8-bit float).
 *
 * Conventions for every call:
 *   - Pointers marked [device] are device memory of the CURRENT CUDA device,
 *     allocated and owned by the caller; the library keeps no pointer after return.
 *     The library allocates no memory.  Pointers marked [host] are host memory.
 *   - bf16 tensors are passed as uint16_t bit patterns (bfloat16).
 *   - Every tensor is dense row-major, in the shapes stated, 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return after enqueueing.  Argument checks run on the host
 *     before any launch; a failed check returns an error and launches nothing.
 *   - Inputs must not alias outputs.  W0 must be finite.
 *   - No call writes to the frozen weight (codes, dq_codes, dq_scales).
 *   - Errors: QLORA_ERR_CUDA if a launch fails; QLORA_ERR_UNSUPPORTED_DEVICE if
 *     the current device is not compute capability 10.0 (there is no fallback).
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qlora_status {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,        /* NULL where a tensor is required, bad enum, host pointer */
  QLORA_ERR_SHAPE = 2,              /* a size constraint of the call is violated */
  QLORA_ERR_ALIGNMENT = 3,          /* a tensor pointer is not 16-byte aligned */
  QLORA_ERR_WORKSPACE = 4,          /* workspace NULL or smaller than the call's minimum (see
                                       qlora_workspace_bytes) */
  QLORA_ERR_UNSUPPORTED_DEVICE = 5, /* current device is not sm_100 */
  QLORA_ERR_CUDA = 6,               /* a CUDA runtime call or kernel launch failed */
  QLORA_ERR_TIMEOUT = 7             /* a bounded wait inside a kernel gave up (qlora_ws_status) */
} qlora_status;

/* Output element type of qlora_dequantize / qlora_merge. */
typedef enum qlora_dtype { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* Operation whose workspace size qlora_workspace_bytes() reports. */
typedef enum qlora_op { QLORA_OP_FWD = 1, QLORA_OP_BWD = 2 } qlora_op;

/* Fixed format constants. */
#define QLORA_BLOCK 64   /* weights per absmax block */
#define QLORA_GROUP 256  /* absmax values per double-quantisation fp32 scale */

/* Weight formats (qlora_nf4_weight.dq_format). */
#define QLORA_DQ_E4M3 0   /* NF4, absmax codes OCP FP8 E4M3, s = max / 448 ("LoRA & QLoRA": an 8-bit float) */
#define QLORA_DQ_U8 1     /* NF4, absmax codes linear unsigned integers, s = max / 255 ("8 bits", pigeon guide) */
#define QLORA_FMT_INT16 2 /* symmetric integers from qlora_quantize_int: level = code - 8, one fp32
                             scale per 16 weights in dq_scales, no absmax codes (dq_codes unused) */

/*
 * The frozen, quantised weight (non-owning view; all pointers [device]).
 *   codes     : uint8[in*out/2]  NF4 codes of the flattened row-major (in, out) W0;
 *               element 2k in the low nibble of byte k, element 2k+1 in the high nibble.
 *   dq_codes  : uint8[in*out/64] 8-bit code of each block's absmax (block b = elements
 *               64b .. 64b+63 of the flattened W0), in the format dq_format.
 *   dq_scales : fp32[ceil(in*out/64/256)] scale of each group of 256 consecutive blocks.
 *   in, out   : matrix shape.
 *   dq_format : QLORA_DQ_E4M3 (0, what a zero-initialised descriptor holds),
 *               QLORA_DQ_U8, or QLORA_FMT_INT16 for a weight from qlora_quantize_int
 *               (then dq_codes may be NULL and dq_scales holds fp32[in*out/16];
 *               w' = fl32((code - 8) * dq_scales[e/16]) for element e); anything
 *               else is QLORA_ERR_INVALID_ARG.  Every call taking a descriptor
 *               accepts all three; an INT16 weight's forward always takes the
 *               fused GEMM (the small-M path is NF4 only).
 * Dequantised weight ("What QLoRA adds over LoRA"; "LLMs · QLoRA" levels[idx]*scale):
 *   absmax'_b = fl32(e4m3(dq_codes[b]) * dq_scales[b/256])   (E4M3)
 *             = fl32(dq_codes[b] * dq_scales[b/256])         (U8)
 *   w'        = fl32(nf4_level[code] * absmax'_b)   (fl32 = IEEE binary32 round-to-nearest)
 * and the matmuls use bf16(w') (round to nearest even).
 */
typedef struct qlora_nf4_weight {
  const uint8_t* codes;
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t in;
  int64_t out;
  int32_t dq_format;
} qlora_nf4_weight;

/*
 * Quantise W0 once ("How it works" step 1; "LLMs · QLoRA" quantiser; "What QLoRA
 * adds over LoRA" NF4 and double quantisation).
 *   W0        [device] fp32 (in, out).
 *   codes     [device] out: uint8[in*out/2].
 *   dq_codes  [device] out: uint8[in*out/64].
 *   dq_scales [device] out: fp32[ceil(in*out/64/256)].
 * Per block b: a_b = max |w| over the block; x = fl32(w / a_b) (IEEE division;
 * an all-zero block gives x = 0); code = index of the nearest NF4 level, ties to
 * the lower index.  Per group g of 256 blocks: s_g = fl32(max_b a_b / 448),
 * dq_codes[b] = E4M3 round-to-nearest-even, saturating at 448, of fl32(a_b / s_g)
 * (0 when s_g = 0).  Codes are bit-exact: they do not depend on launch shape.
 * Requires in >= 1, out >= 1, in*out % 64 == 0.  W0, codes, dq_codes and dq_scales
 * 16-byte aligned.
 */
QLORA_API qlora_status qlora_quantize_nf4(const float* W0, int64_t in, int64_t out, uint8_t* codes,
                                uint8_t* dq_codes, float* dq_scales, void* stream);

/*
 * qlora_quantize_nf4 with a choice of absmax code format (dq_format, as in
 * qlora_nf4_weight).  QLORA_DQ_U8: per group s_g = fl32(max_b a_b / 255) and
 * dq_codes[b] = min(255, rint(fl32(a_b / s_g))) with ties to even (0 when
 * s_g = 0).  The NF4 codes are the same in both formats (they use the exact
 * absmax).  Unknown formats give QLORA_ERR_INVALID_ARG.
 */
QLORA_API qlora_status qlora_quantize_nf4_ex(const float* W0, int64_t in, int64_t out, uint8_t* codes,
                                             uint8_t* dq_codes, float* dq_scales, int dq_format, void* stream);

/*
 * One weight of a batch quantisation: W0 [device] fp32 (in, out) and its outputs,
 * as in qlora_quantize_nf4.
 */
typedef struct qlora_quantize_job {
  const float* W0;
  int64_t in;
  int64_t out;
  uint8_t* codes;
  uint8_t* dq_codes;
  float* dq_scales;
} qlora_quantize_job;

/*
 * qlora_quantize_nf4_ex for n weights ("How it works" step 1 for every frozen
 * linear of a model; "What QLoRA adds over LoRA": adapters on every linear
 * layer): the same codes, absmax codes and scales, bit for bit, as n separate
 * calls.  Up
 * to 32 weights share one launch, whose persistent grid runs through all of their
 * groups in one sequence, so the weights do not each end with a partly idle wave.
 *   jobs  [host] n descriptors (read during the call only); every job must meet
 *         qlora_quantize_nf4's requirements.
 * QLORA_ERR_INVALID_ARG for n < 0, a NULL jobs array with n > 0, a NULL pointer
 * in a job or an unknown dq_format; QLORA_ERR_SHAPE for a job's bad shape: these
 * are checked for every job before anything is launched.  Whether each pointer
 * is 16-byte aligned device memory of the current device is checked for the 32
 * jobs of a launch just before that launch (QLORA_ERR_INVALID_ARG or
 * QLORA_ERR_ALIGNMENT; the launches before it stay issued).  n = 0 does nothing.
 */
QLORA_API qlora_status qlora_quantize_nf4_batch(const qlora_quantize_job* jobs, int n, int dq_format,
                                                void* stream);

/*
 * The second base quantiser, of the pages' simulation ("QLoRA (low-rank adapters
 * on a quantized model)", "The code, line by line": symmetric uniform integers,
 * one scale per 16 consecutive entries of the flattened (in, out) matrix; no NF4
 * and no double quantisation; "What the simulations show": 2, 3 and 4 bits, 2-bit
 * being ternary {-s, 0, s}).  Per group of 16 weights, Q = 2^(bits-1) - 1:
 *   s = fl32(max |w| / Q),  q = clamp(rint(fl32(w / s)), -Q, Q) (ties to even;
 *   0 when s = 0),  stored as the nibble q + 8 (packing as for NF4);
 *   w' = fl32(q s).
 *   W0      [device] fp32 (in, out).
 *   bits    2, 3 or 4, else QLORA_ERR_INVALID_ARG.
 *   codes   [device] out: uint8[in*out/2].
 *   scales  [device] out: fp32[in*out/16].
 *   All pointers 16-byte aligned (QLORA_ERR_ALIGNMENT otherwise).
 * Requires in*out % 16 == 0.  Bit-exact.  The result can be used by every call
 * that takes a qlora_nf4_weight, with dq_format = QLORA_FMT_INT16 (in*out must
 * then be a multiple of 64, as for NF4).
 */
QLORA_API qlora_status qlora_quantize_int(const float* W0, int64_t in, int64_t out, int bits, uint8_t* codes,
                                          float* scales, void* stream);

/* Dense w' (QLORA_F32) or bf16(w') (QLORA_BF16), (in, out), of a weight quantised
 * by qlora_quantize_int.  Bit-exact. */
QLORA_API qlora_status qlora_dequantize_int(const uint8_t* codes, const float* scales, int64_t in, int64_t out,
                                            void* W_out, int out_dtype, void* stream);

/*
 * Dequantise the frozen weight to a dense (in, out) matrix: W_out[k][n] = w'
 * (QLORA_F32) or bf16(w') (QLORA_BF16).  Bit-exact.
 *   w      [host] descriptor of [device] tensors.
 *   W_out  [device] out: fp32 or bf16 (in, out).
 * Requires in*out % 64 == 0.
 */
QLORA_API qlora_status qlora_dequantize(const qlora_nf4_weight* w, void* W_out, int out_dtype, void* stream);

/*
 * Forward of the adapted layer ("How it works" steps 2-3; "LoRA & QLoRA"
 * Mathematical Formulation h = W0 x + B(A x)):
 *   V = bf16(X A)  (fp32 accumulation),   Y = bf16(X bf16(w') + V B)  (fp32 accumulation).
 * For M <= 16 and an NF4 weight a dequant-GEMV computes the base term as
 * sum_k bf16(x_k a'_k) bf16(l_k) (the block absmax folded into the activation; the
 * same sum in exact arithmetic); otherwise the fused dequant GEMM runs.
 *   w      [host] descriptor of [device] tensors.
 *   X      [device] bf16 (M, in).
 *   A      [device] bf16 (in, r).          B [device] bf16 (r, out).
 *   Y      [device] out: bf16 (M, out).
 *   V_save [device] out: bf16 (M, r), the saved X A for the backward; may be NULL
 *          (then V lives in the workspace).
 *   ws     [device] workspace of at least qlora_workspace_bytes(QLORA_OP_FWD, ...)
 *          bytes, initialised once by qlora_ws_init().
 * Requires M >= 1, in % 64 == 0, out % 64 == 0, 8 <= r <= 256, r % 8 == 0.
 */
QLORA_API qlora_status qlora_linear_fwd(const qlora_nf4_weight* w, const uint16_t* X, int64_t M,
                              const uint16_t* A, const uint16_t* B, int r, uint16_t* Y,
                              uint16_t* V_save, void* ws, size_t ws_bytes, void* stream);

/*
 * The forward above for callers that cannot allocate device memory (no paper
 * counterpart: the pages describe the method, not how a library hands out
 * scratch space).  Some callers have no device allocator to give a workspace
 * with: a host program using only this C ABI, a plugin inside a runtime that
 * owns all device memory, or a path where a cudaMalloc and its possible device
 * synchronisation is not acceptable.  This entry point takes the same arguments
 * minus the workspace and uses a fixed array of QLORA_STATIC_WS_BYTES inside the
 * library's own device memory instead (held by every GPU that loads the library
 * until the process exits); it allocates nothing.
 *   Returns QLORA_ERR_WORKSPACE, launching nothing, when the smallest forward
 *   workspace of these sizes (everything but the fused GEMM's split partial
 *   tiles: the 1280-byte prefix and V, M x r bf16 rounded up to 256 bytes) is
 *   larger than QLORA_STATIC_WS_BYTES.  The GEMM then always keeps its tiles
 *   whole, which can cost up to one wave of tiles against qlora_linear_fwd with
 *   a full-size workspace.
 *   The array's device address is looked up on the current device with
 *   cudaGetSymbolAddress, and kept per device for the cases where the lookup is
 *   not made (QLORA_ERR_INVALID_ARG if no earlier call on the device made it).
 *   Every call shares the one array and zeroes its split counters first; calls
 *   whose work overlaps on the GPU (other streams, other threads) race and must
 *   not be issued.  A bounded wait that gives up inside a kernel sets the array's
 *   status word, which stays set until qlora_static_ws_status reads it.
 */
#define QLORA_STATIC_WS_BYTES (16u << 20)
QLORA_API qlora_status qlora_linear_fwd_static_ws(const qlora_nf4_weight* w, const uint16_t* X, int64_t M,
                                                  const uint16_t* A, const uint16_t* B, int r, uint16_t* Y,
                                                  uint16_t* V_save, void* stream);

/* qlora_ws_status for the array of qlora_linear_fwd_static_ws on the current
 * device: synchronise `stream`, then QLORA_ERR_TIMEOUT (and clear the word) if a
 * bounded wait in a kernel of a static-workspace call gave up since the last
 * check, else QLORA_OK.  It finds the array as the forward does. */
QLORA_API qlora_status qlora_static_ws_status(void* stream);

/*
 * Backward of the adapted layer ("How it works" step 4; "The code, line by line":
 * dA = dW B^T, dB = A^T dW, here in the factored form that never forms dW):
 *   U  = bf16(dY B^T)
 *   dX = bf16(dY bf16(w')^T + U A^T)     (written only if dX != NULL)
 *   dA = X^T U         (fp32, overwritten)
 *   dB = V^T dY        (fp32, overwritten), V = X A (the saved V, or recomputed)
 * The frozen weight receives no gradient.
 *   X  [device] bf16 (M, in).   V [device] bf16 (M, r) from the forward, or NULL.
 *   dY [device] bf16 (M, out).  A, B as in the forward.
 *   dX [device] out: bf16 (M, in), or NULL.
 *   dA [device] out: fp32 (in, r).   dB [device] out: fp32 (r, out).
 *   ws [device] at least qlora_workspace_bytes(QLORA_OP_BWD, ...) bytes.
 * Requires the forward's shape constraints.
 */
QLORA_API qlora_status qlora_linear_bwd(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V,
                              const uint16_t* dY, int64_t M, const uint16_t* A,
                              const uint16_t* B, int r, uint16_t* dX, float* dA, float* dB,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * Options of the _ex calls (and of qlora_linear_bwd_adam).
 *   adapter_scale  s in Y = X bf16(w') + s (X A) B: the LoRA scaling alpha / r
 *                  ("LoRA & QLoRA", "Scaling Factor alpha": it only rescales the
 *                  learning rate of A and B, which the pages' lab leaves out);
 *                  1 is the plain layer.  Applied where V = bf16(s X A) and
 *                  U = bf16(s dY B^T) are formed, so dX, dA and dB carry it.
 *                  A saved V is the scaled one.  Finite, else QLORA_ERR_INVALID_ARG.
 *   flags          QLORA_ACCUMULATE_GRADS: the backward adds into dA and dB
 *                  instead of overwriting them (gradient accumulation over
 *                  micro-batches); not allowed for the forward or with Adam.
 *   dropout_keep   [device] uint8 (M, r), row-major, 1 = keep, 0 = drop, or NULL
 *                  for no dropout.  Dropout on the low-rank intermediate
 *                  ("LoRA & QLoRA", "Dropout": applied to A x during training),
 *                  inverted: V = s (X A) keep / (1 - p), and the backward uses
 *                  U = s keep / (1 - p) (dY B^T), so the forward and the backward
 *                  of one micro-batch must get the same mask (the caller draws
 *                  it, e.g. Bernoulli(1 - p), and keeps it).  Read only.
 *   dropout_p      the drop probability p in [0, 1) the kept values are rescaled
 *                  by; checked only with a mask, else QLORA_ERR_INVALID_ARG.
 * A NULL options pointer means adapter_scale = 1, no flags and no dropout.
 */
#define QLORA_ACCUMULATE_GRADS 1u
typedef struct {
  float adapter_scale;
  uint32_t flags;
  const uint8_t* dropout_keep;
  float dropout_p;
} qlora_linear_opts;

/* qlora_linear_fwd with options (arguments otherwise as there). */
QLORA_API qlora_status qlora_linear_fwd_ex(const qlora_nf4_weight* w, const uint16_t* X, int64_t M,
                                           const uint16_t* A, const uint16_t* B, int r, uint16_t* Y,
                                           uint16_t* V_save, const qlora_linear_opts* opts, void* ws,
                                           size_t ws_bytes, void* stream);

/* qlora_linear_bwd with options (arguments otherwise as there).  With
 * QLORA_ACCUMULATE_GRADS, dA and dB must hold the sums so far (fp32). */
QLORA_API qlora_status qlora_linear_bwd_ex(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V,
                                           const uint16_t* dY, int64_t M, const uint16_t* A, const uint16_t* B,
                                           int r, uint16_t* dX, float* dA, float* dB,
                                           const qlora_linear_opts* opts, void* ws, size_t ws_bytes,
                                           void* stream);

/*
 * Adam / AdamW on the adapters, fused into the backward ("QLoRA (low-rank adapters
 * on a quantized model)", "The code, line by line": opt = Adam(A + B, lr=lr) is
 * given dA and dB only; "LoRA and QLoRA: Efficient Fine-Tuning Explained", "A real
 * run", trains with AdamW).  The
 * rule (Kingma & Ba with bias correction, weight decay decoupled as in AdamW):
 *   theta <- theta (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *   theta <- theta - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * in fp32 for every element of A (g = dA) and of B (g = dB).
 */
typedef struct {
  float lr;             /* >= 0 */
  float beta1, beta2;   /* in [0, 1) */
  float eps;            /* > 0 */
  float weight_decay;   /* >= 0; 0 is plain Adam */
  int64_t step;         /* t, 1-based: the bias corrections use b^t */
} qlora_adam_hparams;

/* The adapters' optimizer state, caller-owned fp32 device arrays, 16-byte aligned:
 * master copies A32 (in, r) and B32 (r, out), and the first (m) and second (v)
 * moments of each in the same layouts.  Updated in place. */
typedef struct {
  float* A32;
  float* B32;
  float* mA;
  float* vA;
  float* mB;
  float* vB;
} qlora_adam_state;

/*
 * One training step's backward with the optimizer step fused in: the gradients
 * of qlora_linear_bwd (dX written if dX != NULL), and instead of writing dA and
 * dB, one Adam step on (A32, mA, vA) with dA and on (B32, mB, vB) with dB, then
 * A = bf16(A32) and B = bf16(B32) in place.  dA and dB never reach memory.  dX
 * and U use the adapters as they were on entry (every read of A or B is ordered
 * before their update).
 *   X, V, dY, dX, ws, M, r: as for qlora_linear_bwd.
 *   A, B  [device] bf16, read, then overwritten with the updated adapters.
 *   st    [host] pointers to the optimizer state (device arrays, as above).
 *   hp    [host] hyper-parameters; QLORA_ERR_INVALID_ARG if out of range.
 *   opts  [host] options or NULL (adapter_scale; QLORA_ACCUMULATE_GRADS is refused).
 */
QLORA_API qlora_status qlora_linear_bwd_adam(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V,
                                             const uint16_t* dY, int64_t M, uint16_t* A, uint16_t* B, int r,
                                             uint16_t* dX, const qlora_adam_state* st,
                                             const qlora_adam_hparams* hp, const qlora_linear_opts* opts,
                                             void* ws, size_t ws_bytes, void* stream);

/*
 * Merge the adapters into a dense weight ("How it works" step 5):
 *   W_out = w' + A B   (fp32 accumulation; QLORA_F32 or QLORA_BF16 output, (in, out)).
 * Requires in % 64 == 0, out % 64 == 0, 8 <= r <= 256, r % 8 == 0.
 */
QLORA_API qlora_status qlora_merge(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r,
                         void* W_out, int out_dtype, void* stream);

/*
 * LoftQ-style initialisation of the adapters ("QLoRA (low-rank adapters on a
 * quantized model)", "Going further": start A and B from an SVD of W0 - Q(W0)
 * instead of B = 0).  Three steps: qlora_loftq_residual below, a rank-r (or
 * thin) singular value decomposition R = U diag(S) Vh by any library, and
 * qlora_loftq_split, which splits it symmetrically into A B.
 *
 * qlora_loftq_residual: R[k][n] = fl32(W0[k][n] - w'), w' the dequantised weight
 * of `w` (any format), for a weight quantised from this W0.  Bit-exact.
 *   W0  [device] fp32 (in, out).   w [host] descriptor of [device] tensors.
 *   R   [device] out: fp32 (in, out).
 * Requires in*out % 64 == 0.
 */
QLORA_API qlora_status qlora_loftq_residual(const float* W0, const qlora_nf4_weight* w, float* R, void* stream);

/*
 * qlora_loftq_split: the adapters from the leading r singular triplets,
 *   s_j = fl32(sqrt(S[j])) (IEEE square root),
 *   A[i][j] = bf16(fl32(U[i][j] s_j)),  B[j][o] = bf16(fl32(s_j Vh[j][o]))
 * for i < in, j < r, o < out, so that A B = U_r diag(S_r) Vh_r up to the
 * roundings (A^T A = B B^T = diag(S_r) in exact arithmetic).  Bit-exact.
 *   U   [device] fp32, row i at U + i ldu (ldu >= r); columns 0..r-1 are read.
 *   S   [device] fp32[r] or longer, >= 0 (singular values).
 *   Vh  [device] fp32, row j at Vh + j ldv (ldv >= out); rows 0..r-1 are read.
 *   A   [device] out: bf16 (in, r).   B [device] out: bf16 (r, out).
 *   All pointers 16-byte aligned; QLORA_ERR_SHAPE for r < 1 or short strides.
 */
QLORA_API qlora_status qlora_loftq_split(const float* U, int64_t ldu, const float* S, const float* Vh,
                                         int64_t ldv, int64_t in, int64_t out, int r, uint16_t* A,
                                         uint16_t* B, void* stream);

/* ---------------------------------------------------------------- helpers */

/* Bytes of workspace qlora_linear_fwd / qlora_linear_bwd use at these sizes on
 * the current device (0 for an unknown op or invalid sizes).  Host only: it reads
 * the device's SM count, no device memory.
 * Layout: a 1280-byte prefix (the 256-byte status word, then 1 KB of counters
 * of the fused dequant GEMM); V (M x r bf16, rounded up to 256 bytes); for the
 * backward U (the same size); then the GEMM's partial tiles: when the layer's
 * 256 x 256 output tiles do not divide evenly over the SMs, the K-steps of the
 * last tiles are shared between CTAs, which hand over one 256 KB fp32 partial
 * tile per SM.  A workspace that stops before the partial tiles is accepted too:
 * the GEMM then keeps every tile whole (slower by up to one wave of tiles). */
QLORA_API size_t qlora_workspace_bytes(int op, int64_t M, int64_t in, int64_t out, int r);

/* Zero the whole workspace (once, before its first use; QLORA_ERR_WORKSPACE if
 * it is shorter than the 1280-byte prefix).  Its first 256 bytes hold a status
 * word that the kernels set when a bounded wait gives up and qlora_ws_status()
 * clears; the GEMM's counters after it are zero again whenever a call's kernels
 * end; the rest is scratch (V, U, partial tiles) that every call rewrites.
 * Forward and backward calls of any sizes may share one workspace (the prefix
 * has one layout), but calls that share one must be ordered on one stream. */
QLORA_API qlora_status qlora_ws_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then report QLORA_ERR_TIMEOUT if a bounded wait in a
 * kernel that used this workspace gave up since the last check (and clear it),
 * else QLORA_OK.  Device work of a call that timed out left its outputs undefined. */
QLORA_API qlora_status qlora_ws_status(void* ws, void* stream);

/* The quantisers take no workspace: a bounded wait inside qlora_quantize_nf4(_ex)
 * that gives up (its bulk copies of W0 did not land within the limit) sets a
 * status word of the library on the device instead.  This call synchronises
 * `stream`, then returns QLORA_ERR_TIMEOUT (and clears the word) if that
 * happened on the current device since the last check, else QLORA_OK.  The codes
 * of a quantisation that timed out are undefined. */
QLORA_API qlora_status qlora_quantize_status(void* stream);

/* The 16 NF4 levels, ascending (code = index) [host]. */
QLORA_API void qlora_nf4_codebook(float out[16]);

/* Adapter parameters of one layer: r (in + out) ("How it works", adapter size). */
QLORA_API int64_t qlora_adapter_params(int64_t in, int64_t out, int r);

/* ---------------------------------------------------------------- measurement */

/* Kernels that qlora_time_kernel() can bracket with events. */
typedef enum qlora_kernel {
  QLORA_KERNEL_QUANTIZE = 1,   /* NF4 + double-quant encoder (qlora_quantize_nf4) */
  QLORA_KERNEL_DEQUANTIZE = 2, /* dense dequantisation (qlora_dequantize) */
  QLORA_KERNEL_MERGE = 3,      /* adapter merge (qlora_merge) */
  QLORA_KERNEL_FWD_GEMM = 4,   /* fused dequant GEMM of the forward */
  QLORA_KERNEL_DX_GEMM = 5,    /* fused dequant GEMM of dX */
  QLORA_KERNEL_RANK_R = 6,     /* the rank-r kernels: V, U, dA, dB (and their split sums) */
  QLORA_KERNEL_GEMV = 7        /* small-M forward (M <= 16) */
} qlora_kernel;

/* Arm launch timing for benchmarks: the next n launches of kernel `which` are
 * each bracketed by cudaEventRecord(starts[i]) / cudaEventRecord(stops[i]) on the
 * launching stream (starts/stops: [host] arrays of cudaEvent_t owned by the
 * caller), as external event records so that they also time launches captured
 * in a CUDA graph.  n = 0 disarms.  Process-wide state; not for concurrent callers.
 * Returns QLORA_ERR_INVALID_ARG for an unknown kernel or NULL arrays with n > 0. */
QLORA_API qlora_status qlora_time_kernel(int which, void* const* starts, void* const* stops, int n);

/* Most CTAs the fused dequant GEMMs use (0, the default: every SM, as CTA pairs
 * on the two SMs of a TPC; a count c gives max(1, c / 2) pairs, capped at the
 * pairs the device holds at once).  A testing and tuning knob: a small count makes
 * small layers exercise the shared-K-step schedule.  Process-wide; takes effect
 * for calls (and workspace sizes) after it.  QLORA_ERR_INVALID_ARG if ctas < 0. */
QLORA_API qlora_status qlora_gemm_set_ctas(int ctas);

/* Test of the failure path (no counterpart on the pages): one kernel runs a
 * single bounded wait that nothing can complete -- kind 0 on an mbarrier of its
 * own with no arrivals, kind 1 on the last of the workspace's GEMM counters
 * (zero, awaited to reach 1, advanced by nothing) -- with a limit of limit_us
 * microseconds (1 .. 1,000,000), after which it raises a bit in the workspace's
 * status word and returns, as every wait in the library's kernels does at its
 * 2 s limit.  qlora_ws_status then reports QLORA_ERR_TIMEOUT.  The kernel has no
 * copies or tensor-core work in flight, so the context stays usable.
 *   ws  [device] a workspace of at least 1280 bytes (the prefix), initialised by
 *       qlora_ws_init; the counter is left at zero.
 * QLORA_ERR_INVALID_ARG for another kind or limit, QLORA_ERR_WORKSPACE for a
 * missing or short workspace. */
QLORA_API qlora_status qlora_selftest_wait_timeout(void* ws, size_t ws_bytes, int kind, uint32_t limit_us,
                                                   void* stream);

/* Number of kernel launches libqlora has issued in this process. */
QLORA_API uint64_t qlora_launch_count(void);

/* Human-readable name of a status code (static string). */
QLORA_API const char* qlora_status_string(qlora_status s);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
