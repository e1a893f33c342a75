// The C ABI of libqlora: host-side argument checks, workspace layout, launches.
// Declarations, argument meaning, layouts and error behaviour: include/qlora.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>
#include <string.h>

#include <atomic>

#include "../../include/qlora.h"
#include "common.cuh"
#include "kernels.h"

using qlora::WeightView;

namespace {


size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device must be compute capability 10.0 (B200 / sm_100).
qlora_status check_device() {
  static int checked[64] = {};   // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return QLORA_ERR_UNSUPPORTED_DEVICE;
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    checked[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return checked[dev] == 1 ? QLORA_OK : QLORA_ERR_UNSUPPORTED_DEVICE;
}

// A required tensor: non-NULL, device (or managed) memory of the current device, 16-byte aligned.
qlora_status check_ptr(const void* p, bool required = true) {
  if (!p) return required ? QLORA_ERR_INVALID_ARG : QLORA_OK;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  cudaGetDevice(&dev);
  if (a.device != dev) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(p)) return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}

#define QLORA_TRY(expr)                  \
  do {                                   \
    qlora_status _s = (expr);            \
    if (_s != QLORA_OK) return _s;       \
  } while (0)

#define QLORA_CUDA(expr)                                 \
  do {                                                   \
    if ((expr) != cudaSuccess) return QLORA_ERR_CUDA;    \
  } while (0)

bool rank_ok(int r) { return r >= 8 && r <= 256 && r % 8 == 0; }

bool linear_shape_ok(int64_t M, int64_t in, int64_t out, int r) {
  return M >= 1 && M <= (int64_t(1) << 31) - 1 && in >= 64 && out >= 64 && in % 64 == 0 && out % 64 == 0 &&
         in <= (int64_t(1) << 24) && out <= (int64_t(1) << 24) && rank_ok(r);
}

qlora_status check_weight_shape(const qlora_nf4_weight* w) {
  if (!w || !w->codes || !w->dq_scales) return QLORA_ERR_INVALID_ARG;
  if (w->dq_format != QLORA_DQ_E4M3 && w->dq_format != QLORA_DQ_U8 && w->dq_format != QLORA_FMT_INT16)
    return QLORA_ERR_INVALID_ARG;
  if (w->dq_format != QLORA_FMT_INT16 && !w->dq_codes) return QLORA_ERR_INVALID_ARG;
  if (w->in < 1 || w->out < 1 || w->in > (int64_t(1) << 40) / w->out || (w->in * w->out) % QLORA_BLOCK != 0)
    return QLORA_ERR_SHAPE;
  return QLORA_OK;
}

qlora_status check_weight(const qlora_nf4_weight* w) {
  QLORA_TRY(check_weight_shape(w));
  QLORA_TRY(check_ptr(w->codes));
  QLORA_TRY(check_ptr(w->dq_codes, w->dq_format != QLORA_FMT_INT16));
  QLORA_TRY(check_ptr(w->dq_scales));
  return QLORA_OK;
}

WeightView view(const qlora_nf4_weight* w) {
  return WeightView{w->codes, w->dq_codes, w->dq_scales, w->in, w->out, w->dq_format};
}

// Workspace layout (byte offsets), shared by the size query and the calls:
// the fixed prefix (status word, the GEMM's split counters), V (when the
// caller does not keep it), U (backward), and last the fused GEMM's partial
// tiles for the tiles whose K-steps several CTAs share.  A smaller workspace
// may leave the partial tiles out: the GEMM then keeps every tile whole.
struct WsLayout {
  size_t v_off, u_off, part_off, min_total, total;
};

constexpr size_t kFixedBytes = qlora::kWsFixedBytes;

WsLayout ws_layout(int op, int64_t M, int64_t in, int64_t out, int r) {
  WsLayout L{};
  const size_t mr = align256(static_cast<size_t>(M) * r * 2);
  size_t off = kFixedBytes;
  L.v_off = off;
  off += mr;
  size_t part = 0;
  if (op == QLORA_OP_FWD) {
    L.u_off = 0;
    if (!qlora::gemv_supported(M, in, out)) part = qlora::fwd_gemm_split_bytes(M, in, out, r);
  } else {
    L.u_off = off;
    off += mr;
    part = qlora::dx_gemm_split_bytes(M, in, out, r);
  }
  L.part_off = off;
  L.min_total = off;
  L.total = off + align256(part);
  return L;
}

struct SplitRegion {
  uint32_t* counters;
  void* partials;
  size_t partial_bytes;
};

// The GEMM's hand-over buffers: the partial tiles only in a full-size workspace.
SplitRegion split_region(void* ws, size_t ws_bytes, const WsLayout& L) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  SplitRegion R{reinterpret_cast<uint32_t*>(base + qlora::kWsStatusBytes), nullptr, 0};
  if (ws_bytes >= L.total && L.total > L.min_total) {
    R.partials = base + L.part_off;
    R.partial_bytes = ws_bytes - L.part_off;
  }
  return R;
}

std::atomic<uint64_t> g_launches{0};

struct TimingHook {
  int which = 0;
  void* const* starts = nullptr;
  void* const* stops = nullptr;
  int n = 0, i = 0;
} g_hook;

}  // namespace

namespace qlora {
size_t ws_min_bytes(int op, int64_t M, int64_t in, int64_t out, int r) {
  if ((op != QLORA_OP_FWD && op != QLORA_OP_BWD) || !linear_shape_ok(M, in, out, r)) return 0;
  return ws_layout(op, M, in, out, r).min_total;
}
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
// Record `e` on `stream`; inside a stream capture as an external event node, so
// that it is recorded at every replay of the graph.
static void record_event(void* e, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(e), stream, cudaEventRecordExternal);
  else
    cudaEventRecord(static_cast<cudaEvent_t>(e), stream);
}
void timing_before(int which, cudaStream_t stream) {
  if (g_hook.which == which && g_hook.i < g_hook.n) record_event(g_hook.starts[g_hook.i], stream);
}
void timing_after(int which, cudaStream_t stream) {
  if (g_hook.which == which && g_hook.i < g_hook.n) {
    record_event(g_hook.stops[g_hook.i], stream);
    ++g_hook.i;
  }
}
}  // namespace qlora

extern "C" {

qlora_status qlora_time_kernel(int which, void* const* starts, void* const* stops, int n) {
  if (n < 0 || which < QLORA_KERNEL_QUANTIZE || which > QLORA_KERNEL_GEMV) return QLORA_ERR_INVALID_ARG;
  if (n > 0 && (!starts || !stops)) return QLORA_ERR_INVALID_ARG;
  g_hook.which = n > 0 ? which : 0;
  g_hook.starts = starts;
  g_hook.stops = stops;
  g_hook.n = n;
  g_hook.i = 0;
  return QLORA_OK;
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_SHAPE: return "unsupported shape";
    case QLORA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "bounded wait in a kernel timed out";
  }
  return "unknown status";
}

void qlora_nf4_codebook(float out[16]) {
  if (!out) return;
  for (int i = 0; i < 16; ++i) out[i] = qlora::nf4_level(i);
}

int64_t qlora_adapter_params(int64_t in, int64_t out, int r) { return static_cast<int64_t>(r) * (in + out); }

size_t qlora_workspace_bytes(int op, int64_t M, int64_t in, int64_t out, int r) {
  if ((op != QLORA_OP_FWD && op != QLORA_OP_BWD) || !linear_shape_ok(M, in, out, r)) return 0;
  return ws_layout(op, M, in, out, r).total;
}

qlora_status qlora_gemm_set_ctas(int ctas) {
  if (ctas < 0) return QLORA_ERR_INVALID_ARG;
  qlora::set_gemm_ctas(ctas);
  return QLORA_OK;
}

qlora_status qlora_ws_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < qlora::kWsFixedBytes) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(ws));
  QLORA_CUDA(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_ws_status(void* ws, void* stream) {
  if (!ws) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(ws));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  QLORA_CUDA(cudaStreamSynchronize(s));
  uint32_t flag = 0;
  QLORA_CUDA(cudaMemcpy(&flag, ws, sizeof(flag), cudaMemcpyDeviceToHost));
  if (flag != 0) {
    QLORA_CUDA(cudaMemset(ws, 0, sizeof(flag)));
    return QLORA_ERR_TIMEOUT;
  }
  return QLORA_OK;
}

qlora_status qlora_quantize_status(void* stream) {
  QLORA_TRY(check_device());
  uint32_t flags = 0;
  QLORA_CUDA(qlora::quantize_status_take(static_cast<cudaStream_t>(stream), &flags));
  return flags != 0 ? QLORA_ERR_TIMEOUT : QLORA_OK;
}

qlora_status qlora_selftest_wait_timeout(void* ws, size_t ws_bytes, int kind, uint32_t limit_us, void* stream) {
  if (kind != 0 && kind != 1) return QLORA_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 1000000u) return QLORA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < qlora::kWsFixedBytes) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(ws));
  uint8_t* base = static_cast<uint8_t*>(ws);
  // the last of the GEMM's counters: zero, and advanced by nothing here
  const uint32_t* counter =
      reinterpret_cast<const uint32_t*>(base + qlora::kWsStatusBytes) + (qlora::kMaxGemmCtas - 1);
  QLORA_CUDA(qlora::launch_selftest_wait(reinterpret_cast<uint32_t*>(base), counter, kind,
                                         static_cast<uint64_t>(limit_us) * 1000u, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4(const float* W0, int64_t in, int64_t out, uint8_t* codes, uint8_t* dq_codes,
                                float* dq_scales, void* stream) {
  return qlora_quantize_nf4_ex(W0, in, out, codes, dq_codes, dq_scales, QLORA_DQ_E4M3, stream);
}

qlora_status qlora_quantize_nf4_ex(const float* W0, int64_t in, int64_t out, uint8_t* codes, uint8_t* dq_codes,
                                   float* dq_scales, int dq_format, void* stream) {
  if (!W0 || !codes || !dq_codes || !dq_scales) return QLORA_ERR_INVALID_ARG;
  if (dq_format != QLORA_DQ_E4M3 && dq_format != QLORA_DQ_U8) return QLORA_ERR_INVALID_ARG;
  if (in < 1 || out < 1 || in > (int64_t(1) << 40) / out || (in * out) % QLORA_BLOCK != 0) return QLORA_ERR_SHAPE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(W0));
  QLORA_TRY(check_ptr(codes));
  QLORA_TRY(check_ptr(dq_codes));
  QLORA_TRY(check_ptr(dq_scales));
  QLORA_CUDA(qlora::launch_quantize_nf4(W0, in * out, codes, dq_codes, dq_scales, static_cast<cudaStream_t>(stream),
                                        dq_format == QLORA_DQ_U8));
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4_batch(const qlora_quantize_job* jobs, int n, int dq_format, void* stream) {
  if (n < 0 || (n > 0 && !jobs)) return QLORA_ERR_INVALID_ARG;
  if (dq_format != QLORA_DQ_E4M3 && dq_format != QLORA_DQ_U8) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const qlora_quantize_job& j = jobs[i];
    if (!j.W0 || !j.codes || !j.dq_codes || !j.dq_scales) return QLORA_ERR_INVALID_ARG;
    if (j.in < 1 || j.out < 1 || j.in > (int64_t(1) << 40) / j.out || (j.in * j.out) % QLORA_BLOCK != 0)
      return QLORA_ERR_SHAPE;
  }
  if (n == 0) return QLORA_OK;
  QLORA_TRY(check_device());
  // The pointers of each launch's weights are checked just before that launch, so
  // that the host checks of the next ones overlap the device work (a pointer
  // error stops the batch there: the launches before it have been issued).
  std::vector<qlora::QuantizeJob> q(static_cast<size_t>(n));
  for (int c = 0; c < n; c += qlora::kQMaxJobs) {
    const int cn = std::min(qlora::kQMaxJobs, n - c);
    for (int i = c; i < c + cn; ++i) {
      const qlora_quantize_job& j = jobs[i];
      QLORA_TRY(check_ptr(j.W0));
      QLORA_TRY(check_ptr(j.codes));
      QLORA_TRY(check_ptr(j.dq_codes));
      QLORA_TRY(check_ptr(j.dq_scales));
      q[i] = qlora::QuantizeJob{j.W0, j.in * j.out, j.codes, j.dq_codes, j.dq_scales};
    }
    QLORA_CUDA(qlora::launch_quantize_nf4_batch(q.data() + c, cn, static_cast<cudaStream_t>(stream),
                                                dq_format == QLORA_DQ_U8));
  }
  return QLORA_OK;
}

static bool int_shape_ok(int64_t in, int64_t out) {
  return in >= 1 && out >= 1 && in <= (int64_t(1) << 40) / out && (in * out) % 16 == 0;
}

qlora_status qlora_quantize_int(const float* W0, int64_t in, int64_t out, int bits, uint8_t* codes, float* scales,
                                void* stream) {
  if (!W0 || !codes || !scales || bits < 2 || bits > 4) return QLORA_ERR_INVALID_ARG;
  if (!int_shape_ok(in, out)) return QLORA_ERR_SHAPE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(W0));
  QLORA_TRY(check_ptr(codes));
  QLORA_TRY(check_ptr(scales));
  QLORA_CUDA(qlora::launch_int_quantize(W0, in * out, bits, codes, scales, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_dequantize_int(const uint8_t* codes, const float* scales, int64_t in, int64_t out, void* W_out,
                                  int out_dtype, void* stream) {
  if (!codes || !scales || !W_out || (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16))
    return QLORA_ERR_INVALID_ARG;
  if (!int_shape_ok(in, out)) return QLORA_ERR_SHAPE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_ptr(codes));
  QLORA_TRY(check_ptr(scales));
  QLORA_TRY(check_ptr(W_out));
  QLORA_CUDA(qlora::launch_int_dequantize(codes, scales, in * out, out_dtype == QLORA_BF16, W_out,
                                          static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_dequantize(const qlora_nf4_weight* w, void* W_out, int out_dtype, void* stream) {
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16 || !W_out) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(W_out));
  QLORA_CUDA(qlora::launch_dequantize(w->codes, w->dq_codes, w->dq_scales, w->in * w->out, out_dtype == QLORA_BF16,
                                      W_out, static_cast<cudaStream_t>(stream), w->dq_format));
  return QLORA_OK;
}

qlora_status qlora_loftq_residual(const float* W0, const qlora_nf4_weight* w, float* R, void* stream) {
  if (!W0 || !R) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(W0));
  QLORA_TRY(check_ptr(R));
  QLORA_CUDA(qlora::launch_dequantize(w->codes, w->dq_codes, w->dq_scales, w->in * w->out, false, R,
                                      static_cast<cudaStream_t>(stream), w->dq_format, W0));
  return QLORA_OK;
}

qlora_status qlora_loftq_split(const float* U, int64_t ldu, const float* S, const float* Vh, int64_t ldv, int64_t in,
                               int64_t out, int r, uint16_t* A, uint16_t* B, void* stream) {
  if (!U || !S || !Vh || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (in < 1 || out < 1 || r < 1 || ldu < r || ldv < out || in > (int64_t(1) << 40) / (ldu > r ? ldu : r) ||
      static_cast<int64_t>(r) > (int64_t(1) << 40) / (ldv > out ? ldv : out) || (in + out) * r >= (int64_t(1) << 40))
    return QLORA_ERR_SHAPE;
  QLORA_TRY(check_device());
  for (const void* p : {static_cast<const void*>(U), static_cast<const void*>(S), static_cast<const void*>(Vh),
                        static_cast<const void*>(A), static_cast<const void*>(B)})
    QLORA_TRY(check_ptr(p));
  QLORA_CUDA(qlora::launch_loftq_split(U, ldu, S, Vh, ldv, in, out, r, A, B, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_merge(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, void* W_out,
                         int out_dtype, void* stream) {
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16 || !A || !B || !W_out) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  if (!linear_shape_ok(1, w->in, w->out, r) || w->in > (int64_t(1) << 21)) return QLORA_ERR_SHAPE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(A));
  QLORA_TRY(check_ptr(B));
  QLORA_TRY(check_ptr(W_out));
  QLORA_CUDA(qlora::launch_merge(w->codes, w->dq_codes, w->dq_scales, A, B, r, w->in, w->out,
                                 out_dtype == QLORA_BF16, W_out, static_cast<cudaStream_t>(stream), w->dq_format));
  return QLORA_OK;
}

// Options of the _ex calls (adapter scale, flags, dropout), checked on the host.
struct LinearOpts {
  float scale = 1.0f;
  bool accumulate = false;
  qlora::Dropout drop;
};

static qlora_status read_opts(const qlora_linear_opts* o, LinearOpts& lo) {
  lo = LinearOpts{};
  if (!o) return QLORA_OK;
  if (!std::isfinite(o->adapter_scale) || (o->flags & ~static_cast<uint32_t>(QLORA_ACCUMULATE_GRADS)) != 0u)
    return QLORA_ERR_INVALID_ARG;
  lo.scale = o->adapter_scale;
  lo.accumulate = (o->flags & QLORA_ACCUMULATE_GRADS) != 0u;
  if (o->dropout_keep) {
    if (!(o->dropout_p >= 0.0f && o->dropout_p < 1.0f)) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_ptr(o->dropout_keep));
    lo.drop.keep = o->dropout_keep;
    lo.drop.keep_scale = static_cast<float>(1.0 / (1.0 - static_cast<double>(o->dropout_p)));
  }
  return QLORA_OK;
}

static qlora_status fwd_impl(const qlora_nf4_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                             const uint16_t* B, int r, uint16_t* Y, uint16_t* V_save, void* ws, size_t ws_bytes,
                             void* stream, const LinearOpts& lo) {
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  if (!linear_shape_ok(M, w->in, w->out, r)) return QLORA_ERR_SHAPE;
  if (!ws || ws_bytes < ws_layout(QLORA_OP_FWD, M, w->in, w->out, r).min_total) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(X));
  QLORA_TRY(check_ptr(A));
  QLORA_TRY(check_ptr(B));
  QLORA_TRY(check_ptr(Y));
  QLORA_TRY(check_ptr(V_save, false));
  const WsLayout L = ws_layout(QLORA_OP_FWD, M, w->in, w->out, r);
  if (!ws || ws_bytes < L.min_total) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_ptr(ws));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  uint16_t* V = V_save ? V_save : reinterpret_cast<uint16_t*>(base + L.v_off);
  const WeightView wv = view(w);
  if (w->dq_format != QLORA_FMT_INT16 && qlora::gemv_supported(M, w->in, w->out)) {
    QLORA_CUDA(qlora::launch_xa_small(X, A, M, w->in, r, V, s, lo.scale, lo.drop));
    QLORA_CUDA(qlora::launch_gemv(wv, X, V, B, M, r, Y, status, s));
  } else {
    QLORA_CUDA(qlora::launch_xa(X, A, M, w->in, r, V, status, s, lo.scale, lo.drop));
    const SplitRegion sr = split_region(ws, ws_bytes, L);
    QLORA_CUDA(qlora::launch_fwd_gemm(wv, X, V, B, M, r, Y, status, sr.counters, sr.partials, sr.partial_bytes, s));
  }
  return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_nf4_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                              const uint16_t* B, int r, uint16_t* Y, uint16_t* V_save, void* ws, size_t ws_bytes,
                              void* stream) {
  return fwd_impl(w, X, M, A, B, r, Y, V_save, ws, ws_bytes, stream, LinearOpts{});
}

qlora_status qlora_linear_fwd_ex(const qlora_nf4_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                                 const uint16_t* B, int r, uint16_t* Y, uint16_t* V_save,
                                 const qlora_linear_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  LinearOpts lo;
  QLORA_TRY(read_opts(opts, lo));
  if (lo.accumulate) return QLORA_ERR_INVALID_ARG;   // the forward has no gradients
  return fwd_impl(w, X, M, A, B, r, Y, V_save, ws, ws_bytes, stream, lo);
}

static qlora_status bwd_impl(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V, const uint16_t* dY,
                             int64_t M, const uint16_t* A, const uint16_t* B, int r, uint16_t* dX, float* dA,
                             float* dB, void* ws, size_t ws_bytes, void* stream, const LinearOpts& lo) {
  if (!X || !dY || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  if (!linear_shape_ok(M, w->in, w->out, r)) return QLORA_ERR_SHAPE;
  if (!ws || ws_bytes < ws_layout(QLORA_OP_BWD, M, w->in, w->out, r).min_total) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(X));
  QLORA_TRY(check_ptr(V, false));
  QLORA_TRY(check_ptr(dY));
  QLORA_TRY(check_ptr(A));
  QLORA_TRY(check_ptr(B));
  QLORA_TRY(check_ptr(dX, false));
  QLORA_TRY(check_ptr(dA));
  QLORA_TRY(check_ptr(dB));
  const WsLayout L = ws_layout(QLORA_OP_BWD, M, w->in, w->out, r);
  if (!ws || ws_bytes < L.min_total) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_ptr(ws));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  uint16_t* U = reinterpret_cast<uint16_t*>(base + L.u_off);
  const WeightView wv = view(w);
  if (!V) {
    uint16_t* Vw = reinterpret_cast<uint16_t*>(base + L.v_off);
    QLORA_CUDA(qlora::launch_xa(X, A, M, w->in, r, Vw, status, s, lo.scale, lo.drop));
    V = Vw;
  }
  QLORA_CUDA(qlora::launch_dybt(dY, B, M, w->out, r, U, status, s, lo.scale, lo.drop));
  QLORA_CUDA(qlora::launch_dbda(V, dY, X, U, M, w->in, w->out, r, dA, dB, status, s, nullptr, nullptr,
                                lo.accumulate));
  if (dX) {
    const SplitRegion sr = split_region(ws, ws_bytes, L);
    QLORA_CUDA(qlora::launch_dx_gemm(wv, dY, U, A, M, r, dX, status, sr.counters, sr.partials, sr.partial_bytes, s));
  }
  return QLORA_OK;
}

qlora_status qlora_linear_bwd(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V, const uint16_t* dY,
                              int64_t M, const uint16_t* A, const uint16_t* B, int r, uint16_t* dX, float* dA,
                              float* dB, void* ws, size_t ws_bytes, void* stream) {
  return bwd_impl(w, X, V, dY, M, A, B, r, dX, dA, dB, ws, ws_bytes, stream, LinearOpts{});
}

qlora_status qlora_linear_bwd_ex(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V, const uint16_t* dY,
                                 int64_t M, const uint16_t* A, const uint16_t* B, int r, uint16_t* dX, float* dA,
                                 float* dB, const qlora_linear_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  LinearOpts lo;
  QLORA_TRY(read_opts(opts, lo));
  return bwd_impl(w, X, V, dY, M, A, B, r, dX, dA, dB, ws, ws_bytes, stream, lo);
}

qlora_status qlora_linear_bwd_adam(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* V,
                                   const uint16_t* dY, int64_t M, uint16_t* A, uint16_t* B, int r, uint16_t* dX,
                                   const qlora_adam_state* st, const qlora_adam_hparams* hp,
                                   const qlora_linear_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !dY || !A || !B || !st || !hp) return QLORA_ERR_INVALID_ARG;
  LinearOpts lo;
  QLORA_TRY(read_opts(opts, lo));
  if (lo.accumulate) return QLORA_ERR_INVALID_ARG;   // the step consumes the gradients
  if (!st->A32 || !st->B32 || !st->mA || !st->vA || !st->mB || !st->vB) return QLORA_ERR_INVALID_ARG;
  if (!(hp->lr >= 0.0f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
      !(hp->eps > 0.0f) || !(hp->weight_decay >= 0.0f) || hp->step < 1 || !std::isfinite(hp->lr))
    return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(check_weight_shape(w));
  if (!linear_shape_ok(M, w->in, w->out, r)) return QLORA_ERR_SHAPE;
  if (!ws || ws_bytes < ws_layout(QLORA_OP_BWD, M, w->in, w->out, r).min_total) return QLORA_ERR_WORKSPACE;
  QLORA_TRY(check_device());
  QLORA_TRY(check_weight(w));
  QLORA_TRY(check_ptr(X));
  QLORA_TRY(check_ptr(V, false));
  QLORA_TRY(check_ptr(dY));
  QLORA_TRY(check_ptr(A));
  QLORA_TRY(check_ptr(B));
  QLORA_TRY(check_ptr(dX, false));
  for (const float* q : {st->A32, st->B32, st->mA, st->vA, st->mB, st->vB}) QLORA_TRY(check_ptr(q));
  const WsLayout L = ws_layout(QLORA_OP_BWD, M, w->in, w->out, r);
  QLORA_TRY(check_ptr(ws));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  uint16_t* U = reinterpret_cast<uint16_t*>(base + L.u_off);
  const WeightView wv = view(w);

  // bias corrections and the constants of the rule, in double then rounded once
  const double t = static_cast<double>(hp->step);
  qlora::AdamParams pa{};
  pa.lr = hp->lr;
  pa.b1 = hp->beta1;
  pa.b2 = hp->beta2;
  pa.omb1 = static_cast<float>(1.0 - static_cast<double>(hp->beta1));
  pa.omb2 = static_cast<float>(1.0 - static_cast<double>(hp->beta2));
  pa.eps = hp->eps;
  pa.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * static_cast<double>(hp->weight_decay));
  pa.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp->beta1), t));
  pa.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp->beta2), t));
  if (!(pa.bc1 > 0.0f) || !(pa.bc2 > 0.0f)) return QLORA_ERR_INVALID_ARG;
  qlora::AdamParams pA = pa, pB = pa;
  pA.theta = st->A32;
  pA.m = st->mA;
  pA.v = st->vA;
  pA.p16 = A;
  pB.theta = st->B32;
  pB.m = st->mB;
  pB.v = st->vB;
  pB.p16 = B;

  // Every read of A or B comes before its update: V, U and dX read them first,
  // then one launch takes the B and A steps.
  if (!V) {
    uint16_t* Vw = reinterpret_cast<uint16_t*>(base + L.v_off);
    QLORA_CUDA(qlora::launch_xa(X, A, M, w->in, r, Vw, status, s, lo.scale, lo.drop));
    V = Vw;
  }
  QLORA_CUDA(qlora::launch_dybt(dY, B, M, w->out, r, U, status, s, lo.scale, lo.drop));
  if (dX) {
    const SplitRegion sr = split_region(ws, ws_bytes, L);
    QLORA_CUDA(qlora::launch_dx_gemm(wv, dY, U, A, M, r, dX, status, sr.counters, sr.partials, sr.partial_bytes, s));
  }
  QLORA_CUDA(qlora::launch_dbda(V, dY, X, U, M, w->in, w->out, r, nullptr, nullptr, status, s, &pA, &pB));
  return QLORA_OK;
}

}  // extern "C"
