// Forward of the adapted layer for callers that cannot allocate device memory.
//
// qlora_linear_fwd needs a caller-provided workspace.  Some callers have no way
// to provide one: a host program linked against this library through its C ABI
// that has no device allocator of its own, a plugin or custom operator inside a
// runtime that owns all device memory and exposes no scratch allocator, or a
// latency-critical path where a cudaMalloc (which may synchronise the device)
// is not acceptable once the program is running.  For them this file keeps a
// fixed-size scratch array in the library's own device memory and runs the
// same forward with it.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its kStaticWsBytes until the process exits.  In host code the
// array's name is only a host-side stand-in, so its device address is looked up
// with cudaGetSymbolAddress on the device that is current (cheap, and correct
// again after the device's context was reset).  The lookup is skipped while
// `stream` is capturing; the address kept per device by an earlier call is used
// then.  All calls share the array
// and it keeps the previous call's contents, so each call first zeroes the
// GEMM's split counters, which must start at zero; the status word is left as
// it is until qlora_static_ws_status reads and clears it.  Two calls whose work
// overlaps on the GPU (different streams, or different host threads) race on
// the array.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qlora.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticWsBytes = QLORA_STATIC_WS_BYTES;

static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_setup_mutex;
void* g_static_ws_addr[64] = {};

// Device address of g_static_ws on the current device: looked up again outside
// a capture of `stream`, taken from the per-device cache inside one.
qlora_status static_ws_address(void** out, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return QLORA_ERR_UNSUPPORTED_DEVICE;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (cs == cudaStreamCaptureStatusNone || !g_static_ws_addr[dev]) {
    if (cs != cudaStreamCaptureStatusNone) return QLORA_ERR_INVALID_ARG;   // no earlier call on this device
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    g_static_ws_addr[dev] = ptr;
  }
  *out = g_static_ws_addr[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" qlora_status qlora_linear_fwd_static_ws(const qlora_nf4_weight* w, const uint16_t* X, int64_t M,
                                                   const uint16_t* A, const uint16_t* B, int r, uint16_t* Y,
                                                   uint16_t* V_save, void* stream) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  // the smallest workspace the forward accepts (everything but the GEMM's split
  // partial tiles): the GEMM keeps its tiles whole here
  const size_t need = qlora::ws_min_bytes(QLORA_OP_FWD, M, w->in, w->out, r);
  if (need == 0) return QLORA_ERR_SHAPE;
  if (need > kStaticWsBytes) return QLORA_ERR_WORKSPACE;   // larger than the fixed array
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  const qlora_status st = static_ws_address(&ws, s);
  if (st != QLORA_OK) return st;
  if (cudaMemsetAsync(static_cast<unsigned char*>(ws) + qlora::kWsStatusBytes, 0, qlora::kWsCounterBytes, s) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  return qlora_linear_fwd(w, X, M, A, B, r, Y, V_save, ws, need, stream);
}

extern "C" qlora_status qlora_static_ws_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  const qlora_status st = static_ws_address(&ws, s);
  if (st != QLORA_OK) return st;
  return qlora_ws_status(ws, stream);
}
