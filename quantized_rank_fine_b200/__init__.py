"""Python binding of libqlora, the QLoRA adapted linear layer for B200 (sm_100a).

Argument marshalling only: every function passes device pointers, sizes and the
current CUDA stream to the C ABI declared in ``include/qlora.h`` and raises
``QLoRAError`` on a non-zero status.  PyTorch provides device memory and
streams; all arithmetic runs in the library's CUDA kernels.  There is no CPU
path: importing works without a GPU (for the build and host-side checks), but
every call that launches work needs ``libqlora.so`` and an sm_100 device, and
fails loudly otherwise.
"""

from __future__ import annotations

import ctypes
import os
from contextlib import nullcontext as _nullcontext
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_F32, QLORA_BF16 = 0, 1
QLORA_OP_FWD, QLORA_OP_BWD = 1, 2
BLOCK, GROUP = 64, 256

STATUS_NAMES = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGNMENT",
    4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_UNSUPPORTED_DEVICE", 6: "QLORA_ERR_CUDA",
    7: "QLORA_ERR_TIMEOUT",
}

# Every symbol the header declares.
EXPORTS = (
    "qlora_quantize_nf4", "qlora_dequantize", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_merge",
    "qlora_workspace_bytes", "qlora_ws_init", "qlora_ws_status", "qlora_nf4_codebook",
    "qlora_adapter_params", "qlora_status_string", "qlora_time_kernel", "qlora_launch_count",
    "qlora_linear_fwd_static_ws", "qlora_linear_bwd_adam", "qlora_linear_fwd_ex", "qlora_linear_bwd_ex",
    "qlora_gemm_set_ctas", "qlora_quantize_nf4_ex", "qlora_quantize_int", "qlora_dequantize_int",
    "qlora_static_ws_status", "qlora_quantize_status", "qlora_selftest_wait_timeout",
    "qlora_loftq_residual", "qlora_loftq_split", "qlora_quantize_nf4_batch",
)

# Weight formats (NF4Weight.dq_format): NF4 with E4M3 or linear uint8 absmax
# codes, or the symmetric INT format of qlora_quantize_int (one scale per 16).
QLORA_DQ_E4M3, QLORA_DQ_U8, QLORA_FMT_INT16 = 0, 1, 2

# Flag of qlora_linear_opts.flags.
QLORA_ACCUMULATE_GRADS = 1

# Kernel ids of qlora_time_kernel.
KERNEL_QUANTIZE, KERNEL_DEQUANTIZE, KERNEL_MERGE, KERNEL_FWD_GEMM, KERNEL_DX_GEMM, KERNEL_RANK_R = 1, 2, 3, 4, 5, 6
KERNEL_GEMV = 7


class QLoRAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class _Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("dq_codes", ctypes.c_void_p), ("dq_scales", ctypes.c_void_p),
                ("in_", ctypes.c_int64), ("out", ctypes.c_int64), ("dq_format", ctypes.c_int32)]


class _QuantizeJob(ctypes.Structure):
    _fields_ = [("W0", ctypes.c_void_p), ("in_", ctypes.c_int64), ("out", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("dq_codes", ctypes.c_void_p), ("dq_scales", ctypes.c_void_p)]


class _AdamHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


class _LinearOpts(ctypes.Structure):
    _fields_ = [("adapter_scale", ctypes.c_float), ("flags", ctypes.c_uint32),
                ("dropout_keep", ctypes.c_void_p), ("dropout_p", ctypes.c_float)]


class _AdamState(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("A32", "B32", "mA", "vA", "mB", "vB")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libqlora.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m quantized_rank_fine_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        wp = ctypes.POINTER(_Weight)
        sig = {
            "qlora_quantize_nf4": (i32, [vp, i64, i64, vp, vp, vp, vp]),
            "qlora_dequantize": (i32, [wp, vp, i32, vp]),
            "qlora_linear_fwd": (i32, [wp, vp, i64, vp, vp, i32, vp, vp, vp, sz, vp]),
            "qlora_linear_bwd": (i32, [wp, vp, vp, vp, i64, vp, vp, i32, vp, vp, vp, vp, sz, vp]),
            "qlora_merge": (i32, [wp, vp, vp, i32, vp, i32, vp]),
            "qlora_workspace_bytes": (sz, [i32, i64, i64, i64, i32]),
            "qlora_ws_init": (i32, [vp, sz, vp]),
            "qlora_ws_status": (i32, [vp, vp]),
            "qlora_nf4_codebook": (None, [ctypes.POINTER(ctypes.c_float)]),
            "qlora_adapter_params": (i64, [i64, i64, i32]),
            "qlora_status_string": (ctypes.c_char_p, [i32]),
            "qlora_time_kernel": (i32, [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32]),
            "qlora_launch_count": (ctypes.c_uint64, []),
            "qlora_gemm_set_ctas": (i32, [i32]),
            "qlora_quantize_nf4_ex": (i32, [vp, i64, i64, vp, vp, vp, i32, vp]),
            "qlora_quantize_nf4_batch": (i32, [ctypes.POINTER(_QuantizeJob), i32, i32, vp]),
            "qlora_quantize_int": (i32, [vp, i64, i64, i32, vp, vp, vp]),
            "qlora_dequantize_int": (i32, [vp, vp, i64, i64, vp, i32, vp]),
            "qlora_linear_fwd_static_ws": (i32, [wp, vp, i64, vp, vp, i32, vp, vp, vp]),
            "qlora_static_ws_status": (i32, [vp]),
            "qlora_loftq_residual": (i32, [vp, wp, vp, vp]),
            "qlora_loftq_split": (i32, [vp, i64, vp, vp, i64, i64, i64, i32, vp, vp, vp]),
            "qlora_quantize_status": (i32, [vp]),
            "qlora_selftest_wait_timeout": (i32, [vp, sz, i32, ctypes.c_uint32, vp]),
            "qlora_linear_bwd_adam": (i32, [wp, vp, vp, vp, i64, vp, vp, i32, vp, ctypes.POINTER(_AdamState),
                                            ctypes.POINTER(_AdamHparams), ctypes.POINTER(_LinearOpts), vp, sz,
                                            vp]),
            "qlora_linear_fwd_ex": (i32, [wp, vp, i64, vp, vp, i32, vp, vp, ctypes.POINTER(_LinearOpts), vp, sz,
                                          vp]),
            "qlora_linear_bwd_ex": (i32, [wp, vp, vp, vp, i64, vp, vp, i32, vp, vp, vp,
                                          ctypes.POINTER(_LinearOpts), vp, sz, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise QLoRAError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


@dataclass
class NF4Weight:
    """The frozen quantised weight: packed codes, 8-bit absmax codes (E4M3, or
    linear uint8 with dq_format = QLORA_DQ_U8), fp32 group scales."""
    codes: torch.Tensor       # uint8 [in*out/2]
    dq_codes: torch.Tensor    # uint8 [in*out/64]
    dq_scales: torch.Tensor   # float32 [ceil(in*out/64/256)]
    n_in: int
    n_out: int
    dq_format: int = 0        # QLORA_DQ_E4M3

    def c_struct(self) -> _Weight:
        return _Weight(_ptr(self.codes), _ptr(self.dq_codes), _ptr(self.dq_scales), self.n_in, self.n_out,
                       self.dq_format)


def qlora_nf4_codebook() -> list:
    buf = (ctypes.c_float * 16)()
    lib().qlora_nf4_codebook(buf)
    return list(buf)


def qlora_adapter_params(n_in: int, n_out: int, r: int) -> int:
    return lib().qlora_adapter_params(n_in, n_out, r)


def qlora_status_string(status: int) -> str:
    return lib().qlora_status_string(status).decode()


def qlora_launch_count() -> int:
    return lib().qlora_launch_count()


def qlora_gemm_set_ctas(ctas: int) -> None:
    """Most CTAs the fused GEMMs use (0: one per SM); a testing/tuning knob."""
    _check(lib().qlora_gemm_set_ctas(ctas), "qlora_gemm_set_ctas")


class KernelTimer:
    """Bracket the next n launches of one kernel kind with CUDA events recorded
    by the library on the launching stream (qlora_time_kernel)."""

    def __init__(self, which: int, n: int):
        self.starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        self.stops = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in self.starts + self.stops:
            e.record()          # materialise the cudaEvent_t handles
        self._s = (ctypes.c_void_p * n)(*[e.cuda_event for e in self.starts])
        self._e = (ctypes.c_void_p * n)(*[e.cuda_event for e in self.stops])
        _check(lib().qlora_time_kernel(which, self._s, self._e, n), "qlora_time_kernel")
        self.n = n

    def disarm(self):
        lib().qlora_time_kernel(KERNEL_QUANTIZE, None, None, 0)

    def times_ms(self, count: int | None = None) -> list:
        count = self.n if count is None else count
        return [self.starts[i].elapsed_time(self.stops[i]) for i in range(count)]


def qlora_workspace_bytes(op: int, M: int, n_in: int, n_out: int, r: int) -> int:
    return lib().qlora_workspace_bytes(op, M, n_in, n_out, r)


class Workspace:
    """Caller-owned scratch of the forward/backward calls (a device uint8 tensor),
    grown on demand and initialised once through qlora_ws_init."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int, stream=None) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            _check(lib().qlora_ws_init(_ptr(self.buf), self.buf.numel(), _stream(stream)), "qlora_ws_init")
        return self.buf

    def status(self, stream=None) -> int:
        if self.buf is None:
            return 0
        return lib().qlora_ws_status(_ptr(self.buf), _stream(stream))


def qlora_quantize_nf4(W0: torch.Tensor, stream=None, out: NF4Weight | None = None,
                       dq_format: int | None = None) -> NF4Weight:
    """W0 fp32 (in, out) on the GPU -> NF4Weight (outputs allocated unless given).
    dq_format: QLORA_DQ_E4M3 (default) or QLORA_DQ_U8 (linear uint8 absmax codes);
    a given `out` keeps its own format unless one is passed."""
    n_in, n_out = W0.shape
    n = n_in * n_out
    if out is None:
        dev = W0.device
        out = NF4Weight(torch.empty(n // 2, dtype=torch.uint8, device=dev),
                        torch.empty(n // BLOCK, dtype=torch.uint8, device=dev),
                        torch.empty((n // BLOCK + GROUP - 1) // GROUP, dtype=torch.float32, device=dev),
                        n_in, n_out)
    if dq_format is not None:
        out.dq_format = dq_format
    if out.dq_format == QLORA_DQ_E4M3:
        _check(lib().qlora_quantize_nf4(_ptr(W0), n_in, n_out, _ptr(out.codes), _ptr(out.dq_codes),
                                        _ptr(out.dq_scales), _stream(stream)), "qlora_quantize_nf4")
    else:
        _check(lib().qlora_quantize_nf4_ex(_ptr(W0), n_in, n_out, _ptr(out.codes), _ptr(out.dq_codes),
                                           _ptr(out.dq_scales), out.dq_format, _stream(stream)),
               "qlora_quantize_nf4_ex")
    return out


def qlora_quantize_nf4_batch(W0s, stream=None, outs=None, dq_format: int = QLORA_DQ_E4M3) -> list:
    """Several fp32 (in, out) weights on the GPU -> one NF4Weight each, in as few
    launches as the library needs (qlora_quantize_nf4_batch); the same bytes as
    quantising them one by one."""
    if outs is None:
        outs = []
        for W0 in W0s:
            n_in, n_out = W0.shape
            n, dev = n_in * n_out, W0.device
            outs.append(NF4Weight(torch.empty(n // 2, dtype=torch.uint8, device=dev),
                                  torch.empty(n // BLOCK, dtype=torch.uint8, device=dev),
                                  torch.empty((n // BLOCK + GROUP - 1) // GROUP, dtype=torch.float32, device=dev),
                                  n_in, n_out))
    jobs = (_QuantizeJob * max(1, len(W0s)))()
    for i, (W0, o) in enumerate(zip(W0s, outs)):
        o.dq_format = dq_format
        jobs[i] = _QuantizeJob(_ptr(W0), W0.shape[0], W0.shape[1], _ptr(o.codes), _ptr(o.dq_codes),
                               _ptr(o.dq_scales))
    _check(lib().qlora_quantize_nf4_batch(jobs, len(W0s), dq_format, _stream(stream)), "qlora_quantize_nf4_batch")
    return outs


def qlora_quantize_status(stream=None) -> int:
    """Synchronise the stream and read (then clear) the quantisers' device status
    word: 0, or QLORA_ERR_TIMEOUT if a bounded wait in a quantisation gave up."""
    return lib().qlora_quantize_status(_stream(stream))


def qlora_selftest_wait_timeout(workspace: "Workspace", kind: int, limit_us: int, stream=None) -> None:
    """Run one bounded wait that can only run out (kind 0: an mbarrier, kind 1: a
    workspace counter), with a limit of limit_us; afterwards workspace.status()
    reports QLORA_ERR_TIMEOUT."""
    buf = workspace.get(1280, stream)
    _check(lib().qlora_selftest_wait_timeout(_ptr(buf), buf.numel(), kind, limit_us, _stream(stream)),
           "qlora_selftest_wait_timeout")


def qlora_quantize_int(W0: torch.Tensor, bits: int, stream=None, out=None):
    """Symmetric uniform INT quantisation with one scale per 16 weights (bits 2,
    3 or 4; 2 is ternary): W0 fp32 (in, out) on the GPU -> (codes uint8
    [in*out/2], scales fp32 [in*out/16]), allocated unless `out` gives them."""
    n_in, n_out = W0.shape
    n = n_in * n_out
    if out is None:
        codes = torch.empty(n // 2, dtype=torch.uint8, device=W0.device)
        scales = torch.empty(n // 16, dtype=torch.float32, device=W0.device)
    else:
        codes, scales = out
    _check(lib().qlora_quantize_int(_ptr(W0), n_in, n_out, bits, _ptr(codes), _ptr(scales), _stream(stream)),
           "qlora_quantize_int")
    return codes, scales


def int_weight(codes: torch.Tensor, scales: torch.Tensor, n_in: int, n_out: int) -> "NF4Weight":
    """The weight descriptor of a qlora_quantize_int result, for the layer calls
    (forward, backward, dequantize, merge)."""
    return NF4Weight(codes, None, scales, n_in, n_out, QLORA_FMT_INT16)


def qlora_dequantize_int(codes: torch.Tensor, scales: torch.Tensor, n_in: int, n_out: int,
                         dtype=torch.float32, stream=None, out=None) -> torch.Tensor:
    """Dense w' (fp32) or bf16(w') of a weight from qlora_quantize_int."""
    code = QLORA_BF16 if dtype == torch.bfloat16 else QLORA_F32
    if out is None:
        out = torch.empty((n_in, n_out), dtype=dtype, device=codes.device)
    _check(lib().qlora_dequantize_int(_ptr(codes), _ptr(scales), n_in, n_out, _ptr(out), code, _stream(stream)),
           "qlora_dequantize_int")
    return out


def qlora_dequantize(w: NF4Weight, dtype=torch.float32, stream=None, out=None) -> torch.Tensor:
    code = QLORA_BF16 if dtype == torch.bfloat16 else QLORA_F32
    if out is None:
        out = torch.empty((w.n_in, w.n_out), dtype=dtype, device=w.codes.device)
    ws = w.c_struct()
    _check(lib().qlora_dequantize(ctypes.byref(ws), _ptr(out), code, _stream(stream)), "qlora_dequantize")
    return out


def qlora_merge(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, dtype=torch.float32, stream=None,
                out=None) -> torch.Tensor:
    code = QLORA_BF16 if dtype == torch.bfloat16 else QLORA_F32
    if out is None:
        out = torch.empty((w.n_in, w.n_out), dtype=dtype, device=w.codes.device)
    ws = w.c_struct()
    _check(lib().qlora_merge(ctypes.byref(ws), _ptr(A), _ptr(B), A.shape[1], _ptr(out), code, _stream(stream)),
           "qlora_merge")
    return out


def _opts(adapter_scale: float, accumulate: bool = False, dropout_keep=None, dropout_p: float = 0.0):
    return _LinearOpts(adapter_scale, QLORA_ACCUMULATE_GRADS if accumulate else 0,
                       _ptr(dropout_keep) if dropout_keep is not None else None, dropout_p)


def dropout_mask(M: int, r: int, p: float, generator=None, device="cuda") -> torch.Tensor:
    """A dropout keep mask for the low-rank intermediate: uint8 (M, r), 1 with
    probability 1 - p.  Pass the same mask to the forward and the backward of one
    micro-batch."""
    if not 0.0 <= p < 1.0:
        raise ValueError("p must lie in [0, 1)")
    u = torch.rand((M, r), generator=generator, device=device)
    return (u >= p).to(torch.uint8)


def qlora_linear_fwd(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, workspace: Workspace,
                     save_V: bool = True, stream=None, Y=None, V=None, adapter_scale: float = 1.0,
                     dropout_keep=None, dropout_p: float = 0.0):
    """Returns (Y, V) with V = s X A (None when save_V is False); s =
    adapter_scale (alpha / r), 1 for the plain layer.  With dropout_keep (uint8
    (M, r) on the device, 1 = keep) V is dropped out: s (X A) keep / (1 - p)."""
    M, r = X.shape[0], A.shape[1]
    if Y is None:
        Y = torch.empty((M, w.n_out), dtype=torch.bfloat16, device=X.device)
    if save_V and V is None:
        V = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    nb = qlora_workspace_bytes(QLORA_OP_FWD, M, w.n_in, w.n_out, r)
    buf = workspace.get(nb, stream)
    ws = w.c_struct()
    if adapter_scale == 1.0 and dropout_keep is None:
        _check(lib().qlora_linear_fwd(ctypes.byref(ws), _ptr(X), M, _ptr(A), _ptr(B), r, _ptr(Y),
                                      _ptr(V) if save_V else None, _ptr(buf), buf.numel(), _stream(stream)),
               "qlora_linear_fwd")
    else:
        o = _opts(adapter_scale, False, dropout_keep, dropout_p)
        _check(lib().qlora_linear_fwd_ex(ctypes.byref(ws), _ptr(X), M, _ptr(A), _ptr(B), r, _ptr(Y),
                                         _ptr(V) if save_V else None, ctypes.byref(o), _ptr(buf), buf.numel(),
                                         _stream(stream)), "qlora_linear_fwd_ex")
    return Y, (V if save_V else None)


def qlora_linear_bwd(w: NF4Weight, X: torch.Tensor, V, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     workspace: Workspace, need_dX: bool = True, stream=None, dX=None, dA=None, dB=None,
                     adapter_scale: float = 1.0, accumulate: bool = False, dropout_keep=None,
                     dropout_p: float = 0.0):
    """Returns (dX or None, dA fp32 (in, r), dB fp32 (r, out)).  With accumulate,
    dA and dB (given) receive the sums instead of being overwritten.  Under
    dropout pass the forward's mask and p."""
    if accumulate and (dA is None or dB is None):
        raise ValueError("accumulate needs the dA and dB to add into")
    M, r = X.shape[0], A.shape[1]
    dev = X.device
    if need_dX and dX is None:
        dX = torch.empty((M, w.n_in), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((w.n_in, r), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((r, w.n_out), dtype=torch.float32, device=dev)
    nb = qlora_workspace_bytes(QLORA_OP_BWD, M, w.n_in, w.n_out, r)
    buf = workspace.get(nb, stream)
    ws = w.c_struct()
    if adapter_scale == 1.0 and not accumulate and dropout_keep is None:
        _check(lib().qlora_linear_bwd(ctypes.byref(ws), _ptr(X), _ptr(V), _ptr(dY), M, _ptr(A), _ptr(B), r,
                                      _ptr(dX) if need_dX else None, _ptr(dA), _ptr(dB), _ptr(buf), buf.numel(),
                                      _stream(stream)), "qlora_linear_bwd")
    else:
        o = _opts(adapter_scale, accumulate, dropout_keep, dropout_p)
        _check(lib().qlora_linear_bwd_ex(ctypes.byref(ws), _ptr(X), _ptr(V), _ptr(dY), M, _ptr(A), _ptr(B), r,
                                         _ptr(dX) if need_dX else None, _ptr(dA), _ptr(dB), ctypes.byref(o),
                                         _ptr(buf), buf.numel(), _stream(stream)), "qlora_linear_bwd_ex")
    return (dX if need_dX else None), dA, dB


def adam_state(A: torch.Tensor, B: torch.Tensor) -> dict:
    """Fresh optimizer state for one layer's adapters: fp32 master copies of A and
    B and zero moments (device tensors, the layouts of A and B)."""
    return {"A32": A.float().contiguous(), "B32": B.float().contiguous(),
            "mA": torch.zeros(A.shape, dtype=torch.float32, device=A.device),
            "vA": torch.zeros(A.shape, dtype=torch.float32, device=A.device),
            "mB": torch.zeros(B.shape, dtype=torch.float32, device=B.device),
            "vB": torch.zeros(B.shape, dtype=torch.float32, device=B.device)}


def qlora_linear_bwd_adam(w: NF4Weight, X: torch.Tensor, V, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                          state: dict, step: int, workspace: Workspace, lr: float = 1e-3, beta1: float = 0.9,
                          beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                          need_dX: bool = True, stream=None, dX=None, adapter_scale: float = 1.0,
                          dropout_keep=None, dropout_p: float = 0.0):
    """Backward with one fused Adam/AdamW step on the adapters: updates `state`
    (fp32 A32, B32, mA, vA, mB, vB) and the bf16 A and B in place; returns dX or None."""
    M, r = X.shape[0], A.shape[1]
    if need_dX and dX is None:
        dX = torch.empty((M, w.n_in), dtype=torch.bfloat16, device=X.device)
    nb = qlora_workspace_bytes(QLORA_OP_BWD, M, w.n_in, w.n_out, r)
    buf = workspace.get(nb, stream)
    ws = w.c_struct()
    st = _AdamState(*[_ptr(state[k]) for k in ("A32", "B32", "mA", "vA", "mB", "vB")])
    hp = _AdamHparams(lr, beta1, beta2, eps, weight_decay, step)
    o = _opts(adapter_scale, False, dropout_keep, dropout_p)
    _check(lib().qlora_linear_bwd_adam(ctypes.byref(ws), _ptr(X), _ptr(V), _ptr(dY), M, _ptr(A), _ptr(B), r,
                                       _ptr(dX) if need_dX else None, ctypes.byref(st), ctypes.byref(hp),
                                       ctypes.byref(o), _ptr(buf), buf.numel(), _stream(stream)),
           "qlora_linear_bwd_adam")
    return dX if need_dX else None


# ---------------------------------------------------------------- compositions
# Built from the library's kernels (and, for the initialisation, a library SVD);
# they are not on the per-step path.

def requantize_merged(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, stream=None) -> NF4Weight:
    """Merge the adapters into the weight and quantise the merge again (the round
    trip that keeps a merged model 4-bit): Q(deq(Wq) + A B), with the library's
    merge (fp32) and quantiser."""
    return qlora_quantize_nf4(qlora_merge(w, A, B, torch.float32, stream=stream), stream=stream)


def qlora_loftq_residual(W0: torch.Tensor, w: NF4Weight, stream=None, out=None) -> torch.Tensor:
    """R = fl32(W0 - deq(Wq)), fp32 (in, out), for a weight quantised from W0."""
    if out is None:
        out = torch.empty((w.n_in, w.n_out), dtype=torch.float32, device=W0.device)
    ws = w.c_struct()
    _check(lib().qlora_loftq_residual(_ptr(W0), ctypes.byref(ws), _ptr(out), _stream(stream)),
           "qlora_loftq_residual")
    return out


def qlora_loftq_split(U: torch.Tensor, S: torch.Tensor, Vh: torch.Tensor, r: int, stream=None):
    """The adapters (A bf16 (in, r), B bf16 (r, out)) from the leading r singular
    triplets of U diag(S) Vh (fp32 device tensors, U (in, k), Vh (k, out))."""
    n_in, n_out = U.shape[0], Vh.shape[1]
    A = torch.empty((n_in, r), dtype=torch.bfloat16, device=U.device)
    B = torch.empty((r, n_out), dtype=torch.bfloat16, device=U.device)
    _check(lib().qlora_loftq_split(_ptr(U), U.shape[1], _ptr(S), _ptr(Vh), Vh.shape[1], n_in, n_out, r, _ptr(A),
                                   _ptr(B), _stream(stream)), "qlora_loftq_split")
    return A, B


def loftq_init(W0: torch.Tensor, r: int, stream=None):
    """Quantise W0 and start the adapters from the rank-r truncated SVD of the
    quantisation residual R = W0 - deq(Q(W0)) = U S V^T, split as A = U_r S_r^1/2,
    B = S_r^1/2 V_r^T (bf16), instead of B = 0.  Returns (NF4Weight, A, B).
    The quantiser, the residual and the split are library kernels; the SVD is
    torch.linalg.svd on the device (a library decomposition, run once at
    initialisation)."""
    if stream is not None and not isinstance(stream, torch.cuda.Stream):
        raise TypeError("loftq_init takes a torch.cuda.Stream (the SVD runs on it too)")
    with torch.cuda.stream(stream) if stream is not None else _nullcontext():
        w = qlora_quantize_nf4(W0)
        R = qlora_loftq_residual(W0, w)
        U, S, Vh = torch.linalg.svd(R, full_matrices=False)
        A, B = qlora_loftq_split(U.contiguous(), S.contiguous(), Vh.contiguous(), r)
    return w, A, B
