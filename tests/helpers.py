"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding, run the float64 oracle on the same bytes, and compare."""

from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import linear, nf4

# Tolerances for floating-point outputs (bf16 inputs, fp32 accumulation).
REL_FRO = 1e-2
MAX_ABS = 2e-2


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    if not os.path.exists(q.LIB_PATH):
        from quantized_rank_fine_b200 import build
        build.build()
    q.lib()


def assert_close(got, ref, name, rel_fro=REL_FRO, max_abs=MAX_ABS):
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    rf = linear.rel_fro(g, ref)
    ma = linear.max_abs_ratio(g, ref)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    assert rf <= rel_fro and ma <= max_abs, f"{name}: rel_fro={rf:.3e} max_abs_ratio={ma:.3e}"
    return rf, ma


def quantize_both(W0: torch.Tensor):
    """GPU quantisation of W0 and the oracle's, as numpy arrays."""
    w = q.qlora_quantize_nf4(W0.cuda().contiguous())
    torch.cuda.synchronize()
    gpu = (w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy())
    ref = nf4.quantize_nf4(W0.cpu().numpy())
    return w, gpu, ref


def assert_quant_equal(gpu, ref, what=""):
    names = ("codes", "dq_codes", "dq_scales")
    for n, g, r in zip(names, gpu, ref):
        g = np.ascontiguousarray(g)
        r = np.ascontiguousarray(r)
        if n == "dq_scales":
            g, r = g.view(np.uint32), r.astype(np.float32).view(np.uint32)
        bad = np.flatnonzero(g != r)
        assert bad.size == 0, f"{what} {n}: {bad.size} mismatches, first at {bad[:5]}: {g[bad[:5]]} vs {r[bad[:5]]}"


def layer_on_gpu(n_in, n_out, M, r, seed=0, zero_B=False, tag=""):
    """Seeded inputs on the GPU (drawn there for speed) plus the quantised weight."""
    t = synth.layer_inputs(n_in, n_out, M, r, device="cuda", seed=seed, zero_B=zero_B, tag=tag)
    w = q.qlora_quantize_nf4(t["W0"])
    return t, w


def oracle_weight(w: q.NF4Weight) -> np.ndarray:
    """bf16(w') from the GPU-produced codes, computed by the oracle (codes are
    checked bit-exact against the oracle's own quantiser elsewhere)."""
    return nf4.dequantize_bf16(w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy(),
                               w.n_in, w.n_out)


def run_fwd_bwd(t, w, ws=None, need_dX=True):
    ws = ws or q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws, need_dX=need_dX)
    torch.cuda.synchronize()
    assert ws.status() == 0, "a kernel wait timed out"
    return {"Y": Y, "V": V, "dX": dX, "dA": dA, "dB": dB}


def full_check(t, w, out):
    """Every output of one forward + backward against the oracle on the same bytes."""
    Wq = oracle_weight(w)
    Y, V = linear.forward(t["X"], t["A"], t["B"], Wq)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    assert_close(out["Y"], Y, "Y")
    assert_close(out["V"], V, "V")
    assert_close(out["dX"], g["dX"], "dX")
    assert_close(out["dA"], g["dA"], "dA")
    assert_close(out["dB"], g["dB"], "dB")


class BlockedClose:
    """The two tolerance measures of `assert_close` (relative Frobenius error and
    max-abs error over max |ref|) accumulated over row blocks, so that outputs
    too large to hold in float64 at once are still compared element by element."""

    def __init__(self, name):
        self.name = name
        self.num2 = self.den2 = 0.0
        self.max_diff = self.max_ref = 0.0

    def add(self, got, ref):
        g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
        ref = np.asarray(ref, np.float64)
        assert g.shape == ref.shape, f"{self.name}: shape {g.shape} vs {ref.shape}"
        assert np.all(np.isfinite(g)), f"{self.name}: non-finite values"
        d = g - ref
        self.num2 += float(np.sum(d * d))
        self.den2 += float(np.sum(ref * ref))
        self.max_diff = max(self.max_diff, float(np.max(np.abs(d))) if d.size else 0.0)
        self.max_ref = max(self.max_ref, float(np.max(np.abs(ref))) if ref.size else 0.0)

    def check(self, rel_fro=REL_FRO, max_abs=MAX_ABS):
        rf = (self.num2 ** 0.5) / (self.den2 ** 0.5) if self.den2 > 0 else (0.0 if self.num2 == 0 else np.inf)
        ma = self.max_diff / self.max_ref if self.max_ref > 0 else (0.0 if self.max_diff == 0 else np.inf)
        assert rf <= rel_fro and ma <= max_abs, f"{self.name}: rel_fro={rf:.3e} max_abs_ratio={ma:.3e}"
        return rf, ma


def _rows(t, lo, hi):
    """Rows lo..hi of a device bf16 tensor as float64 numpy."""
    return t[lo:hi].double().cpu().numpy()


def full_check_blocked(t, w, out, block=1024, Wq=None):
    """`full_check` for outputs of any size: every row of Y, V and dX, and dA, dB
    in full, against the float64 oracle evaluated block of token rows by block
    (the oracle's own functions on each block; dA and dB summed over blocks)."""
    if Wq is None:
        Wq = oracle_weight(w)
    Wq = np.asarray(Wq, np.float64)
    A = t["A"].double().cpu().numpy()
    B = t["B"].double().cpu().numpy()
    M = t["X"].shape[0]
    cY, cV, cdX = BlockedClose("Y"), BlockedClose("V"), BlockedClose("dX")
    dA = np.zeros((A.shape[0], A.shape[1]))
    dB = np.zeros((B.shape[0], B.shape[1]))
    for lo in range(0, M, block):
        hi = min(M, lo + block)
        X, dY = _rows(t["X"], lo, hi), _rows(t["dY"], lo, hi)
        Yr, Vr = linear.forward(X, A, B, Wq)
        g = linear.backward(X, A, B, Wq, dY)
        cY.add(out["Y"][lo:hi], Yr)
        cV.add(out["V"][lo:hi], Vr)
        cdX.add(out["dX"][lo:hi], g["dX"])
        dA += g["dA"]
        dB += g["dB"]
    for c in (cY, cV, cdX):
        c.check()
    assert_close(out["dA"], dA, "dA")
    assert_close(out["dB"], dB, "dB")


def oracle_pool(workers=None):
    """A process pool over the host cores for the oracle's quantiser (map
    `oracle.nf4.quantize_nf4` over fp32 numpy matrices; the children import only
    the oracle and numpy).  Started with `spawn`, since a child forked from a
    process that has used CUDA can hang; a child that dies raises
    BrokenProcessPool instead of leaving the map waiting."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    workers = workers or len(os.sched_getaffinity(0))
    return ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))


# Canary guard regions around outputs: a kernel that writes past either end of
# an output it was given changes these bytes.  They stand in for a memory checker
# on ragged shapes, where tile edges are cut.
GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


def guarded(shape, dtype, device="cuda"):
    """(buffer, view): `view` is a contiguous output tensor of `shape` inside
    `buffer`, with GUARD_BYTES canary bytes before and after it (16-byte aligned)."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((2 * GUARD_BYTES + n,), GUARD_BYTE, dtype=torch.uint8, device=device)
    return buf, buf[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(tuple(shape))


def assert_guards(bufs, what=""):
    torch.cuda.synchronize()
    for i, buf in enumerate(bufs):
        ok = bool((buf[:GUARD_BYTES] == GUARD_BYTE).all()) and bool((buf[-GUARD_BYTES:] == GUARD_BYTE).all())
        assert ok, f"{what}: a write landed outside output {i}"
