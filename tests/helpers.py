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
