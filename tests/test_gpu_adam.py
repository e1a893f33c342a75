"""GPU parity of the backward with the fused Adam / AdamW step on the adapters
(qlora_linear_bwd_adam) against the float64 oracle: gradients from the oracle's
backward, then the oracle's Adam step."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import adam, linear
from tests.helpers import assert_close, layer_on_gpu, oracle_weight, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _f64(t):
    return t.detach().double().cpu().numpy()


def _prior_state(A, B, gA, gB, tag):
    """Seeded moments on the scale of the gradients (so that the step is well
    conditioned): m ~ N(0, s^2), v = n^2 + s^2/2 with n ~ N(0, s^2)."""
    sA, sB = float(np.std(gA)), float(np.std(gB))
    st = {"A32": A.float().contiguous(), "B32": B.float().contiguous(),
          "mA": synth.normal(f"{tag}mA", tuple(A.shape), sA, device="cuda"),
          "mB": synth.normal(f"{tag}mB", tuple(B.shape), sB, device="cuda")}
    st["vA"] = synth.normal(f"{tag}vA", tuple(A.shape), sA, device="cuda") ** 2 + 0.5 * sA * sA
    st["vB"] = synth.normal(f"{tag}vB", tuple(B.shape), sB, device="cuda") ** 2 + 0.5 * sB * sB
    return st


@pytest.mark.parametrize("n_in,n_out,M,r,wd", [(256, 512, 96, 16, 0.0), (1024, 768, 300, 24, 0.01),
                                               (4096, 4096, 512, 16, 0.0)])
def test_fused_adam_step_matches_oracle(n_in, n_out, M, r, wd):
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="adam")
    Wq = oracle_weight(w)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    st = _prior_state(t["A"], t["B"], g["dA"], g["dB"], f"adam{n_in}")
    st0 = {k: _f64(v) for k, v in st.items()}
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd)

    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    dX_plain, _, _ = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws)
    A, B = t["A"].clone(), t["B"].clone()
    dX = q.qlora_linear_bwd_adam(w, t["X"], V, t["dY"], A, B, st, 5, ws, **hp)
    torch.cuda.synchronize()
    assert ws.status() == 0

    A1, B1, ref = adam.adapter_adam_step(st0["A32"], st0["B32"], g["dA"], g["dB"],
                                         {k: st0[k] for k in ("mA", "vA", "mB", "vB")}, 5, **hp)
    # the step itself (theta' - theta), and the new moments
    assert_close(_f64(st["A32"]) - st0["A32"], A1 - st0["A32"], "A step")
    assert_close(_f64(st["B32"]) - st0["B32"], B1 - st0["B32"], "B step")
    for k in ("mA", "vA", "mB", "vB"):
        assert_close(_f64(st[k]), ref[k], k)
    # the layer's bf16 adapters are the rounded masters; dX used the adapters on entry
    assert torch.equal(A, st["A32"].to(torch.bfloat16))
    assert torch.equal(B, st["B32"].to(torch.bfloat16))
    assert torch.equal(dX, dX_plain)


def test_first_step_from_zero_state():
    """t = 1 from zero moments: every element moves by at most lr, against the sign
    of its gradient wherever the gradient is not tiny, and m = (1 - b1) g."""
    t, w = layer_on_gpu(512, 256, 128, 8, tag="adam1")
    g = linear.backward(t["X"], t["A"], t["B"], oracle_weight(w), t["dY"])
    st = q.adam_state(t["A"], t["B"])
    A0, B0 = _f64(st["A32"]), _f64(st["B32"])
    ws = q.Workspace()
    A, B = t["A"].clone(), t["B"].clone()
    q.qlora_linear_bwd_adam(w, t["X"], None, t["dY"], A, B, st, 1, ws, lr=1e-2, need_dX=False)
    torch.cuda.synchronize()
    lr = 1e-2
    for theta0, theta1, gr, m in ((A0, _f64(st["A32"]), g["dA"], _f64(st["mA"])),
                                  (B0, _f64(st["B32"]), g["dB"], _f64(st["mB"]))):
        step = theta1 - theta0
        assert np.max(np.abs(step)) <= lr * (1 + 1e-5)
        big = np.abs(gr) > 0.05 * np.max(np.abs(gr))
        assert np.all(np.sign(step[big]) == -np.sign(gr[big]))
        assert_close(m, 0.1 * gr, "m after one step")


def test_zero_B_leaves_A_exactly():
    """B = 0 makes dA exactly 0 (U = dY B^T = 0), so from zero state A, mA and vA
    do not change at all, while B moves."""
    t, w = layer_on_gpu(256, 256, 64, 8, zero_B=True, tag="adam0")
    st = q.adam_state(t["A"], t["B"])
    A32 = st["A32"].clone()
    ws = q.Workspace()
    A, B = t["A"].clone(), t["B"].clone()
    q.qlora_linear_bwd_adam(w, t["X"], None, t["dY"], A, B, st, 1, ws, need_dX=False)
    torch.cuda.synchronize()
    assert torch.equal(st["A32"], A32)
    assert torch.count_nonzero(st["mA"]) == 0 and torch.count_nonzero(st["vA"]) == 0
    assert torch.equal(A, t["A"])
    assert torch.count_nonzero(st["B32"]) > 0


def test_repeated_steps_track_the_oracle():
    """Three consecutive fused steps (t = 5, 6, 7, fixed batch, seeded prior
    moments) against three oracle steps, each oracle step on the oracle's own
    adapters."""
    t, w = layer_on_gpu(256, 384, 80, 16, tag="adam3")
    Wq = oracle_weight(w)
    g0 = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    st = _prior_state(t["A"], t["B"], g0["dA"], g0["dB"], "adam3")
    ref_A, ref_B = _f64(st["A32"]), _f64(st["B32"])
    ref_st = {k: _f64(st[k]) for k in ("mA", "vA", "mB", "vB")}
    A, B = t["A"].clone(), t["B"].clone()
    ws = q.Workspace()
    for step in (5, 6, 7):
        # the oracle's gradients at its own current adapters (bf16, as the layer sees them)
        Ab = torch.tensor(ref_A, dtype=torch.float32).to(torch.bfloat16)
        Bb = torch.tensor(ref_B, dtype=torch.float32).to(torch.bfloat16)
        g = linear.backward(t["X"], Ab, Bb, Wq, t["dY"])
        ref_A, ref_B, ref_st = adam.adapter_adam_step(ref_A, ref_B, g["dA"], g["dB"], ref_st, step, lr=1e-3)
        q.qlora_linear_bwd_adam(w, t["X"], None, t["dY"], A, B, st, step, ws, lr=1e-3, need_dX=False)
    torch.cuda.synchronize()
    A0, B0 = _f64(t["A"]), _f64(t["B"])
    assert_close(_f64(st["A32"]) - A0, ref_A - A0, "A after 3 steps")
    assert_close(_f64(st["B32"]) - B0, ref_B - B0, "B after 3 steps")


def test_fused_adam_with_adapter_scale():
    """The fused step uses the scaled layer's gradients (s = 2)."""
    t, w = layer_on_gpu(512, 256, 64, 8, tag="adams")
    Wq = oracle_weight(w)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"], 2.0)
    st = _prior_state(t["A"], t["B"], g["dA"], g["dB"], "adams")
    st0 = {k: _f64(v) for k, v in st.items()}
    ws = q.Workspace()
    A, B = t["A"].clone(), t["B"].clone()
    q.qlora_linear_bwd_adam(w, t["X"], None, t["dY"], A, B, st, 5, ws, need_dX=False, adapter_scale=2.0)
    torch.cuda.synchronize()
    A1, B1, _ = adam.adapter_adam_step(st0["A32"], st0["B32"], g["dA"], g["dB"],
                                       {k: st0[k] for k in ("mA", "vA", "mB", "vB")}, 5, lr=1e-3)
    assert_close(_f64(st["A32"]) - st0["A32"], A1 - st0["A32"], "A step (scaled)")
    assert_close(_f64(st["B32"]) - st0["B32"], B1 - st0["B32"], "B step (scaled)")
