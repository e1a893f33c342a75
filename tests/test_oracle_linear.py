"""Pins of the forward / backward / merge oracle (CPU only)."""

import numpy as np
import pytest
import torch

import synth
from oracle import linear, nf4
from tests.conftest import read_golden


def _layer(n_in=64, n_out=128, M=16, r=8, zero_B=False, seed=0):
    t = synth.layer_inputs(n_in, n_out, M, r, seed=seed, zero_B=zero_B)
    codes, dqc, dqs = nf4.quantize_nf4(t["W0"].numpy())
    Wq = nf4.dequantize_bf16(codes, dqc, dqs, n_in, n_out)
    return t, Wq


def test_forward_textbook_matmul_hand_built_weight():
    """in = out = 64, hand-built codes and constants: with B = 0 the forward is the
    plain matmul of X with the hand-computed weight level[code] * 0.25."""
    rng = np.random.default_rng(7)
    flat = rng.integers(0, 16, 64 * 64).astype(np.uint8)
    codes = nf4.pack_nibbles(flat)
    dqc = np.full(64, 0x30, dtype=np.uint8)            # E4M3 0x30 = 0.5
    dqs = np.array([0.5], dtype=np.float32)             # absmax' = 0.25 everywhere
    lv = nf4.nf4_codebook().astype(np.float64)
    W_hand = (lv[flat] * 0.25).reshape(64, 64)          # exact in bf16 range? keep fp32
    Wq = nf4.dequantize(codes, dqc, dqs, 64, 64).astype(np.float64)
    assert np.array_equal(Wq, W_hand.astype(np.float32).astype(np.float64))
    X = rng.standard_normal((5, 64))
    A = rng.standard_normal((64, 8))
    Y, V = linear.forward(X, A, np.zeros((8, 64)), Wq)
    assert np.allclose(Y, np.matmul(X, W_hand), rtol=1e-13, atol=1e-13)
    assert np.allclose(V, X @ A)


def test_forward_B_zero_is_quantized_model():
    """B = 0: the layer output is exactly the dequantised base output ("How it
    works" step 2: training starts exactly at the quantized model)."""
    t, Wq = _layer(zero_B=True)
    Y, _ = linear.forward(t["X"], t["A"], t["B"], Wq)
    X = t["X"].double().numpy()
    assert np.array_equal(Y, X @ Wq.astype(np.float64))


def test_merge_identity():
    """X (Wq + A B) equals the adapted forward ("How it works" step 5, merge)."""
    t, Wq = _layer()
    Y, _ = linear.forward(t["X"], t["A"], t["B"], Wq)
    W = linear.merge(Wq, t["A"], t["B"])
    Y2 = t["X"].double().numpy() @ W
    assert linear.rel_fro(Y2, Y) < 1e-12


def test_backward_factored_equals_dense_form():
    """dA = X^T (dY B^T) and dB = (X A)^T dY equal the pages' dW B^T and A^T dW
    with dW = X^T dY ("How it works" step 4; "The code, line by line")."""
    t, Wq = _layer(M=32)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    d = linear.backward_dense(t["X"], t["A"], t["B"], t["dY"])
    assert linear.rel_fro(g["dA"], d["dA"]) < 1e-12
    assert linear.rel_fro(g["dB"], d["dB"]) < 1e-12
    a = linear.adapter_grads(t["X"], t["A"], t["B"], t["dY"])
    assert np.array_equal(a["dA"], g["dA"]) and np.array_equal(a["dB"], g["dB"])


@pytest.mark.parametrize("scale,p", [(1.0, None), (2.5, None), (2.0, 0.3)])
def test_backward_finite_differences(scale, p):
    """Central differences of L = <dY, Y>: L is linear in each of X, A, B alone
    (for a fixed dropout mask too), so the differences are exact up to rounding
    (catches a dropped term, a transposed operand, a sign, the adapter scale or
    the dropout mask missing from one side)."""
    rng = np.random.default_rng(8)
    n_in, n_out, M, r = 64, 64, 16, 8
    X = rng.standard_normal((M, n_in))
    A = rng.standard_normal((n_in, r)) / 8
    B = rng.standard_normal((r, n_out)) * 0.1
    Wq = rng.standard_normal((n_in, n_out)) * 0.02
    dY = rng.standard_normal((M, n_out))
    keep = None if p is None else (rng.random((M, r)) >= p).astype(np.uint8)
    pp = 0.0 if p is None else p
    g = linear.backward(X, A, B, Wq, dY, scale, keep, pp)

    def L(X_, A_, B_):
        return linear.loss_inner(linear.forward(X_, A_, B_, Wq, scale, keep, pp)[0], dY)

    h = 0.5
    for name, P in (("dX", X), ("dA", A), ("dB", B)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args = {"dX": (Pp, A, B), "dA": (X, Pp, B), "dB": (X, A, Pp)}[name]
            argm = {"dX": (Pm, A, B), "dA": (X, Pm, B), "dB": (X, A, Pm)}[name]
            num[idx] = (L(*args) - L(*argm)) / (2 * h)
        assert np.allclose(num, g[name], rtol=1e-9, atol=1e-9), name


def test_scale_is_the_forward_of_scaled_adapters():
    """The scaled layer's output is the plain layer's with A replaced by s A (one
    of the rescalings "Scaling Factor alpha" calls equivalent)."""
    t, Wq = _layer()
    Y_s, _ = linear.forward(t["X"], t["A"], t["B"], Wq, 2.0)
    Y_1, _ = linear.forward(t["X"], 2.0 * t["A"].double().numpy(), t["B"], Wq)
    np.testing.assert_allclose(Y_s, Y_1, rtol=1e-12, atol=1e-12)


def test_B_zero_gives_zero_dA():
    """B = 0: dA is exactly zero, so the first steps move only B ("How it works",
    paragraph after step 5)."""
    t, Wq = _layer(zero_B=True)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    assert np.all(g["dA"] == 0.0)
    assert np.any(g["dB"] != 0.0)


def test_rows_helpers_match_full():
    t, Wq = _layer(M=24)
    Y, V = linear.forward(t["X"], t["A"], t["B"], Wq)
    rows = [0, 5, 23]
    Yr, Vr = linear.forward_rows(t["X"], t["A"], t["B"], Wq, rows)
    assert np.array_equal(Yr, Y[rows]) and np.array_equal(Vr, V[rows])
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    assert np.allclose(linear.dX_rows(t["A"], t["B"], Wq, t["dY"], rows), g["dX"][rows],
                       rtol=1e-13, atol=1e-13)


def test_adapter_param_counts_printed():
    """r (in + out) per layer reproduces every count the pages print."""
    for row in read_golden("adapter_counts.txt"):
        if row[0] == "dense":
            assert round(int(row[1]) * int(row[2]) / 1e6, 1) == float(row[3]) / 1e6
            continue
        n_in, n_out, r, layers, count = map(int, row)
        assert layers * linear.adapter_params(n_in, n_out, r) == count


def test_wq_bytes_untouched_by_oracle_fwd_bwd():
    """The frozen codes are inputs only: forward and backward leave them as they were."""
    t = synth.layer_inputs(64, 64, 8, 8)
    codes, dqc, dqs = nf4.quantize_nf4(t["W0"].numpy())
    snap = (codes.copy(), dqc.copy(), dqs.copy())
    Wq = nf4.dequantize_bf16(codes, dqc, dqs, 64, 64)
    linear.forward(t["X"], t["A"], t["B"], Wq)
    linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    assert all(np.array_equal(a, b) for a, b in zip(snap, (codes, dqc, dqs)))


def test_synth_inputs_are_seeded_and_distributed():
    """Same name and seed -> same bytes; the stated distributions."""
    a = synth.layer_inputs(256, 256, 64, 8)
    b = synth.layer_inputs(256, 256, 64, 8)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a["W0"].dtype == torch.float32 and a["X"].dtype == torch.bfloat16
    assert abs(a["W0"].std().item() - 0.02) < 1e-3
    assert abs(a["A"].float().std().item() - 1 / 16) < 5e-3
    assert abs(a["B"].float().std().item() - 0.01) < 1e-3


def test_dropout_keep_all_and_drop_all():
    """A mask that keeps everything at p = 0 is the plain layer; a mask that drops
    everything leaves the frozen base alone: Y = X Wq, dA = dB = 0 exactly, dX =
    dY Wq^T."""
    t, Wq = _layer()
    M, r = t["X"].shape[0], t["A"].shape[1]
    Y0, V0 = linear.forward(t["X"], t["A"], t["B"], Wq)
    Y1, V1 = linear.forward(t["X"], t["A"], t["B"], Wq, 1.0, np.ones((M, r), np.uint8), 0.0)
    assert np.array_equal(Y0, Y1) and np.array_equal(V0, V1)
    zero = np.zeros((M, r), np.uint8)
    Yd, Vd = linear.forward(t["X"], t["A"], t["B"], Wq, 1.0, zero, 0.5)
    X, W = t["X"].double().numpy(), np.asarray(Wq, np.float64)
    assert np.array_equal(Yd, X @ W) and not np.any(Vd)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"], 1.0, zero, 0.5)
    assert not np.any(g["dA"]) and not np.any(g["dB"])
    assert np.array_equal(g["dX"], t["dY"].double().numpy() @ W.T)


def test_dropout_preserves_the_mean():
    """Inverted dropout: averaged over masks drawn with keep probability 1 - p,
    the dropped V and the layer output match the undropped ones (the 1 / (1 - p)
    rescale; a missing or inverted rescale is off by a factor of 2 here)."""
    rng = np.random.default_rng(3)
    n_in, n_out, M, r, p = 32, 24, 6, 4, 0.5
    X = rng.standard_normal((M, n_in))
    A = rng.standard_normal((n_in, r))
    B = rng.standard_normal((r, n_out))
    Wq = rng.standard_normal((n_in, n_out)) * 0.02
    Y_ref, V_ref = linear.forward(X, A, B, Wq)
    n = 4000
    V_sum = np.zeros_like(V_ref)
    for _ in range(n):
        keep = (rng.random((M, r)) >= p).astype(np.uint8)
        V_sum += linear.forward(X, A, B, Wq, 1.0, keep, p)[1]
    V_mean = V_sum / n
    # per element the sample mean has standard deviation |V| sqrt(p / ((1 - p) n))
    tol = 5 * np.abs(V_ref) * np.sqrt(p / ((1 - p) * n)) + 1e-12
    assert np.all(np.abs(V_mean - V_ref) <= tol)


def test_dropout_probability_out_of_range():
    t, Wq = _layer()
    keep = np.ones((t["X"].shape[0], t["A"].shape[1]), np.uint8)
    with pytest.raises(ValueError):
        linear.forward(t["X"], t["A"], t["B"], Wq, 1.0, keep, 1.0)
