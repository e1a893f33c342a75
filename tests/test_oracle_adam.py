"""Pins of the adapter Adam / AdamW oracle (CPU only): torch's optimizers as a
library routine, the first-step closed form, and the invariants of the rule."""

import numpy as np
import pytest
import torch

from oracle import adam


def _torch_steps(opt_cls, theta0, grads, **kw):
    """Run torch's optimizer on a float64 copy of theta0 with the given gradients."""
    p = torch.nn.Parameter(torch.tensor(theta0, dtype=torch.float64))
    opt = opt_cls([p], **kw)
    for g in grads:
        p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    st = opt.state[p]
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_matches_torch_adamw_over_several_steps(wd):
    """Three steps from zero moments agree with torch.optim.AdamW (float64)."""
    rng = np.random.default_rng(3)
    theta = rng.standard_normal((32, 8))
    grads = [rng.standard_normal((32, 8)) * s for s in (1.0, 0.3, 2.0)]
    ref = _torch_steps(torch.optim.AdamW, theta, grads, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=wd)
    m = np.zeros_like(theta)
    v = np.zeros_like(theta)
    for t, g in enumerate(grads, start=1):
        theta, m, v = adam.adam_step(theta, g, m, v, t, lr=1e-3, weight_decay=wd)
    for got, want in zip((theta, m, v), ref):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)


def test_no_decay_matches_torch_adam():
    """weight_decay = 0 is plain Adam (torch.optim.Adam, float64)."""
    rng = np.random.default_rng(4)
    theta = rng.standard_normal((16, 16))
    grads = [rng.standard_normal((16, 16)) for _ in range(4)]
    ref = _torch_steps(torch.optim.Adam, theta, grads, lr=2e-3, betas=(0.8, 0.99), eps=1e-6)
    m = np.zeros_like(theta)
    v = np.zeros_like(theta)
    for t, g in enumerate(grads, start=1):
        theta, m, v = adam.adam_step(theta, g, m, v, t, lr=2e-3, beta1=0.8, beta2=0.99, eps=1e-6)
    np.testing.assert_allclose(theta, ref[0], rtol=1e-12, atol=1e-15)


def test_first_step_closed_form():
    """From zero moments the bias-corrected step is lr * g / (|g| + eps): about
    lr * sign(g) for |g| >> eps, and exactly 0 where g = 0."""
    g = np.array([3.0, -0.5, 1e-3, 0.0, -7e-9])
    theta = np.array([1.0, 2.0, -1.0, 0.5, 0.25])
    lr, eps = 1e-2, 1e-8
    t1, m1, v1 = adam.adam_step(theta, g, np.zeros(5), np.zeros(5), 1, lr=lr, eps=eps)
    np.testing.assert_allclose(t1, theta - lr * g / (np.abs(g) + eps), rtol=1e-14, atol=1e-17)
    assert t1[3] == theta[3]
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-14)   # 1 - 0.999 is not 0.001 in binary64


def test_zero_gradient_zero_moments_leaves_adapters():
    """No gradient and no history: the adapters do not move (and with decay they
    shrink by exactly (1 - lr * wd))."""
    theta = np.linspace(-1, 1, 12)
    z = np.zeros(12)
    t1, _, _ = adam.adam_step(theta, z, z, z, 5, lr=1e-3)
    assert np.array_equal(t1, theta)
    t2, _, _ = adam.adam_step(theta, z, z, z, 5, lr=1e-3, weight_decay=0.1)
    np.testing.assert_allclose(t2, theta * (1 - 1e-4), rtol=1e-15)


def test_first_step_bounded_by_lr():
    """From zero state the first bias-corrected step of every element is at most lr
    and points against the gradient; a sign or bias-correction slip breaks this."""
    rng = np.random.default_rng(9)
    g = rng.standard_normal(1000) * rng.uniform(0, 10, 1000)
    theta = rng.standard_normal(1000)
    t1, _, _ = adam.adam_step(theta, g, np.zeros(1000), np.zeros(1000), 1, lr=1e-3)
    assert np.max(np.abs(t1 - theta)) <= 1e-3 * (1 + 1e-12)
    assert np.all(np.sign(theta - t1) == np.sign(g))


def test_adapter_step_updates_both_and_keeps_shapes():
    rng = np.random.default_rng(1)
    A, B = rng.standard_normal((64, 8)), rng.standard_normal((8, 32))
    dA, dB = rng.standard_normal((64, 8)), rng.standard_normal((8, 32))
    st = {k: np.zeros(s) for k, s in (("mA", A.shape), ("vA", A.shape), ("mB", B.shape), ("vB", B.shape))}
    A1, B1, st1 = adam.adapter_adam_step(A, B, dA, dB, st, 1, lr=1e-3)
    assert A1.shape == A.shape and B1.shape == B.shape
    a_ref, _, _ = adam.adam_step(A, dA, st["mA"], st["vA"], 1, lr=1e-3)
    np.testing.assert_array_equal(A1, a_ref)
    assert set(st1) == {"mA", "vA", "mB", "vB"}


def test_rejects_step_zero():
    with pytest.raises(ValueError):
        adam.adam_step(np.zeros(2), np.zeros(2), np.zeros(2), np.zeros(2), 0, lr=1e-3)
