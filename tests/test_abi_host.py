"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching a device (CPU only)."""

import ctypes
import os
import re

import numpy as np
import pytest

import quantized_rank_fine_b200 as q
from oracle import nf4
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "qlora.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(q.LIB_PATH):
        from quantized_rank_fine_b200 import build
        build.build()
    return q.lib()


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(q.EXPORTS)


def test_codebook_equals_oracle(L):
    """The library's constant levels are the oracle's codebook, bit for bit."""
    got = np.array(q.qlora_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), nf4.nf4_codebook().view(np.uint32))


def test_adapter_params_and_status_strings(L):
    assert q.qlora_adapter_params(4096, 4096, 16) == 131072
    assert q.qlora_adapter_params(768, 2304, 8) == 24576
    for s in range(8):
        assert len(q.qlora_status_string(s)) > 0


def test_workspace_bytes(L):
    assert q.qlora_workspace_bytes(q.QLORA_OP_FWD, 4096, 4096, 4096, 16) >= 256 + 4096 * 16 * 2
    assert q.qlora_workspace_bytes(q.QLORA_OP_BWD, 4096, 4096, 4096, 16) >= 256 + 2 * 4096 * 16 * 2
    assert q.qlora_workspace_bytes(q.QLORA_OP_FWD, 64, 256, 256, 7) == 0      # r % 8 != 0
    assert q.qlora_workspace_bytes(q.QLORA_OP_FWD, 64, 100, 256, 8) == 0      # in % 64 != 0
    assert q.qlora_workspace_bytes(q.QLORA_OP_FWD, 0, 256, 256, 8) == 0       # M = 0
    assert q.qlora_workspace_bytes(9, 64, 256, 256, 8) == 0                   # unknown op


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: every case below fails before device access


def test_quantize_rejects_before_launch(L):
    assert L.qlora_quantize_nf4(None, 64, 64, FAKE, FAKE, FAKE, None) == 1
    assert L.qlora_quantize_nf4(FAKE, 3, 7, FAKE, FAKE, FAKE, None) == 2
    assert L.qlora_quantize_nf4(FAKE, 0, 64, FAKE, FAKE, FAKE, None) == 2


def test_batch_quantize_rejects_before_launch(L):
    job = q._QuantizeJob(0x10000, 64, 64, 0x10000, 0x10000, 0x10000)
    bad_ptr = q._QuantizeJob(0x10000, 64, 64, None, 0x10000, 0x10000)
    bad_shape = q._QuantizeJob(0x10000, 3, 7, 0x10000, 0x10000, 0x10000)
    jobs = (q._QuantizeJob * 2)(job, bad_ptr)
    assert L.qlora_quantize_nf4_batch(jobs, -1, 0, None) == 1          # negative count
    assert L.qlora_quantize_nf4_batch(None, 2, 0, None) == 1           # no descriptors
    assert L.qlora_quantize_nf4_batch(jobs, 1, 7, None) == 1           # unknown absmax format
    assert L.qlora_quantize_nf4_batch(jobs, 2, 0, None) == 1           # a NULL output in job 1
    assert L.qlora_quantize_nf4_batch((q._QuantizeJob * 2)(job, bad_shape), 2, 0, None) == 2
    assert L.qlora_quantize_nf4_batch(None, 0, 0, None) == 0           # nothing to do


def test_linear_rejects_before_launch(L):
    w = q._Weight(0x10000, 0x10000, 0x10000, 256, 256)
    wp = ctypes.byref(w)
    fwd, bwd = L.qlora_linear_fwd, L.qlora_linear_bwd
    assert fwd(wp, None, 64, FAKE, FAKE, 8, FAKE, None, FAKE, 1 << 30, None) == 1        # X NULL
    assert fwd(wp, FAKE, 64, FAKE, FAKE, 12, FAKE, None, FAKE, 1 << 30, None) == 2       # r % 8
    assert fwd(wp, FAKE, 0, FAKE, FAKE, 8, FAKE, None, FAKE, 1 << 30, None) == 2         # M = 0
    assert fwd(wp, FAKE, 64, FAKE, FAKE, 8, FAKE, None, FAKE, 16, None) == 4             # ws too small
    assert fwd(wp, FAKE, 64, FAKE, FAKE, 8, FAKE, None, None, 1 << 30, None) == 4        # ws NULL
    w2 = q._Weight(0x10000, 0x10000, 0x10000, 256, 100)                               # out % 64
    assert fwd(ctypes.byref(w2), FAKE, 64, FAKE, FAKE, 8, FAKE, None, FAKE, 1 << 30, None) == 2
    assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 8, None, None, FAKE, FAKE, 1 << 30, None) == 1
    assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 264, None, FAKE, FAKE, FAKE, 1 << 30, None) == 2
    assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 8, None, FAKE, FAKE, FAKE, 8, None) == 4
    w0 = q._Weight(0, 0x10000, 0x10000, 256, 256)                                      # codes NULL
    assert fwd(ctypes.byref(w0), FAKE, 64, FAKE, FAKE, 8, FAKE, None, FAKE, 1 << 30, None) == 1


def test_bwd_adam_rejects_before_launch(L):
    """The fused backward + Adam step checks its state pointers and
    hyper-parameters on the host, before any device access."""
    w = q._Weight(0x10000, 0x10000, 0x10000, 256, 256)
    wp = ctypes.byref(w)
    st = q._AdamState(*([0x10000] * 6))
    hp = q._AdamHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    f = L.qlora_linear_bwd_adam

    def call(st_, hp_, r=8, ws_bytes=1 << 30, opts=None):
        return f(wp, FAKE, None, FAKE, 64, FAKE, FAKE, r, None, st_, hp_, opts, FAKE, ws_bytes, None)

    assert call(None, ctypes.byref(hp)) == 1                                        # state NULL
    assert call(ctypes.byref(st), None) == 1                                        # hparams NULL
    st0 = q._AdamState(0x10000, 0x10000, 0, 0x10000, 0x10000, 0x10000)              # mA NULL
    assert call(ctypes.byref(st0), ctypes.byref(hp)) == 1
    for bad in (dict(step=0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=0.0), dict(lr=-1.0),
                dict(weight_decay=-0.5), dict(lr=float("nan"))):
        h = q._AdamHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
        for k, v in bad.items():
            setattr(h, k, v)
        assert call(ctypes.byref(st), ctypes.byref(h)) == 1, bad
    assert call(ctypes.byref(st), ctypes.byref(hp), r=12) == 2                      # r % 8
    assert call(ctypes.byref(st), ctypes.byref(hp), ws_bytes=8) == 4                # workspace too small
    acc = q._LinearOpts(1.0, q.QLORA_ACCUMULATE_GRADS)
    assert call(ctypes.byref(st), ctypes.byref(hp), opts=ctypes.byref(acc)) == 1    # accumulate + Adam


def test_ex_options_rejected_before_launch(L):
    """Bad options of the _ex calls are refused on the host."""
    w = q._Weight(0x10000, 0x10000, 0x10000, 256, 256)
    wp = ctypes.byref(w)
    bad_flags = q._LinearOpts(1.0, 0x80)
    nan_scale = q._LinearOpts(float("nan"), 0)
    acc = q._LinearOpts(2.0, q.QLORA_ACCUMULATE_GRADS)
    fwd, bwd = L.qlora_linear_fwd_ex, L.qlora_linear_bwd_ex
    for o in (bad_flags, nan_scale, acc):                                          # acc: no grads in fwd
        assert fwd(wp, FAKE, 64, FAKE, FAKE, 8, FAKE, None, ctypes.byref(o), FAKE, 1 << 30, None) == 1
    for o in (bad_flags, nan_scale):
        assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 8, None, FAKE, FAKE, ctypes.byref(o), FAKE, 1 << 30,
                   None) == 1
    assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 12, None, FAKE, FAKE, ctypes.byref(acc), FAKE, 1 << 30,
               None) == 2                                                          # r % 8
    # dropout: with a keep mask the drop probability must lie in [0, 1)
    for p in (1.0, -0.25, float("nan")):
        o = q._LinearOpts(1.0, 0, FAKE, p)
        assert fwd(wp, FAKE, 64, FAKE, FAKE, 8, FAKE, None, ctypes.byref(o), FAKE, 1 << 30, None) == 1
        assert bwd(wp, FAKE, None, FAKE, 64, FAKE, FAKE, 8, None, FAKE, FAKE, ctypes.byref(o), FAKE, 1 << 30,
                   None) == 1
    # without a mask p is not read: the call gets past the options (r % 8 fails next)
    o = q._LinearOpts(1.0, 0, None, 7.0)
    assert fwd(wp, FAKE, 64, FAKE, FAKE, 12, FAKE, None, ctypes.byref(o), FAKE, 1 << 30, None) == 2


def test_unknown_absmax_format_rejected(L):
    """A weight descriptor or a quantise call with an unknown absmax code format
    is refused before any launch."""
    w = q._Weight(0x10000, 0x10000, 0x10000, 256, 256, 9)
    assert L.qlora_dequantize(ctypes.byref(w), FAKE, 0, None) == 1
    assert L.qlora_linear_fwd(ctypes.byref(w), FAKE, 64, FAKE, FAKE, 8, FAKE, None, FAKE, 1 << 30, None) == 1
    assert L.qlora_quantize_nf4_ex(FAKE, 64, 64, FAKE, FAKE, FAKE, 2, None) == 1
    assert L.qlora_quantize_nf4_ex(FAKE, 64, 64, FAKE, FAKE, FAKE, -1, None) == 1


def test_dequant_merge_reject_before_launch(L):
    w = q._Weight(0x10000, 0x10000, 0x10000, 256, 256)
    assert L.qlora_dequantize(ctypes.byref(w), FAKE, 5, None) == 1                      # bad dtype
    assert L.qlora_dequantize(None, FAKE, 0, None) == 1
    assert L.qlora_merge(ctypes.byref(w), FAKE, FAKE, 4, FAKE, 0, None) == 2           # r < 8
    assert L.qlora_merge(ctypes.byref(w), None, FAKE, 8, FAKE, 0, None) == 1


def test_no_gpu_means_loud_error_not_fallback(L):
    """With no usable sm_100 device the calls report an error instead of computing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.qlora_quantize_nf4(FAKE, 64, 64, FAKE, FAKE, FAKE, None) in (5, 6)


def test_int_quantiser_rejects_before_launch(L):
    """The INT group-16 quantiser refuses bad bit widths, shapes and dtypes on
    the host."""
    for bits in (1, 5, 8):
        assert L.qlora_quantize_int(FAKE, 16, 16, bits, FAKE, FAKE, None) == 1
    assert L.qlora_quantize_int(FAKE, 3, 5, 4, FAKE, FAKE, None) == 2          # in*out % 16
    assert L.qlora_quantize_int(None, 16, 16, 4, FAKE, FAKE, None) == 1
    assert L.qlora_dequantize_int(FAKE, FAKE, 16, 16, FAKE, 7, None) == 1      # dtype
    assert L.qlora_dequantize_int(FAKE, FAKE, 0, 16, FAKE, 0, None) == 2


def test_int16_weight_descriptor_checks(L):
    """An INT16 weight needs no absmax codes (NULL passes the argument checks and
    fails only for lack of a device); an NF4 weight without them is refused."""
    w_int = q._Weight(0x10000, 0, 0x10000, 256, 256, q.QLORA_FMT_INT16)
    assert L.qlora_dequantize(ctypes.byref(w_int), FAKE, 0, None) != 1
    w_nf4 = q._Weight(0x10000, 0, 0x10000, 256, 256, q.QLORA_DQ_E4M3)
    assert L.qlora_dequantize(ctypes.byref(w_nf4), FAKE, 0, None) == 1


def test_selftest_and_status_calls_check_arguments_first(L):
    """The failure-path self-test rejects a bad kind, limit or workspace before it
    looks for a device; the status calls report an error (and do not crash) when
    there is no usable device."""
    fake = ctypes.c_void_p(4096)
    assert L.qlora_selftest_wait_timeout(fake, 4096, 2, 50, None) == 1        # unknown kind
    assert L.qlora_selftest_wait_timeout(fake, 4096, 0, 0, None) == 1         # limit 0
    assert L.qlora_selftest_wait_timeout(fake, 4096, 1, 1000001, None) == 1   # limit above 1 s
    assert L.qlora_selftest_wait_timeout(None, 4096, 0, 50, None) == 4        # no workspace
    assert L.qlora_selftest_wait_timeout(fake, 1279, 0, 50, None) == 4        # shorter than the prefix
    import torch
    if not torch.cuda.is_available():
        assert L.qlora_quantize_status(None) != 0
        assert L.qlora_static_ws_status(None) != 0
