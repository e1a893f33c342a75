"""Symmetric uniform integer quantisation with one scale per 16 weights: the
second base quantiser, of the pages' own simulation (float64 oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix:

* "QLoRA (low-rank adapters on a quantized model)", "The code, line by line":
  the lab quantises with symmetric uniform integers, one scale per 16
  consecutive entries of the flattened (in, out) matrix; "Simplifications": no
  NF4 and no double quantisation (the scales stay fp32).
* Same page, "What the simulations show": the runs use 2, 3 and 4 bits, and
  "2-bit" is ternary, {-s, 0, s}.

Reading (the rounding rule and the step are not printed): for b bits the
integers run over -Q .. Q with Q = 2^(b-1) - 1 (b = 4: -7 .. 7, b = 3: -3 .. 3,
b = 2: -1 .. 1, the ternary case); per group of 16 the step is
s = fl32(max |w| / Q); the code is q = rint(fl32(w / s)) (ties to even) clamped
to [-Q, Q]; the reconstruction is w' = fl32(q s).  An all-zero group has s = 0
and q = 0.

Storage (the pages are silent; one convention shared by both sides): q + 8 in a
4-bit nibble, element 2k in the low nibble of byte k of the flattened matrix,
as for NF4, whatever b is; the scales as fp32 [in * out / 16].
"""

from __future__ import annotations

import numpy as np

from oracle.nf4 import fl32, pack_nibbles, unpack_nibbles

GROUP16 = 16
BITS = (2, 3, 4)


def qmax(bits: int) -> int:
    """Largest integer magnitude of the b-bit symmetric grid."""
    if bits not in BITS:
        raise ValueError("bits must be 2, 3 or 4")
    return (1 << (bits - 1)) - 1


def quantize_int(W0, bits: int):
    """fp32 W0 (in, out) -> (packed codes uint8 [in*out/2], fp32 scales [in*out/16])."""
    Q = qmax(bits)
    w = np.asarray(W0, dtype=np.float32).reshape(-1)
    if w.size % GROUP16:
        raise ValueError("in*out must be a multiple of 16")
    if not np.all(np.isfinite(w)):
        raise ValueError("W0 must be finite")
    g = w.reshape(-1, GROUP16)
    a = np.abs(g).max(axis=1)
    s = fl32(a.astype(np.float64) / Q)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float64)
    y = fl32(g.astype(np.float64) / safe[:, None])             # IEEE quotient in fp32
    q = np.clip(np.rint(y.astype(np.float64)), -Q, Q)
    q = np.where(s[:, None] > 0, q, 0.0).astype(np.int64)
    return pack_nibbles((q + 8).astype(np.uint8).reshape(-1)), s.astype(np.float32)


def dequantize_int(codes, scales, n_in: int, n_out: int) -> np.ndarray:
    """w' = fl32((code - 8) s) as float32 (n_in, n_out)."""
    q = unpack_nibbles(np.asarray(codes, dtype=np.uint8)).astype(np.float64) - 8.0
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)
    return fl32(q.reshape(-1, GROUP16) * s[:, None]).reshape(n_in, n_out)
