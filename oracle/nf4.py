"""NF4 blockwise quantisation with double-quantised absmax (float64 oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What is computed, and where the pages say so:

* Codebook: 16 levels placed at quantiles of N(0, 1), scaled to [-1, 1]
  ("QLoRA (low-rank adapters on a quantized model)", "What QLoRA adds over
  LoRA", NF4 bullet; "LoRA & QLoRA", "4-bit NormalFloat (NF4)", item 3 and the
  NF4 value table).  The pages leave the quantile positions open; the reading
  taken is the asymmetric construction of the QLoRA paper the pages cite
  (8 positive quantiles, 7 negative, one exact zero, offset
  delta = (31/32 + 29/30) / 2).
* Blockwise absmax: one scale per 64 consecutive weights of the flattened
  (in, out) matrix ("LLMs · QLoRA", the ``quantise`` listing: reshape to rows of
  64, absmax per row; "QLoRA (low-rank adapters on a quantized model)",
  "The code, line by line": groups of consecutive entries of the flattened
  (in, out) matrix).
* Nearest-level code: argmin over levels of |w / absmax - level|, ties to the
  lower index ("LLMs · QLoRA", ``quantise`` listing, ``argmin``).
* Double quantisation: absmax values quantised to 8 bits ("QLoRA (low-rank
  adapters on a quantized model)", "What QLoRA adds over LoRA"), as an 8-bit
  float ("LoRA & QLoRA", "Double Quantization").  Reading: OCP FP8 E4M3,
  one fp32 scale per 256 consecutive absmax values, s = fl32(max / 448),
  code = E4M3_RNE_satfinite(fl32(absmax / s)); no mean-centering.
* Alternative double quantisation (``dq_format="u8"``): the same 8 bits read as
  a linear unsigned integer ("QLoRA (low-rank adapters on a quantized model)",
  "What QLoRA adds over LoRA": the per-block scales are quantised to 8 bits,
  no format named).  Per group of 256 absmax values s = fl32(max / 255) and
  code = min(255, rint(fl32(absmax / s))) with ties to even; a' = fl32(code s).
* Dequantisation: level[code] * absmax' in fp32, then bf16 for the matmul
  ("QLoRA (low-rank adapters on a quantized model)", last paragraph of
  "What QLoRA adds over LoRA"; "LLMs · QLoRA", ``levels[idx] * scale``).

Notation: fl32(v) = IEEE binary32 round-to-nearest-even of the exact real v;
every fl32 below is computed as an exact float64 operation followed by one
rounding to float32 (exact products of two fp32 values; for quotients the
float64 double rounding is innocuous since 53 >= 2*24 + 2).
"""

from __future__ import annotations

import math
import statistics
from fractions import Fraction

import numpy as np

BLOCK = 64          # weights per absmax block
GROUP = 256         # absmax values per double-quantisation fp32 scale
E4M3_MAX = 448.0    # largest finite OCP FP8 E4M3 value
U8_MAX = 255.0      # largest linear uint8 absmax code
DQ_FORMATS = ("e4m3", "u8")
DELTA = 0.5 * (31.0 / 32.0 + 29.0 / 30.0)   # quantile offset of the NF4 construction


# --------------------------------------------------------------------------
# small exact helpers
# --------------------------------------------------------------------------

def fl32(x) -> np.ndarray:
    """Round float64 values to the nearest binary32 (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def round_bf16(x32) -> np.ndarray:
    """Round binary32 values to bfloat16 (nearest, ties to even); returns float32.

    bfloat16 keeps the upper 16 bits of the binary32 pattern.  Written out on the
    bit pattern: add half of the dropped range, plus one more when the kept part
    is odd (ties to even), then clear the low 16 bits.  Finite inputs only.
    """
    x = np.ascontiguousarray(np.asarray(x32, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + keep_lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).reshape(x.shape)


# --------------------------------------------------------------------------
# codebooks
# --------------------------------------------------------------------------

def nf4_codebook() -> np.ndarray:
    """The 16 NF4 levels as float32, ascending; code index = rank.

    Positive half: normal quantiles at 8 evenly spaced probabilities from delta
    down to (but excluding) 1/2; negative half: the negated quantiles at 7 evenly
    spaced probabilities from delta down to (excluding) 1/2; plus an exact zero.
    All are divided by the largest quantile so the ends are exactly -1 and +1.
    """
    nd = statistics.NormalDist()
    top = nd.inv_cdf(DELTA)
    pos = [nd.inv_cdf(p) for p in np.linspace(DELTA, 0.5, 9)[:-1]]
    neg = [-nd.inv_cdf(p) for p in np.linspace(DELTA, 0.5, 8)[:-1]]
    levels = sorted(pos + [0.0] + neg)
    return fl32([v / top for v in levels])


def blog_codebook() -> np.ndarray:
    """"LLMs · QLoRA": approximate NF4-style levels, normal quantiles at
    linspace(0.02, 0.98, 16) divided by their largest magnitude (float32 steps,
    as the page computes them)."""
    nd = statistics.NormalDist()
    p = fl32(np.linspace(0.02, 0.98, 16))
    q = fl32([nd.inv_cdf(float(v)) for v in p])
    m = np.max(np.abs(q))
    return fl32(q.astype(np.float64) / np.float64(m))


def uniform4_codebook() -> np.ndarray:
    """"LLMs · QLoRA": the uniform 4-bit grid, 16 points evenly spaced on [-1, 1]."""
    return fl32(np.linspace(-1.0, 1.0, 16))


# --------------------------------------------------------------------------
# blockwise absmax + nearest level
# --------------------------------------------------------------------------

def block_absmax(w32: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """max |w| over each run of ``block`` consecutive elements of the flattened array."""
    w = np.asarray(w32, dtype=np.float32).reshape(-1, block)
    return np.abs(w).max(axis=1)


def scaled(w32: np.ndarray, absmax: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """x = fl32(w / absmax) per element; an all-zero block (absmax 0) gives x = 0."""
    w = np.asarray(w32, dtype=np.float32).reshape(-1, block).astype(np.float64)
    a = np.asarray(absmax, dtype=np.float32).astype(np.float64)[:, None]
    safe = np.where(a > 0.0, a, 1.0)
    x = np.where(a > 0.0, w / safe, 0.0)
    return fl32(x)


def nearest_level(x32: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """argmin_j |x - level_j| with ties to the lower j, in exact arithmetic.

    For ascending levels this is the number of midpoints m_j = (l_j + l_{j+1}) / 2
    that lie strictly below x (a tie x == m_j keeps the lower level).  The
    midpoints are exact in float64 (sums of two binary32 values of nearby
    magnitude), and ``searchsorted(side='left')`` counts #{j : m_j < x}.
    """
    lv = np.asarray(levels, dtype=np.float32).astype(np.float64)
    mids = (lv[:-1] + lv[1:]) / 2.0
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    return np.searchsorted(mids, x, side="left").astype(np.uint8)


def quantise_blockwise(w32: np.ndarray, levels: np.ndarray, block: int = BLOCK):
    """"LLMs · QLoRA" ``quantise``: per block absmax, nearest level, and the
    reconstruction level[code] * absmax (fp32).  No double quantisation.
    Returns (dequantised float32 flat array, codes uint8 flat array)."""
    w = np.asarray(w32, dtype=np.float32).reshape(-1)
    a = block_absmax(w, block)
    codes = nearest_level(scaled(w, a, block), levels).reshape(-1, block)
    lv = np.asarray(levels, dtype=np.float32).astype(np.float64)
    deq = fl32(lv[codes] * a.astype(np.float64)[:, None])
    return deq.reshape(-1), codes.reshape(-1)


# --------------------------------------------------------------------------
# OCP FP8 E4M3 (bias 7, no infinities, 0x7F / 0xFF are NaN, max finite 448)
# --------------------------------------------------------------------------

def e4m3_decode(code) -> np.ndarray:
    """Exact value of E4M3 bit patterns (float64; NaN for the NaN patterns)."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


_E4M3_POS = e4m3_decode(np.arange(0x7F))   # codes 0..126: all finite values >= 0, ascending


def e4m3_encode(y) -> np.ndarray:
    """Non-negative finite reals -> E4M3 code, round to nearest, ties to the
    even code (mantissa LSB 0), values above 448 saturate to 448 (0x7E)."""
    v = np.asarray(y, dtype=np.float64)
    if np.any(~np.isfinite(v)) or np.any(v < 0):
        raise ValueError("e4m3_encode takes finite non-negative values")
    hi = np.clip(np.searchsorted(_E4M3_POS, v, side="left"), 0, 0x7E)  # first table value >= v
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = _E4M3_POS[hi] - v
    d_lo = v - _E4M3_POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(v >= E4M3_MAX, 0x7E, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------
# NF4 + double quantisation of a whole weight matrix
# --------------------------------------------------------------------------

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Element 2k in the low nibble and 2k+1 in the high nibble of byte k."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


def double_quant(absmax: np.ndarray, group: int = GROUP, dq_format: str = "e4m3"):
    """Per group of ``group`` consecutive absmax values: s = fl32(max / 448),
    c_b = E4M3(fl32(a_b / s)) (``dq_format="e4m3"``), or s = fl32(max / 255),
    c_b = min(255, rint(fl32(a_b / s))) with ties to even (``"u8"``).  A group
    whose scale is 0 stores codes 0.  Returns (uint8 codes [nb], float32 scales
    [ceil(nb / group)])."""
    if dq_format not in DQ_FORMATS:
        raise ValueError(f"unknown double-quant format {dq_format!r}")
    top = E4M3_MAX if dq_format == "e4m3" else U8_MAX
    a = np.asarray(absmax, dtype=np.float32)
    nb = a.size
    ng = (nb + group - 1) // group
    codes = np.zeros(nb, dtype=np.uint8)
    scales = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        seg = a[g * group:(g + 1) * group]
        s = fl32(np.float64(seg.max()) / top)
        scales[g] = s
        if s > 0:
            y = fl32(seg.astype(np.float64) / np.float64(s))
            if dq_format == "e4m3":
                codes[g * group:(g + 1) * group] = e4m3_encode(y)
            else:
                codes[g * group:(g + 1) * group] = np.minimum(np.rint(y.astype(np.float64)), U8_MAX).astype(np.uint8)
    return codes, scales


def quantize_nf4(W0: np.ndarray, dq_format: str = "e4m3"):
    """fp32 W0 (in, out), row-major -> (packed NF4 codes [in*out/2],
    E4M3 (or linear uint8) absmax codes [in*out/64], fp32 group scales
    [ceil(in*out/64/256)]).

    Weights are coded against the exact fp32 absmax first; the absmax values are
    quantised afterwards (the order the pages list the two steps in)."""
    w = np.asarray(W0, dtype=np.float32)
    if w.size % BLOCK:
        raise ValueError("in*out must be a multiple of 64")
    if not np.all(np.isfinite(w)):
        raise ValueError("W0 must be finite")
    a = block_absmax(w)
    codes = nearest_level(scaled(w, a), nf4_codebook())
    dq_codes, dq_scales = double_quant(a, dq_format=dq_format)
    return pack_nibbles(codes), dq_codes, dq_scales


def absmax_dequant(dq_codes: np.ndarray, dq_scales: np.ndarray, group: int = GROUP,
                   dq_format: str = "e4m3") -> np.ndarray:
    """a'_b = fl32(e4m3(c_b) * s_g), or fl32(c_b * s_g) for ``"u8"`` (float32 [nb])."""
    if dq_format not in DQ_FORMATS:
        raise ValueError(f"unknown double-quant format {dq_format!r}")
    c = np.asarray(dq_codes, dtype=np.uint8)
    s = np.asarray(dq_scales, dtype=np.float32).astype(np.float64)
    g = np.arange(c.size) // group
    v = e4m3_decode(c) if dq_format == "e4m3" else c.astype(np.float64)
    return fl32(v * s[g])


def dequantize(codes, dq_codes, dq_scales, n_in: int, n_out: int, dq_format: str = "e4m3") -> np.ndarray:
    """w' = fl32(level[code] * a'_b) as float32 (n_in, n_out)."""
    lv = nf4_codebook().astype(np.float64)
    c = unpack_nibbles(codes).reshape(-1, BLOCK)
    a = absmax_dequant(dq_codes, dq_scales, dq_format=dq_format).astype(np.float64)
    return fl32(lv[c] * a[:, None]).reshape(n_in, n_out)


def dequantize_bf16(codes, dq_codes, dq_scales, n_in: int, n_out: int, dq_format: str = "e4m3") -> np.ndarray:
    """bf16(w'): the operand the matmuls use (float32 array holding bf16 values)."""
    return round_bf16(dequantize(codes, dq_codes, dq_scales, n_in, n_out, dq_format))


# --------------------------------------------------------------------------
# brute-force reference used by the pins (small inputs only)
# --------------------------------------------------------------------------

def nearest_level_exact(x: float, levels) -> int:
    """Direct argmin over the 16 levels in exact rational arithmetic."""
    fx = Fraction(float(x))
    best, best_d = 0, None
    for j, l in enumerate(levels):
        d = abs(fx - Fraction(float(l)))
        if best_d is None or d < best_d:
            best, best_d = j, d
    return best


def bits_per_weight(block: int = BLOCK, group: int = GROUP, code_bits: int = 4,
                    const_bits: int = 8, scale_bits: int = 32) -> float:
    """Storage per weight: code + 8-bit constant per block + fp32 scale per group."""
    return code_bits + const_bits / block + scale_bits / (block * group)


def isclose_rel(a: float, b: float, tol: float) -> bool:
    return math.isclose(a, b, rel_tol=tol)
