"""E4M3 quantisation for the low-precision logits option, from the format definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages cite quantised deployments of the model (axbrief.com brief, "deployment on a
24 GB GPU": GGUF Q8_0 ... Q4_K_M sizes; molayo1419.me blog, summary: a 4-bit load) but
define no quantisation of this stage.  Reading taken here: the vocabulary head W is stored
as 8-bit E4M3 codes with one power-of-two scale for the whole tensor, the hidden states
are quantised per position (row) the same way at every step, and the logits are
z = 2^(e_h + e_W) (h_q . W_q) / T on the decoded values.  The self-conditioning vector
keeps the bf16 embedding E.

E4M3 ("fn" variant of the 8-bit floating-point formats): sign bit, 4 exponent bits with
bias 7, 3 mantissa bits.  Exponent field 0 holds the subnormals m/8 * 2^-6; field 15 with
mantissa 7 is NaN; there are no infinities; the largest finite value is 1.75 * 2^8 = 448.

A power-of-two scale makes x * 2^-e exact, so the only rounding is the E4M3 rounding
(round to nearest, ties to the even mantissa), a deterministic function of the exact value.

Parity status: pinned by tests/test_oracle_fp8.py (the code table from the bit fields,
round trips, ties to even, nearest-value property, an independent library conversion on
in-range values, the scale's minimality, and the logit error bound).
"""

import numpy as np

E4M3_MAX = 448.0
_SUB = 2.0 ** -9          # subnormal step (and the smallest positive value)
_MIN_NORMAL = 2.0 ** -6


def decode(codes):
    """E4M3 codes (uint8) -> float64 values (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    field = (c >> 3) & 0xF
    mant = c & 0x7
    mag = np.where(field == 0, mant * _SUB, (1.0 + mant / 8.0) * np.exp2(field - 7.0))
    mag = np.where((field == 15) & (mant == 7), np.nan, mag)
    return sign * mag


def encode(x):
    """float64 -> E4M3 codes: round to nearest, ties to even mantissa; magnitudes above 448
    saturate to 448 (the quantisers below never produce them); NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    out = np.zeros(x.shape, dtype=np.int64)
    normal = a >= _MIN_NORMAL
    # subnormal range: a multiple of 2^-9, rounded to even; 8 * 2^-9 is the first normal (code 8)
    q = np.rint(np.where(normal, 0.0, a) / _SUB).astype(np.int64)
    out = np.where(normal, 0, q)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, e2 = np.frexp(np.where(normal, a, 1.0))      # a = f 2^e2 with f in [0.5, 1)
        E = e2 - 1                                       # a in [2^E, 2^(E+1))
        m = np.rint((np.where(normal, a, 1.0) / np.exp2(E) - 1.0) * 8.0).astype(np.int64)
    E = np.where(m == 8, E + 1, E)
    m = np.where(m == 8, 0, m)
    code_n = (E + 7) * 8 + m
    code_n = np.minimum(code_n, 0x7E)                   # saturate at 448
    out = np.where(normal, code_n, out)
    out = np.where(np.isnan(x), 0x7F, out)
    out = out | np.where(neg & ~np.isnan(x), 0x80, 0)
    return out.astype(np.uint8)


def pow2_exponent(amax):
    """The smallest integer e with amax * 2^-e <= 448 (0 for an all-zero tensor)."""
    amax = float(amax)
    if amax == 0.0 or not np.isfinite(amax):
        return 0
    _, e = np.frexp(amax / E4M3_MAX)                     # a first guess, then exact comparisons
    e = int(e)
    while np.ldexp(amax, -e) > E4M3_MAX:                 # amax 2^-e is exact: a power-of-two scaling
        e += 1
    while np.ldexp(amax, -(e - 1)) <= E4M3_MAX:
        e -= 1
    return e


def quantize_tensor(x):
    """One power-of-two scale for the whole tensor: (codes uint8, e) with x ~ decode(codes) * 2^e."""
    x = np.asarray(x, dtype=np.float64)
    e = pow2_exponent(np.max(np.abs(x)) if x.size else 0.0)
    return encode(x * np.exp2(-e)), e


def quantize_rows(x):
    """One power-of-two scale per row: (codes [n, d] uint8, e [n] int32)."""
    x = np.asarray(x, dtype=np.float64)
    e = np.array([pow2_exponent(v) for v in np.max(np.abs(x), axis=1)], dtype=np.int32)
    return encode(x * np.exp2(-e.astype(np.float64))[:, None]), e


def dequantize_tensor(codes, e):
    return decode(codes) * np.exp2(float(e))


def dequantize_rows(codes, e):
    return decode(codes) * np.exp2(np.asarray(e, dtype=np.float64))[:, None]
