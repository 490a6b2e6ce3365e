"""Bit-exact encodings of the method, written from their definitions (oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

binary16 (IEEE 754-2008 section 3.6, "binary16"): 1 sign bit, 5 exponent bits
with bias 15, 10 fraction bits.  Normal numbers are (-1)^s 2^(E-15) (1 + f/1024)
for E in 1..30, subnormals (-1)^s 2^-14 (f/1024), the largest finite value is
65504, and roundTiesToEven rounding (section 4.3.1) sends |v| >= 65520 to inf.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# binary16 conversion, from the definition
# ----------------------------------------------------------------------------

F16_MAX = 65504.0
F16_OVERFLOW = 65520.0  # midpoint between 65504 and 2^16; ties-to-even goes up


_CHUNK = 1 << 18


def rn16_bits(v) -> np.ndarray:
    """Round float64 values to binary16 (round half to even); return the bits.

    Evaluated in fixed-size chunks (see `_rn16_bits_chunk`) so large arrays do
    not allocate large temporaries.
    """
    v = np.asarray(v, dtype=np.float64)
    flat = np.ascontiguousarray(v).reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    for i in range(0, flat.size, _CHUNK):
        out[i:i + _CHUNK] = _rn16_bits_chunk(flat[i:i + _CHUNK])
    return out.reshape(v.shape)


def _rn16_bits_chunk(v) -> np.ndarray:
    """Round float64 values to binary16 (round half to even); return the bits.

    Works on the exact float64 encoding: the value is m 2^(E-1075) with the
    53-bit integer significand m.  The binary16 quantum of the value's binade is
    2^max(e-10, -24) (e the unbiased exponent), so the rounded significand is
    m shifted right by the exponent difference, rounded half-to-even on the
    discarded bits.  Sign, exponent and fraction are then assembled.  Values
    >= 2^16 and rounding carries past 65504 become inf; NaN maps to 0x7E00.
    """
    v = np.ascontiguousarray(v, dtype=np.float64)
    u = v.view(np.uint64)
    sign = ((u >> np.uint64(63)).astype(np.uint16) << np.uint16(15))
    E64 = ((u >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    frac = u & np.uint64((1 << 52) - 1)
    m = frac | np.uint64(1 << 52)
    e = E64 - 1023
    qe = np.maximum(e - 10, -24)                 # exponent of the binary16 quantum
    shift = qe - (E64 - 1075)                    # >= 42 for every finite value < 2^16
    big = shift >= 64
    sh = np.clip(shift, 1, 63).astype(np.uint64)
    n = m >> sh
    rem = m & ((np.uint64(1) << sh) - np.uint64(1))
    half = np.uint64(1) << (sh - np.uint64(1))
    up = (rem > half) | ((rem == half) & ((n & np.uint64(1)) == np.uint64(1)))
    n = (n + up.astype(np.uint64)).astype(np.int64)
    n = np.where(big, 0, n)
    normal = e >= -14
    carry = normal & (n >= 2048)
    e_n = np.where(carry, e + 1, e)
    n_n = np.where(carry, 1024, n)
    bits_nrm = ((e_n + 15) << 10) + (n_n - 1024)
    bits = np.where(normal, bits_nrm, n)         # subnormal: bits == n (n == 1024 is 0x0400)
    bits = np.where(normal & (e_n > 15), 0x7C00, bits)
    bits = np.where(e >= 16, 0x7C00, bits)       # |v| >= 2^16 (and inf)
    bits = np.where((E64 == 0), 0, bits)         # zero and float64 subnormals round to 0
    out = (bits.astype(np.uint16) | sign)
    nan = (E64 == 0x7FF) & (frac != 0)
    return np.where(nan, np.uint16(0x7E00), out).astype(np.uint16)


def f16_bits_to_f64(bits) -> np.ndarray:
    """Decode binary16 bit patterns to float64 (exact), from the definition."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    s = np.where((b >> 15) & 1, -1.0, 1.0)
    E = (b >> 10) & 0x1F
    f = (b & 0x3FF).astype(np.float64)
    val = np.where(E == 0, np.ldexp(f, -24),
                   np.ldexp(1.0 + f / 1024.0, (E - 15).astype(np.int64)))
    val = np.where(E == 31, np.where(f == 0, np.inf, np.nan), val)
    return s * val


# ----------------------------------------------------------------------------
# HEAL operand split  [HEAL, section "2. 「誤差補償」のトリック（計算用）"]
# ----------------------------------------------------------------------------
# The explainer describes a main product done in standard 16-bit containers
# and a fast "clean-up" product that recovers what the main product spilled.
# Reading used here: an fp32 value x (times an exact power of two 2^e) is
# carried as a pair of binary16 values
#     hi = rn16(x 2^e),   lo = rn16((x 2^e - hi) 2^11),
# so that x 2^e ~= hi + 2^-11 lo.  The 2^11 pre-scale keeps lo in the normal
# binary16 range (Ootomo & Yokota 2022), giving a reconstruction error of at
# most 2^-22 |x| whenever 2^-14 <= |x 2^e| < 65520.

LO_SCALE_LOG2 = 11
PACK_BN = 128  # output columns per packed weight panel (layout constant)


def heal_split(x, e=0):
    """Split fp32 values into (hi_bits, lo_bits) binary16 patterns.

    `e` is an integer exponent broadcast against x (0 for activations, the
    per-column exponent for weights).  Returns (hi, lo, overflow_mask).
    """
    v = np.ldexp(np.asarray(x, dtype=np.float32).astype(np.float64), np.asarray(e, dtype=np.int64))
    hi = rn16_bits(v)
    hv = f16_bits_to_f64(hi)
    overflow = ~np.isfinite(hv) & np.isfinite(v)
    r = np.where(np.isfinite(hv), np.ldexp(v - np.where(np.isfinite(hv), hv, 0.0), LO_SCALE_LOG2), 0.0)
    lo = rn16_bits(r)
    return hi, lo, overflow


def heal_reconstruct(hi, lo, e=0) -> np.ndarray:
    """float64 value of a (hi, lo) pair: (hi + 2^-11 lo) 2^-e."""
    return np.ldexp(f16_bits_to_f64(hi) + np.ldexp(f16_bits_to_f64(lo), -LO_SCALE_LOG2),
                    -np.asarray(e, dtype=np.int64))


def column_exponents(W) -> np.ndarray:
    """Static per-output-column exponent e_n of a weight matrix W[K, N].

    e_n is the integer with max_k |W[k, n]| 2^e_n in [2^14, 2^15): frexp gives
    max = m 2^E with m in [0.5, 1), so e_n = 15 - E.  An all-zero column gets 0.
    Clamped to [-120, 120] so that 2^e_n and 2^-e_n are normal fp32 numbers.
    """
    W = np.asarray(W, dtype=np.float32)
    mx = np.max(np.abs(W), axis=0).astype(np.float64)
    _, E = np.frexp(mx)
    e = np.where(mx > 0, 15 - E.astype(np.int64), 0)
    return np.clip(e, -120, 120).astype(np.int8)


def heal_pack_weight(W):
    """Packed weight image and column exponents for the compensated GEMM.

    W is fp32 [K, N] (y = x W), N a multiple of PACK_BN.  The image is binary16
    bit patterns laid out [N/128][2][128][K]: panel j holds, for its 128 output
    columns n = 128 j + r, first the hi rows then the lo rows, each row
    contiguous along K.  Returns (packed uint16 [N/128, 2, 128, K], e int8 [N]).
    """
    W = np.asarray(W, dtype=np.float32)
    K, N = W.shape
    assert N % PACK_BN == 0
    e = column_exponents(W)
    hi, lo, _ = heal_split(W, e[None, :].astype(np.int64))
    P = np.empty((N // PACK_BN, 2, PACK_BN, K), dtype=np.uint16)
    P[:, 0] = hi.T.reshape(N // PACK_BN, PACK_BN, K)
    P[:, 1] = lo.T.reshape(N // PACK_BN, PACK_BN, K)
    return P, e


# ----------------------------------------------------------------------------
# INT16 KV-cache quantiser  [HEAL, section "1. 「スマート・パッキング」のトリック"]
# ----------------------------------------------------------------------------
# The explainer packs K and V into INT16 "packing tape".  Reading used here:
# symmetric, one scale per (token, kv head):  s = fl32(max_d |x_d| / 32767),
# q_d = clamp(round_half_even(fl32(x_d / s)), -32767, 32767), with IEEE fp32
# division (not a reciprocal multiply); max == 0 (or an underflowed s == 0)
# gives s = 0 and q = 0.  -32768 is never produced.

QMAX = 32767


def kv_quant_int16(x):
    """Quantise fp32 x[..., D] per leading index; returns (codes int16, scale fp32)."""
    x = np.asarray(x, dtype=np.float32)
    mx = np.max(np.abs(x), axis=-1)                     # exact in fp32
    s = (mx / np.float32(QMAX)).astype(np.float32)      # one IEEE fp32 division
    with np.errstate(divide="ignore", invalid="ignore"):
        quo = (x / s[..., None]).astype(np.float32)     # IEEE fp32 division
    q = np.rint(quo)                                    # round half to even
    q = np.where((s == 0)[..., None], 0.0, q)
    q = np.clip(q, -QMAX, QMAX).astype(np.int16)
    return q, s


def kv_dequant(codes, scale) -> np.ndarray:
    """Exact float64 value of INT16 codes times their fp32 scale."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


# ----------------------------------------------------------------------------
# Dual-FP16 unpack of an INT16 code  [HEAL, section "1. スマート・パッキング",
# the package is opened into two small (16-bit) buckets for computation]
# ----------------------------------------------------------------------------
# Reading used here: q = 256 h + l with h = q >> 8 (signed high byte, -128..127)
# and l = q & 255 (0..255).  Both h and l (and 256 h) are exact binary16 values,
# so the pair carries the 15-bit code without loss through 16-bit arithmetic.

def dual_fp16_unpack(codes):
    q = np.asarray(codes, dtype=np.int16).astype(np.int64)
    h = q >> 8
    l = q & 0xFF
    return h, l
