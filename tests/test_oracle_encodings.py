"""Pins for the oracle's bit-exact encodings (CPU only).

Each encoding is checked against something other than itself: hand-derived
golden cases (tests/golden/*.txt, with their derivations), an independent
library conversion (numpy's float16 cast, torch's round-half-even), closed-form
error bounds and exact rational arithmetic.
"""
import os
import warnings
from fractions import Fraction

import numpy as np
import torch

from oracle import encodings as enc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_fp16():
    rows = []
    with open(os.path.join(GOLDEN, "fp16_rne.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            expr, bits = line.split()
            rows.append((float(eval(expr)), int(bits, 16)))
    return rows


def test_rn16_golden_cases():
    rows = _golden_fp16()
    got = enc.rn16_bits(np.array([r[0] for r in rows]))
    for (v, want), g in zip(rows, got):
        assert int(g) == want, (v, hex(int(g)), hex(want))


def _rounding_relevant_fp32():
    """fp32 patterns around every binary16 rounding boundary: for each fp32
    binade that can round to a finite nonzero binary16, every kept-bit pattern
    (up to 1024 of them) combined with the discarded-bit tails 0, 1, half-1,
    half, half+1 and all-ones."""
    out = []
    for e in range(-26, 17):
        drop = 13 if e >= -14 else min(23, 13 + (-14 - e))
        keep_bits = 23 - drop
        half = 1 << (drop - 1)
        tails = np.array([0, 1, half - 1, half, half + 1, (1 << drop) - 1], dtype=np.uint64)
        kept = np.arange(1 << keep_bits, dtype=np.uint64) << np.uint64(drop)
        mant = (kept[:, None] | tails[None, :]).reshape(-1)
        expf = np.uint64(e + 127) << np.uint64(23)
        for sgn in (0, 1):
            out.append((np.uint64(sgn) << np.uint64(31)) | expf | mant)
    return np.concatenate(out).astype(np.uint32).view(np.float32)


def test_rn16_matches_numpy_cast_on_every_rounding_boundary():
    x = _rounding_relevant_fp32()
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")              # signalling NaNs among the random bit patterns
        want = x.astype(np.float16).view(np.uint16)
        xd = x.astype(np.float64)
    got = enc.rn16_bits(xd)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]


def test_rn16_matches_numpy_cast_on_random_fp32():
    r = np.random.Generator(np.random.PCG64(1234)).integers(0, 2**32, size=1 << 21, dtype=np.uint64)
    x = r.astype(np.uint32).view(np.float32)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")              # signalling NaNs among the random bit patterns
        want = x.astype(np.float16).view(np.uint16)
        xd = x.astype(np.float64)
    got = enc.rn16_bits(xd)
    ok = (got == want) | np.isnan(x)
    assert ok.all()


def test_rn16_matches_numpy_cast_on_every_fp32():
    """All 2^32 fp32 bit patterns, in blocks of 2^24 over spawned processes."""
    import concurrent.futures as cf
    import multiprocessing as mp
    from rn16_sweep import check_block
    block = 1 << 24
    workers = max(1, min(8, os.cpu_count() or 1))
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        results = list(ex.map(check_block, range(0, 1 << 32, block), [block] * ((1 << 32) // block)))
    n_bad = sum(r[0] for r in results)
    assert n_bad == 0, [r[1] for r in results if r[0]][:3]


def test_f16_decode_exhaustive_and_roundtrip():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    want = b.view(np.float16).astype(np.float64)
    got = enc.f16_bits_to_f64(b)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    fin = np.isfinite(want)
    assert (enc.rn16_bits(got[fin]) == b[fin]).all()


def test_heal_split_reconstruction_bound():
    g = np.random.Generator(np.random.PCG64(7))
    mag = np.exp2(g.uniform(-14, 15.99, size=200000))
    x = (mag * np.where(g.random(200000) < 0.5, -1, 1)).astype(np.float32)
    hi, lo, ovf = enc.heal_split(x)
    assert not ovf.any()
    rec = enc.heal_reconstruct(hi, lo)
    err = np.abs(rec - x.astype(np.float64))
    assert (err <= np.abs(x.astype(np.float64)) * 2.0**-22).all()
    # hi is the nearest binary16 value (independent cast)
    assert (hi == x.astype(np.float16).view(np.uint16)).all()


def test_heal_split_residual_is_exact():
    # x - hi is computed in float64; check it against exact rational arithmetic
    g = np.random.Generator(np.random.PCG64(8))
    x = g.standard_normal(300).astype(np.float32)
    hi, lo, _ = enc.heal_split(x)
    hv = enc.f16_bits_to_f64(hi)
    for xi, hvi, loi in zip(x, hv, lo):
        r = Fraction(float(xi)) - Fraction(float(hvi))
        r_scaled = r * 2048
        lo_want = enc.rn16_bits(np.array([float(r_scaled)]))[0]
        assert float(r_scaled) == r_scaled  # exactly representable
        assert lo_want == loi


def test_heal_split_fp16_exact_inputs_have_zero_lo():
    vals = np.array([1.0, -3.5, 1024.0, 2.0**-14, 65504.0, 0.0], dtype=np.float32)
    hi, lo, _ = enc.heal_split(vals)
    assert (enc.f16_bits_to_f64(lo) == 0).all()
    assert (enc.f16_bits_to_f64(hi) == vals).all()


def test_heal_split_flags_overflow():
    _, _, ovf = enc.heal_split(np.array([65519.0, 65520.0, -70000.0, 1.0], dtype=np.float32))
    assert ovf.tolist() == [False, True, True, False]


def test_column_exponents_closed_form():
    W = np.array([[0.02, 3.0, 0.0, 1e5],
                  [-0.07, 1.0, 0.0, -2.0]], dtype=np.float32)
    e = enc.column_exponents(W).astype(np.int64)
    for n in range(W.shape[1]):
        mx = float(np.max(np.abs(W[:, n])))
        if mx == 0:
            assert e[n] == 0
        else:
            assert 2.0**14 <= mx * 2.0**e[n] < 2.0**15
    assert e[2] == 0


def test_pack_weight_layout_and_values():
    K, N = 64, 256
    # W[k, n] built from small integers and a per-column power of two so the
    # scaled values are exact binary16 numbers (lo == 0) with a known position.
    k = np.arange(K)[:, None]
    n = np.arange(N)[None, :]
    W = ((k + 1) * 3 + (n % 7)).astype(np.float32) * np.float32(2.0**-6)
    P, e = enc.heal_pack_weight(W)
    assert P.shape == (N // 128, 2, 128, K) and P.dtype == np.uint16
    for j in range(N // 128):
        for r in (0, 5, 64, 127):
            col = 128 * j + r
            hv = enc.f16_bits_to_f64(P[j, 0, r, :])
            lv = enc.f16_bits_to_f64(P[j, 1, r, :])
            assert (hv == W[:, col].astype(np.float64) * 2.0**int(e[col])).all()
            assert (lv == 0).all()
    # a generic matrix reconstructs within 2^-22 relative on normal elements
    g = np.random.Generator(np.random.PCG64(3))
    W2 = (g.standard_normal((128, 128)) * 0.02).astype(np.float32)
    P2, e2 = enc.heal_pack_weight(W2)
    rec = enc.heal_reconstruct(P2[0, 0].T, P2[0, 1].T, e2[None, :].astype(np.int64))
    normal = np.abs(W2) * 2.0**e2[None, :].astype(np.float64) >= 2.0**-14
    err = np.abs(rec - W2.astype(np.float64))
    assert (err[normal] <= 2.0**-22 * np.abs(W2.astype(np.float64))[normal]).all()
    assert (err <= 2.0**-36 * 2.0**-e2[None, :].astype(np.float64) + 2.0**-22 * np.abs(W2)).all()


def _golden_quant():
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, "int16_quant.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            cur[key.strip()] = eval(val)
            if key.strip() == "q":
                cases.append(cur)
                cur = {}
    return cases


def test_kv_quant_golden_cases():
    for c in _golden_quant():
        x = np.array(c["x"], dtype=np.float32)[None, :]
        q, s = enc.kv_quant_int16(x)
        assert q[0].tolist() == c["q"], c
        if c["s"] is not None:
            assert float(s[0]) == c["s"], c


def test_kv_quant_matches_torch_and_bounds():
    g = np.random.Generator(np.random.PCG64(11))
    x = (g.standard_normal((4000, 128)) * np.exp(g.uniform(-5, 5, size=(4000, 1)))).astype(np.float32)
    q, s = enc.kv_quant_int16(x)
    # independent library: torch fp32 max/div and round-half-even
    xt = torch.from_numpy(x)
    st = xt.abs().amax(dim=-1) / torch.tensor(32767.0, dtype=torch.float32)
    qt = torch.round(xt / st[:, None]).clamp(-32767, 32767).to(torch.int16)
    assert np.array_equal(s, st.numpy())
    assert np.array_equal(q, qt.numpy())
    # round-trip bound |x - q s| <= s (1/2 + 2^-9)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s.astype(np.float64)[:, None])
    assert (err <= s.astype(np.float64)[:, None] * (0.5 + 2.0**-9)).all()
    # the max element maps to +-32767 and -32768 is never used
    amax = np.argmax(np.abs(x), axis=1)
    assert (np.abs(q[np.arange(4000), amax]) == 32767).all()
    assert q.min() >= -32767
    # odd symmetry
    qn, sn = enc.kv_quant_int16(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)


def test_dual_fp16_unpack_exhaustive():
    codes = np.arange(-32768, 32768, dtype=np.int64).astype(np.int16)
    h, l = enc.dual_fp16_unpack(codes)
    assert np.array_equal(256 * h + l, codes.astype(np.int64))
    assert h.min() == -128 and h.max() == 127 and l.min() == 0 and l.max() == 255
    for part in (h, l, 256 * h):
        dec = enc.f16_bits_to_f64(enc.rn16_bits(part.astype(np.float64)))
        assert np.array_equal(dec, part.astype(np.float64))
