"""GPU parity of every kernel against the CPU oracle, through the C ABI.

Bit-exact: binary16 hi/lo splits, the packed weight image, INT16 codes and
scales.  fp32 outputs: normwise relative error per row <= 1e-5 against the
float64 oracle.  Inputs follow the workloads' distributions (synth module).
"""
import numpy as np
import pytest
import torch

from invariant_numerics_b200 import synth
from oracle import encodings as enc
from oracle import reference as ref

from gpu_helpers import TOL, bits16, dev, host, rowwise_err, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


# ------------------------------------------------------------- heal_split ----

def test_heal_split_bit_exact(inv):
    g = np.random.Generator(np.random.PCG64(0))
    x = synth.normal_with_outliers((37, 520), seed=1).astype(np.float64)
    x[0, :64] = np.exp2(g.uniform(-30, 15.9, 64)) * np.sign(g.standard_normal(64))   # tiny and large magnitudes
    x[1, :8] = [0.0, -0.0, 1.0, 65504.0, 2.0**-24, 2.0**-25, 1 + 2.0**-11, -3.0]
    x = x.astype(np.float32)
    hi, lo = inv.heal_split(dev(x))
    h_want, l_want, _ = enc.heal_split(x)
    assert np.array_equal(bits16(hi), h_want)
    assert np.array_equal(bits16(lo), l_want)
    assert status() == inv.INV_OK
    # odd column count takes the scalar path
    hi3, lo3 = inv.heal_split(dev(x[:, :7].copy()))
    assert np.array_equal(bits16(hi3), h_want[:, :7]) and np.array_equal(bits16(lo3), l_want[:, :7])


def test_heal_split_range_error(inv):
    x = np.array([[1.0, 70000.0, 2.0, 3.0]], np.float32)
    inv.heal_split(dev(x))
    assert status() == inv.INV_ERR_RANGE
    assert status() == inv.INV_OK  # cleared by the read


def test_pack_weight_bit_exact(inv):
    for K, N, std in ((512, 512, 0.02), (1024, 384, 3.0), (64, 128, 1e-6)):
        W = synth.normal((K, N), seed=K + N, std=std)
        W[0, 0] = 0.0
        if N > 128:
            W[:, 128:256] = 0.0  # an all-zero panel
        P, e = inv.heal_pack_weight(dev(W))
        P_want, e_want = enc.heal_pack_weight(W)
        assert np.array_equal(host(e), e_want)
        assert np.array_equal(bits16(P).reshape(P_want.shape), P_want)


# ------------------------------------------------------------- rmsnorm -------

@pytest.mark.parametrize("hidden", [512, 4096, 68, 8196])
def test_rmsnorm_parity(inv, hidden):
    x = synth.normal((9, hidden), seed=hidden)
    x[3] *= 1e-3
    x[4] = 2.5  # constant row
    gamma = synth.uniform(hidden, seed=hidden + 1, lo=0.5, hi=1.5)
    y, hi, lo = inv.rmsnorm_bi(dev(x), dev(gamma), 1e-6, want_y=True, want_split=True)
    want = ref.rmsnorm(x, gamma, 1e-6)
    assert rowwise_err(host(y), want).max() <= 1e-6
    # the fused split is the oracle's binary16 encoding of the kernel's own fp32 output, bit for bit
    h_want, l_want, _ = enc.heal_split(host(y))
    assert np.array_equal(bits16(hi), h_want)
    assert np.array_equal(bits16(lo), l_want)


def test_rmsnorm_rows_batch_invariant(inv):
    x = synth.normal((256, 4096), seed=3)
    gamma = synth.uniform(4096, seed=4, lo=0.5, hi=1.5)
    xd, gd = dev(x), dev(gamma)
    full = inv.rmsnorm_bi(xd, gd, 1e-6)
    for M in (1, 2, 7, 64, 255):
        part = inv.rmsnorm_bi(xd[:M].contiguous(), gd, 1e-6)
        assert torch.equal(part.view(torch.int32), full[:M].view(torch.int32))
    perm = torch.from_numpy(synth.permutation(256, seed=5)).cuda()
    shuf = inv.rmsnorm_bi(xd[perm].contiguous(), gd, 1e-6)
    assert torch.equal(shuf.view(torch.int32), full[perm].view(torch.int32))


# ------------------------------------------------------------- kv_quant ------

def test_kv_quant_bit_exact(inv):
    T, Hkv, D = 300, 8, 128
    c = synth.channel_scale(Hkv, D, seed=7)
    x = synth.kv_tensor(T, Hkv, D, seed=8, scale=c)
    x[5] = 0.0                                   # all-zero rows -> s = 0, q = 0
    x[6, 0] = 2.0**-140                          # underflowing scale
    x[7, 1, :4] = [32767 * 2.0**-10, 2.5 * 2.0**-10, 3.5 * 2.0**-10, -2.5 * 2.0**-10]
    x[7, 1, 4:] = 0.0
    q_want, s_want = enc.kv_quant_int16(x)
    cache = inv.KVCache(n_slots=3, n_kv_heads=Hkv, max_len=128)
    slot = (np.arange(T) % 3).astype(np.int32)
    pos = (np.arange(T) // 3).astype(np.int32)
    inv.kv_quant_int16(dev(x), dev(slot), dev(pos), cache, "k")
    inv.kv_quant_int16(dev(-x), dev(slot), dev(pos), cache, "v")
    assert status() == inv.INV_OK
    kc, ks, vc, vs = host(cache.k), host(cache.k_scale), host(cache.v), host(cache.v_scale)
    for t in range(T):
        assert np.array_equal(kc[slot[t], :, pos[t]], q_want[t])
        assert np.array_equal(ks[slot[t], :, pos[t]], s_want[t])
        assert np.array_equal(vc[slot[t], :, pos[t]], -q_want[t])
        assert np.array_equal(vs[slot[t], :, pos[t]], s_want[t])


def test_kv_quant_bad_index_reports(inv):
    cache = inv.KVCache(n_slots=1, n_kv_heads=8, max_len=64)
    x = synth.kv_tensor(2, 8, 128, seed=9)
    inv.kv_quant_int16(dev(x), dev(np.array([0, 1], np.int32)), dev(np.array([0, 0], np.int32)), cache, "k")
    assert status() == inv.INV_ERR_INVALID_ARG


# ------------------------------------------------------------- comp_gemm -----

def test_comp_gemm_tiny_config(inv):
    """RMSNorm(512) then the compensated GEMM K = N = 512, M = 1..8."""
    x = synth.normal((8, 512), seed=0)
    gamma = synth.uniform(512, seed=1, lo=0.5, hi=1.5)
    W = synth.normal((512, 512), seed=2, std=0.02)
    P, e = inv.heal_pack_weight(dev(W))
    h_hi, h_lo = inv.rmsnorm_bi(dev(x), dev(gamma), 1e-6, want_y=False, want_split=True)
    want = ref.gemm(ref.rmsnorm(x, gamma, 1e-6), W)
    outs = []
    for M in range(1, 9):
        y = inv.comp_gemm(h_hi[:M].contiguous(), h_lo[:M].contiguous(), P, e)
        assert rowwise_err(host(y), want[:M]).max() <= TOL
        outs.append(y)
    for M in range(1, 9):  # each row bit-identical for every batch size
        assert torch.equal(outs[M - 1].view(torch.int32), outs[-1][:M].view(torch.int32))
    assert status() == inv.INV_OK


def test_comp_gemm_invariance_across_row_placement(inv):
    """Rows land in different tiles and tensor-memory lanes (and, for M < 128,
    in a trimmed A box) depending on M and offset: a row's bits must not
    depend on where it lands."""
    K, N = 1024, 384
    A = synth.normal_with_outliers((600, K), seed=13)
    W = synth.normal((K, N), seed=14, std=0.02)
    P, e = inv.heal_pack_weight(dev(W))
    hi, lo = inv.heal_split(dev(A))
    full = inv.comp_gemm(hi, lo, P, e)
    assert rowwise_err(host(full), ref.gemm(A, W)).max() <= TOL
    for M in (1, 7, 8, 9, 63, 64, 65, 127, 128, 129, 255, 256, 257, 511, 513):
        y = inv.comp_gemm(hi[:M].contiguous(), lo[:M].contiguous(), P, e)
        assert torch.equal(y.view(torch.int32), full[:M].view(torch.int32)), M
    for off in (1, 64, 100):  # the same rows at other positions
        y = inv.comp_gemm(hi[off:off + 130].contiguous(), lo[off:off + 130].contiguous(), P, e)
        assert torch.equal(y.view(torch.int32), full[off:off + 130].view(torch.int32)), off
    assert status() == inv.INV_OK


def test_comp_gemm_invariance_across_column_placement(inv):
    """A column's bits depend on nothing but its own weights and K order: the
    same weight columns give the same bits in another panel or another N."""
    K = 2048
    A = synth.normal_with_outliers((200, K), seed=15)
    W = synth.normal((K, 512), seed=16, std=0.02)
    hi, lo = inv.heal_split(dev(A))
    P, e = inv.heal_pack_weight(dev(W))
    full = inv.comp_gemm(hi, lo, P, e)
    for c0, c1 in ((128, 256), (256, 512), (0, 384)):
        Ps, es = inv.heal_pack_weight(dev(W[:, c0:c1].copy()))
        part = inv.comp_gemm(hi, lo, Ps, es)
        assert torch.equal(part.view(torch.int32), full[:, c0:c1].contiguous().view(torch.int32)), (c0, c1)
    assert status() == inv.INV_OK


@pytest.mark.parametrize("N", [4096, 11008])
def test_comp_gemm_sweep_parity_and_invariance(inv, N):
    K = 4096
    A = synth.normal_with_outliers((1024, K), seed=10)
    W = synth.normal((K, N), seed=11, std=0.02)
    P, e = inv.heal_pack_weight(dev(W))
    hi, lo = inv.heal_split(dev(A))
    full = inv.comp_gemm(hi, lo, P, e)
    rows = np.array([0, 1, 2, 16, 63, 127, 128, 255, 256, 511, 777, 1023])
    want = ref.gemm(A[rows], W)
    err = rowwise_err(host(full)[rows], want)
    assert err.max() <= TOL, err
    e16 = rowwise_err(ref.gemm_fp16_only(A[rows], W), want)
    assert err.max() <= 1e-2 * e16.min()
    for M in (1, 3, 17, 64, 256):
        y = inv.comp_gemm(hi[:M].contiguous(), lo[:M].contiguous(), P, e)
        assert torch.equal(y.view(torch.int32), full[:M].view(torch.int32)), M
    perm = torch.from_numpy(synth.permutation(1024, seed=12)).cuda()
    ys = inv.comp_gemm(hi[perm].contiguous(), lo[perm].contiguous(), P, e)
    assert torch.equal(ys.view(torch.int32), full[perm].view(torch.int32))
    assert status() == inv.INV_OK


def test_comp_gemm_ragged_and_residual(inv):
    M, K, N = 133, 320, 256
    A = synth.normal((M, K), seed=20)
    W = synth.normal((K, N), seed=21, std=0.5)
    R = synth.normal((M, N), seed=22)
    P, e = inv.heal_pack_weight(dev(W))
    hi, lo = inv.heal_split(dev(A))
    y = inv.comp_gemm(hi, lo, P, e, residual=dev(R))
    want = ref.gemm(A, W) + R.astype(np.float64)
    assert rowwise_err(host(y), want).max() <= TOL
    # in place: y aliases the residual
    Rd = dev(R)
    inv.comp_gemm(hi, lo, P, e, residual=Rd, out=Rd)
    assert torch.equal(Rd.view(torch.int32), y.view(torch.int32))


def test_comp_gemm_rejects_bad_shapes(inv):
    hi = torch.zeros((4, 100), dtype=torch.float16, device="cuda")
    P = torch.zeros((1, 2, 128, 100), dtype=torch.float16, device="cuda")
    e = torch.zeros((128,), dtype=torch.int8, device="cuda")
    with pytest.raises(inv.InvError) as ei:
        inv.comp_gemm(hi, hi, P, e)       # K % 64 != 0
    assert ei.value.code == inv.INV_ERR_UNSUPPORTED_SHAPE


# ------------------------------------------------------------- attention -----

def _attn_case(inv, B, Hq, Hkv, lens, seed, max_len):
    D = 128
    c = synth.channel_scale(Hkv, D, seed=seed)
    ocache = ref.KVCache.empty(B, Hkv, max_len, D)
    gcache = inv.KVCache(n_slots=B, n_kv_heads=Hkv, max_len=max_len)
    for b in range(B):
        L = int(lens[b])
        k = synth.kv_tensor(L, Hkv, D, seed=seed + 1, stream=b, scale=c)
        v = synth.kv_tensor(L, Hkv, D, seed=seed + 2, stream=b, scale=c)
        pos = np.arange(L, dtype=np.int32)
        sl = np.full(L, b, np.int32)
        ocache.write("k", k, sl, pos)
        ocache.write("v", v, sl, pos)
        inv.kv_quant_int16(dev(k), dev(sl), dev(pos), gcache, "k")
        inv.kv_quant_int16(dev(v), dev(sl), dev(pos), gcache, "v")
    q = synth.normal((B, Hq, D), seed=seed + 3)
    return q, ocache, gcache


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 4), (4, 4)])
def test_attention_parity_edges(inv, Hq, Hkv):
    # split edges (255, 256, 257) and the decode kernel's 32-key staging halves: a
    # warp's last keys in its first half only (31, 32, 96, 160, 224, 288 = 256 + 32)
    # or one key into its second half (33, 97)
    lens = np.array([1, 2, 31, 32, 33, 63, 64, 96, 97, 160, 224, 255, 256, 257, 288, 700], np.int32)
    B = len(lens)
    q, oc, gc = _attn_case(inv, B, Hq, Hkv, lens, seed=30, max_len=768)
    sigma = np.float32(1 / np.sqrt(128))
    slot = np.arange(B, dtype=np.int32)
    out, hi, lo = inv.attn_decode_fixedsplit(dev(q), gc, dev(slot), dev(lens), float(sigma), want_split=True)
    assert status() == inv.INV_OK
    # the cache the GPU wrote is the oracle's, bit for bit
    assert np.array_equal(host(gc.k)[:, :, :700], oc.k[:, :, :700])
    want = ref.attention_decode(q, oc, slot, lens, sigma)
    err = rowwise_err(host(out).reshape(B * Hq, 128), want.reshape(B * Hq, 128))
    assert err.max() <= TOL, err.max()
    # the combine's fused split is the oracle's binary16 encoding of its fp32 output, bit for bit
    h_want, l_want, _ = enc.heal_split(host(out).reshape(B * Hq, 128))
    assert np.array_equal(bits16(hi).reshape(B * Hq, 128), h_want)
    assert np.array_equal(bits16(lo).reshape(B * Hq, 128), l_want)


def test_attention_config3_parity_and_composition(inv):
    """GQA 32/8, ragged lengths U(128, 8192), split 256."""
    B, Hq, Hkv = 12, 32, 8
    lens = synth.ragged_lengths(B, seed=40)
    q, oc, gc = _attn_case(inv, B, Hq, Hkv, lens, seed=41, max_len=8192)
    sigma = float(np.float32(1 / np.sqrt(128)))
    slot = np.arange(B, dtype=np.int32)
    out = inv.attn_decode_fixedsplit(dev(q), gc, dev(slot), dev(lens), sigma)
    want = ref.attention_decode(q, oc, slot, lens, sigma)
    err = rowwise_err(host(out).reshape(B * Hq, 128), want.reshape(B * Hq, 128))
    assert err.max() <= TOL, err.max()
    # batch composition: each row alone, and the rows reversed
    for b in (0, 5, 11):
        one = inv.attn_decode_fixedsplit(dev(q[b:b + 1].copy()), gc, dev(slot[b:b + 1].copy()),
                                         dev(lens[b:b + 1].copy()), sigma)
        assert torch.equal(one[0].view(torch.int32), out[b].view(torch.int32))
    r = np.arange(B)[::-1].copy()
    rev = inv.attn_decode_fixedsplit(dev(q[r].copy()), gc, dev(slot[r].copy()), dev(lens[r].copy()), sigma)
    assert torch.equal(rev.view(torch.int32), out[torch.from_numpy(r).cuda()].view(torch.int32))
    assert status() == inv.INV_OK


def test_attention_bad_length_reports(inv):
    gc = inv.KVCache(n_slots=1, n_kv_heads=8, max_len=256)
    q = torch.zeros((1, 32, 128), device="cuda")
    inv.attn_decode_fixedsplit(q, gc, dev(np.array([0], np.int32)), dev(np.array([300], np.int32)), 0.1)
    assert status() == inv.INV_ERR_INVALID_ARG


# ------------------------------------------------------------ failure path ---

def test_bounded_wait_times_out_and_context_survives(inv):
    inv.inv_selftest_wait_timeout(2_000_000)  # 2 ms
    assert status() == inv.INV_ERR_TIMEOUT
    x = synth.normal((4, 64), seed=1)
    hi, lo = inv.heal_split(dev(x))
    assert np.array_equal(bits16(hi), enc.heal_split(x)[0])
    assert status() == inv.INV_OK


def test_gemm_consumer_wait_times_out_and_context_survives(inv):
    """The down GEMM of a layer waits on the gate/up GEMM's tile counters; with
    a counter that nothing completes, the wait must give up, record
    INV_ERR_TIMEOUT and let the kernel exit with the context usable."""
    inv.inv_selftest_gemm_wait_timeout(2_000_000)  # 2 ms
    assert status() == inv.INV_ERR_TIMEOUT
    x = synth.normal((4, 64), seed=2)
    hi, lo = inv.heal_split(dev(x))
    assert np.array_equal(bits16(hi), enc.heal_split(x)[0])
    assert status() == inv.INV_OK
