"""The full decode layer on the GPU: parity with the oracle layer, bit-identity
across batch size / composition, and chunked versus one-shot prefill."""
import numpy as np
import pytest
import torch

from invariant_numerics_b200 import synth
from oracle import reference as ref

from gpu_helpers import TOL, dev, host, rowwise_err, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


def make_layer(inv, H, Hq, Hkv, F, max_pos, seed=0):
    D = 128
    s = lambda i, shape: synth.normal(shape, seed=seed, stream=i, std=0.02)
    p = ref.LayerParams(wq=s(1, (H, Hq * D)), wk=s(2, (H, Hkv * D)), wv=s(3, (H, Hkv * D)), wo=s(4, (Hq * D, H)),
                        w_gate=s(5, (H, F)), w_up=s(6, (H, F)), w_down=s(7, (F, H)),
                        g_attn=synth.uniform(H, seed=seed, stream=8, lo=0.5, hi=1.5),
                        g_mlp=synth.uniform(H, seed=seed, stream=9, lo=0.5, hi=1.5),
                        n_heads=Hq, n_kv_heads=Hkv, head_dim=D)
    cfg = inv.LayerConfig(hidden=H, n_heads=Hq, n_kv_heads=Hkv, ffn=F, max_pos=max_pos)
    w = inv.LayerWeights(cfg, dev(p.wq), dev(p.wk), dev(p.wv), dev(p.wo), dev(p.w_gate), dev(p.w_up),
                         dev(p.w_down), dev(p.g_attn), dev(p.g_mlp))
    return p, cfg, w


SMALL = dict(H=256, Hq=8, Hkv=2, F=512, max_pos=1024)


def test_layer_parity_small(inv):
    p, cfg, w = make_layer(inv, **SMALL)
    n_slots, max_len = 3, 512
    oc = ref.KVCache.empty(n_slots, 2, max_len, 128)
    gc = inv.KVCache(n_slots=n_slots, n_kv_heads=2, max_len=max_len)
    # prefill three sequences of different lengths in chunks, then decode
    steps = [
        (np.zeros(300, np.int32), np.arange(300, dtype=np.int32)),
        (np.ones(37, np.int32), np.arange(37, dtype=np.int32)),
        (np.full(5, 2, np.int32), np.arange(5, dtype=np.int32)),
        (np.array([0, 1, 2], np.int32), np.array([300, 37, 5], np.int32)),
        (np.array([2, 0], np.int32), np.array([6, 301], np.int32)),
    ]
    for i, (slot, pos) in enumerate(steps):
        x = synth.normal((len(slot), SMALL["H"]), seed=100 + i)
        y = inv.decode_layer(cfg, w, gc, dev(x), dev(slot), dev(pos))
        want = ref.decode_layer(p, oc, x, slot, pos)
        err = rowwise_err(host(y), want)
        assert err.max() <= TOL, (i, err.max())
    assert status() == inv.INV_OK


def test_layer_batch_invariance_and_composition(inv):
    """Every row's bits are the same for batch sizes 1..256 (one and two GEMM
    row tiles, ragged last tiles) and any shuffled batch composition."""
    p, cfg, w = make_layer(inv, **SMALL, seed=1)
    n_seq, ctx = 256, 200
    gc = inv.KVCache(n_slots=n_seq, n_kv_heads=2, max_len=256)
    # fill every slot with a 200-token context
    for b in range(0, n_seq, 16):
        slots = np.repeat(np.arange(b, b + 16, dtype=np.int32), ctx)
        pos = np.tile(np.arange(ctx, dtype=np.int32), 16)
        x = synth.normal((len(slots), SMALL["H"]), seed=7, stream=b)
        inv.decode_layer(cfg, w, gc, dev(x), dev(slots), dev(pos))
    x = synth.normal((n_seq, SMALL["H"]), seed=8)
    pos = np.full(n_seq, ctx, np.int32)
    ref_out = None
    for B in (256, 200, 128, 37, 8, 1):
        perm = synth.permutation(n_seq, seed=B)
        outs = np.zeros((n_seq, SMALL["H"]), np.float32)
        for a in range(0, n_seq, B):
            idx = perm[a:a + B]
            y = inv.decode_layer(cfg, w, gc, dev(x[idx]), dev(idx.astype(np.int32)), dev(pos[idx]))
            outs[idx] = host(y)
        if ref_out is None:
            ref_out = outs
        else:
            assert np.array_equal(outs.view(np.int32), ref_out.view(np.int32)), B
    assert status() == inv.INV_OK


def test_chunked_prefill_matches_one_shot(inv):
    p, cfg, w = make_layer(inv, **SMALL, seed=2)
    T = 600
    x = synth.normal((T, SMALL["H"]), seed=9)
    pos = np.arange(T, dtype=np.int32)
    a = inv.KVCache(n_slots=1, n_kv_heads=2, max_len=1024)
    b = inv.KVCache(n_slots=1, n_kv_heads=2, max_len=1024)
    one = inv.decode_layer(cfg, w, a, dev(x), dev(np.zeros(T, np.int32)), dev(pos))
    parts = []
    for lo, hi in ((0, 256), (256, 257), (257, 512), (512, 600)):
        parts.append(inv.decode_layer(cfg, w, b, dev(x[lo:hi].copy()), dev(np.zeros(hi - lo, np.int32)),
                                      dev(pos[lo:hi].copy())))
    chunked = torch.cat(parts)
    assert torch.equal(one.view(torch.int32), chunked.view(torch.int32))
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert torch.equal(a.k_scale, b.k_scale) and torch.equal(a.v_scale, b.v_scale)


def test_prefill_layer_bit_identical_to_decode_layer(inv):
    """The prefill form (splits loaded once per chunk) gives the decode form's
    bits for every row and writes the same cache, for chunks that start and
    end inside splits and row blocks."""
    p, cfg, w = make_layer(inv, **SMALL, seed=3)
    T0, T1, T2 = 300, 77, 430    # chunk boundaries off the 256-key and 64-row grids
    xs = synth.normal((T0 + T1 + T2, SMALL["H"]), seed=11)
    a = inv.KVCache(n_slots=2, n_kv_heads=2, max_len=1024)
    b = inv.KVCache(n_slots=2, n_kv_heads=2, max_len=1024)
    start = 0
    for T in (T0, T1, T2):
        x = dev(xs[start:start + T].copy())
        pos = np.arange(start, start + T, dtype=np.int32)
        y_dec = inv.decode_layer(cfg, w, a, x, dev(np.ones(T, np.int32)), dev(pos))
        y_pre = inv.prefill_layer(cfg, w, b, x, 1, start)
        assert torch.equal(y_dec.view(torch.int32), y_pre.view(torch.int32)), start
        start += T
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert torch.equal(a.k_scale, b.k_scale) and torch.equal(a.v_scale, b.v_scale)
    assert status() == inv.INV_OK


def test_layer_rows_with_bad_slot_or_position_are_reported_and_skipped(inv):
    """A row whose slot or position is out of range (checked where the QKV
    GEMM's epilogue writes the cache) records INV_ERR_INVALID_ARG and writes
    nothing; the other rows of the batch get the bits they get without it."""
    p, cfg, w = make_layer(inv, **SMALL)
    H = SMALL["H"]
    caches = [inv.KVCache(n_slots=3, n_kv_heads=2, max_len=512) for _ in range(2)]
    x0 = dev(synth.normal((20, H), seed=300))
    for gc in caches:
        inv.decode_layer(cfg, w, gc, x0, dev(np.zeros(20, np.int32)), dev(np.arange(20, dtype=np.int32)))
    assert status() == inv.INV_OK
    x = synth.normal((5, H), seed=301)
    slot = np.array([0, 1, 7, 2, 1], np.int32)    # row 2: slot out of range
    pos = np.array([20, 0, 0, 0, 600], np.int32)  # row 4: position past the cache
    y_bad = inv.decode_layer(cfg, w, caches[0], dev(x), dev(slot), dev(pos))
    assert status() == inv.INV_ERR_INVALID_ARG
    keep = [0, 1, 3]
    y_good = inv.decode_layer(cfg, w, caches[1], dev(x[keep]), dev(slot[keep]), dev(pos[keep]))
    assert status() == inv.INV_OK
    assert torch.equal(y_bad[keep].view(torch.int32), y_good.view(torch.int32))
    for name in ("k", "v", "k_scale", "v_scale"):
        a, b = getattr(caches[0], name), getattr(caches[1], name)
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4)])
def test_layer_parity_other_group_sizes(inv, Hq, Hkv):
    """G = Hq / Hkv = 1 and 2 through the whole layer (the QKV kernel's head
    tiles map to q, k and v heads by these counts), prefill chunk then decode,
    against the oracle."""
    H, F = 256, 512
    p, cfg, w = make_layer(inv, H, Hq, Hkv, F, max_pos=1024, seed=7)
    oc = ref.KVCache.empty(2, Hkv, 512, 128)
    gc = inv.KVCache(n_slots=2, n_kv_heads=Hkv, max_len=512)
    steps = [
        (np.zeros(261, np.int32), np.arange(261, dtype=np.int32)),
        (np.array([0, 1], np.int32), np.array([261, 0], np.int32)),
        (np.array([1, 0], np.int32), np.array([1, 262], np.int32)),
    ]
    for i, (slot, pos) in enumerate(steps):
        x = synth.normal((len(slot), H), seed=200 + i)
        if i == 0:  # the prompt chunk through prefill_layer (its own attention kernel)
            y = inv.prefill_layer(cfg, w, gc, dev(x), 0, 0)
        else:
            y = inv.decode_layer(cfg, w, gc, dev(x), dev(slot), dev(pos))
        want = ref.decode_layer(p, oc, x, slot, pos)
        err = rowwise_err(host(y), want)
        assert err.max() <= TOL, (i, err.max())
    assert status() == inv.INV_OK
