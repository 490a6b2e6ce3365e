"""Canary bands: every buffer a C-ABI call writes (outputs, workspaces, the KV
cache) is placed between two 4 KB bands of a known byte pattern, and after
the call both bands must be unchanged.  A kernel that writes past either end
of its buffer -- the overflow a sanitizer would report -- changes a band.
Each call also has to give the same bits as the same call on plainly
allocated buffers.  Shapes are ragged (odd row counts, lengths that end
inside a split and a 64-key box) so that tail handling is exercised."""
import ctypes as C

import numpy as np
import pytest
import torch

from invariant_numerics_b200 import synth

from gpu_helpers import dev, status

pytestmark = pytest.mark.gpu

BAND = 4096
PATTERN = 0xA5


class Banded:
    """A tensor of `shape` and `dtype` inside [band | data | band] bytes."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((BAND + n + BAND,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[BAND:BAND + n].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.raw[:BAND] == PATTERN).all()) and bool((self.raw[-BAND:] == PATTERN).all())


def same_bits(a, b) -> bool:
    a, b = a.contiguous(), b.contiguous()
    return torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


def banded_cache(inv, n_slots, n_kv_heads, max_len):
    c = inv.KVCache(n_slots=n_slots, n_kv_heads=n_kv_heads, max_len=max_len)
    bands = {}
    for name in ("k", "v", "k_scale", "v_scale"):
        t = getattr(c, name)
        bands[name] = Banded(tuple(t.shape), t.dtype, fill=t)
        setattr(c, name, bands[name].t)
    return c, bands


def test_heal_split_pack_and_gemm_stay_inside_their_buffers(inv):
    x = dev(synth.normal_with_outliers((37, 4096), seed=1))
    hi, lo = Banded((37, 4096), torch.float16), Banded((37, 4096), torch.float16)
    inv.heal_split(x, hi=hi.t, lo=lo.t)
    ref_hi, ref_lo = inv.heal_split(x)
    assert hi.intact() and lo.intact()
    assert same_bits(hi.t, ref_hi) and same_bits(lo.t, ref_lo)

    K, N = 4096, 384
    W = dev(synth.normal((K, N), seed=2, std=0.02))
    nbytes = inv.lib.heal_packed_weight_bytes(K, N)
    packed = Banded((N // 128, 2, 128, K), torch.float16)
    col_exp = Banded((N,), torch.int8)
    assert nbytes == packed.t.numel() * 2
    rc = inv.lib.heal_pack_weight(inv._ptr(W), K, N, inv._ptr(packed.t), nbytes, inv._ptr(col_exp.t), inv._stream())
    assert rc == inv.INV_OK
    P, e = inv.heal_pack_weight(W)
    assert packed.intact() and col_exp.intact()
    assert same_bits(packed.t, P) and same_bits(col_exp.t, e)

    for M in (1, 17, 37):
        y = Banded((M, N), torch.float32)
        res = dev(synth.normal((M, N), seed=3))
        inv.comp_gemm(hi.t[:M], lo.t[:M], packed.t, col_exp.t, out=y.t)
        assert y.intact()
        assert same_bits(y.t, inv.comp_gemm(hi.t[:M].contiguous(), lo.t[:M].contiguous(), P, e))
        yr = Banded((M, N), torch.float32)
        inv.comp_gemm(hi.t[:M], lo.t[:M], packed.t, col_exp.t, residual=res, out=yr.t)
        assert yr.intact()
        assert same_bits(yr.t, inv.comp_gemm(hi.t[:M].contiguous(), lo.t[:M].contiguous(), P, e, residual=res))
    assert status() == inv.INV_OK


def test_rmsnorm_rope_embed_argmax_stay_inside_their_buffers(inv):
    rows, H = 19, 4096
    x = dev(synth.normal((rows, H), seed=4))
    g = dev(synth.uniform(H, seed=5, lo=0.5, hi=1.5))
    y, yh, yl = Banded((rows, H), torch.float32), Banded((rows, H), torch.float16), Banded((rows, H), torch.float16)
    rc = inv.lib.rmsnorm_bi(inv._ptr(x), inv._ptr(g), rows, H, C.c_float(1e-5), inv._ptr(y.t), inv._ptr(yh.t),
                            inv._ptr(yl.t), inv._stream())
    assert rc == inv.INV_OK
    ry, rh, rl = inv.rmsnorm_bi(x, g, 1e-5, want_split=True)
    assert y.intact() and yh.intact() and yl.intact()
    assert same_bits(y.t, ry) and same_bits(yh.t, rh) and same_bits(yl.t, rl)

    cs, sn = Banded((333, 64), torch.float32), Banded((333, 64), torch.float32)
    rc = inv.lib.rope_tables(333, 10000.0, inv._ptr(cs.t), inv._ptr(sn.t), inv._stream())
    assert rc == inv.INV_OK
    rcs, rsn = inv.rope_tables(333)
    assert cs.intact() and sn.intact() and same_bits(cs.t, rcs) and same_bits(sn.t, rsn)

    table = dev(synth.normal((1000, 96), seed=6))
    ids = dev(np.array([0, 999, 5, 17, 999, 3, 1], np.int32))
    out = Banded((7, 96), torch.float32)
    inv.embed_gather(table, ids, out=out.t)
    assert out.intact() and same_bits(out.t, inv.embed_gather(table, ids))

    logits = dev(synth.normal((5, 32000), seed=7))
    am = Banded((5,), torch.int32)
    inv.argmax_rows(logits, out=am.t)
    assert am.intact() and same_bits(am.t, inv.argmax_rows(logits))
    assert status() == inv.INV_OK


def _fill(inv, cache, lens, Hkv, seed):
    for b, L in enumerate(lens):
        sl = torch.full((int(L),), b, dtype=torch.int32, device="cuda")
        ps = torch.arange(int(L), dtype=torch.int32, device="cuda")
        for i, which in enumerate(("k", "v")):
            inv.kv_quant_int16(dev(synth.normal((int(L), Hkv, 128), seed=seed + i, stream=b)), sl, ps, cache, which)


def test_kv_quant_and_decode_attention_stay_inside_their_buffers(inv):
    Hq, Hkv, max_len = 32, 8, 1280
    lens = np.array([1, 255, 257, 700, 1280, 64, 129], np.int32)
    B = len(lens)
    cache, cbands = banded_cache(inv, B, Hkv, max_len)
    plain = inv.KVCache(n_slots=B, n_kv_heads=Hkv, max_len=max_len)
    _fill(inv, cache, lens, Hkv, seed=20)
    _fill(inv, plain, lens, Hkv, seed=20)
    assert all(b.intact() for b in cbands.values())
    for name in ("k", "v", "k_scale", "v_scale"):
        assert same_bits(getattr(cache, name), getattr(plain, name))

    q = dev(synth.normal((B, Hq, 128), seed=21))
    slot = dev(np.arange(B, dtype=np.int32))
    sigma = float(np.float32(1 / np.sqrt(128)))
    for bound in (max_len, 760):
        lens_b = np.minimum(lens, bound)
        ld_b = dev(lens_b)
        nbytes = inv.attn_decode_workspace_size(B, Hq, bound)
        ws = Banded((nbytes,), torch.uint8)
        out, hi, lo = Banded((B, Hq, 128), torch.float32), Banded((B, Hq, 128), torch.float16), \
            Banded((B, Hq, 128), torch.float16)
        cs = cache.struct()
        rc = inv.lib.attn_decode_fixedsplit(inv._ptr(q), B, Hq, C.byref(cs), inv._ptr(slot), inv._ptr(ld_b), bound,
                                            inv.KV_SPLIT, C.c_float(sigma), inv._ptr(out.t), inv._ptr(hi.t),
                                            inv._ptr(lo.t), inv._ptr(ws.t), nbytes, inv._stream())
        assert rc == inv.INV_OK
        ro, rh, rl = inv.attn_decode_fixedsplit(q, plain, slot, ld_b, sigma, max_len_bound=bound, want_split=True)
        assert ws.intact() and out.intact() and hi.intact() and lo.intact()
        assert same_bits(out.t, ro) and same_bits(hi.t, rh) and same_bits(lo.t, rl)

        L = bound
        rec = Banded((B, Hq, L), torch.uint8)
        outl = Banded((B, Hq, 128), torch.float32)
        ws2 = Banded((nbytes,), torch.uint8)
        rc = inv.lib.attn_decode_lamp(inv._ptr(q), B, Hq, C.byref(cs), inv._ptr(slot), inv._ptr(ld_b), bound,
                                      inv.KV_SPLIT, C.c_float(sigma), C.c_float(0.1), inv._ptr(outl.t), None, None,
                                      inv._ptr(rec.t), L, inv._ptr(ws2.t), nbytes, inv._stream())
        assert rc == inv.INV_OK
        rol, rrec = inv.attn_decode_lamp(q, plain, slot, ld_b, sigma, 0.1, max_len_bound=bound, want_recompute=True)
        assert rec.intact() and outl.intact() and ws2.intact()
        assert same_bits(outl.t, rol)
        for b in range(B):  # flags past a row's length are not written
            n = int(lens_b[b])
            assert same_bits(rec.t[b, :, :n], rrec[b, :, :n])

        outn = Banded((B, Hq, 128), torch.float32)
        inv.attn_decode_fixedsplit_noalloc(q, cache, slot, ld_b, sigma, max_len_bound=bound, out=outn.t)
        assert outn.intact() and same_bits(outn.t, ro)
    assert all(b.intact() for b in cbands.values())
    assert status() == inv.INV_OK


def test_decode_and_prefill_layer_stay_inside_their_buffers(inv):
    from test_gpu_layer import make_layer
    H, Hq, Hkv, F = 256, 8, 2, 512
    p, cfg, w = make_layer(inv, H=H, Hq=Hq, Hkv=Hkv, F=F, max_pos=1024)
    n_slots, max_len = 3, 576
    cache, cbands = banded_cache(inv, n_slots, Hkv, max_len)
    plain = inv.KVCache(n_slots=n_slots, n_kv_heads=Hkv, max_len=max_len)

    # prefill 300 tokens of slot 0 in chunks of 173 and 127
    for a, T in ((0, 173), (173, 127)):
        x = dev(synth.normal((T, H), seed=30 + a))
        nbytes = inv.lib.prefill_layer_workspace_size(C.byref(cfg.struct()), T, max_len)
        ws = Banded((nbytes,), torch.uint8)
        out = Banded((T, H), torch.float32)
        inv.prefill_layer(cfg, w, cache, x, 0, a, out=out.t, workspace=ws.t)
        ref = inv.prefill_layer(cfg, w, plain, x, 0, a)
        assert ws.intact() and out.intact() and same_bits(out.t, ref)
    # decode rows of all three slots (slots 1 and 2 start empty)
    for i, (slot, pos) in enumerate(((np.array([0, 1, 2], np.int32), np.array([300, 0, 0], np.int32)),
                                     (np.array([2, 0], np.int32), np.array([1, 301], np.int32)))):
        B = len(slot)
        x = dev(synth.normal((B, H), seed=40 + i))
        nbytes = inv.decode_layer_workspace_size(cfg, B, max_len)
        ws = Banded((nbytes,), torch.uint8)
        out = Banded((B, H), torch.float32)
        inv.decode_layer(cfg, w, cache, x, dev(slot), dev(pos), out=out.t, workspace=ws.t)
        ref = inv.decode_layer(cfg, w, plain, x, dev(slot), dev(pos))
        assert ws.intact() and out.intact() and same_bits(out.t, ref)
    assert all(b.intact() for b in cbands.values())
    for name in ("k", "v", "k_scale", "v_scale"):
        assert same_bits(getattr(cache, name), getattr(plain, name))
    assert status() == inv.INV_OK
