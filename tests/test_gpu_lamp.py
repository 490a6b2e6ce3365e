"""LAMP selective recompute of the attention scores (attn_decode_lamp) on the
GPU, through the C ABI, against the CPU oracle.

* The low-precision scores are a sequential binary16 accumulation that the
  oracle reproduces exactly: with no score recomputed (tau = +inf) the output
  equals the oracle's all-low-precision attention within 1e-5 (normwise).
* The recompute decision is taken in fp32 on both sides; the two decisions
  must agree on every key whose criterion is not within a relative 1e-5 of
  tau (CUDA expf and the oracle's exp may differ by an ulp there), and the
  GPU's output equals the oracle's output for the GPU's own decisions.
* tau < 0 (every score recomputed) gives the plain attention's bits; rows are
  bit-identical alone and in a batch; the recompute reduces the error of the
  low-precision softmax far more than as many random recomputes would.
"""
import numpy as np
import pytest
import torch

from invariant_numerics_b200 import synth
from oracle import encodings as enc
from oracle import reference as ref

from gpu_helpers import TOL, dev, host, rowwise_err, status

pytestmark = pytest.mark.gpu

SIGMA = float(np.float32(1 / np.sqrt(128)))


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


def _case(inv, lens, Hq=32, Hkv=8, seed=70, max_len=3072, qscale=3.0):
    B = len(lens)
    c = synth.channel_scale(Hkv, 128, seed=seed)
    oc = ref.KVCache.empty(B, Hkv, max_len, 128)
    gc = inv.KVCache(n_slots=B, n_kv_heads=Hkv, max_len=max_len)
    for b in range(B):
        L = int(lens[b])
        pos = np.arange(L, dtype=np.int32)
        sl = np.full(L, b, np.int32)
        for which, st in (("k", 1), ("v", 2)):
            x = synth.kv_tensor(L, Hkv, 128, seed=seed + st, stream=b, scale=c)
            oc.write(which, x, sl, pos)
            inv.kv_quant_int16(dev(x), dev(sl), dev(pos), gc, which)
    q = synth.normal((B, Hq, 128), seed=seed + 3, std=qscale)
    return q, oc, gc


def _oracle_criterion(q, oc, lens, Hq, Hkv):
    """fp32 criterion values of every (row, head, key), from the oracle's
    low-precision scores."""
    G = Hq // Hkv
    q16 = enc.rn16_bits(q.astype(np.float64))
    out = []
    for b, L in enumerate(lens):
        rows = []
        for h in range(Hq):
            y = ref.lamp_low_precision_scores(q16[b, h], oc.k[b, h // G, :L], oc.ks[b, h // G, :L], SIGMA)
            rows.append(ref.lamp_criterion_f32(y))
        out.append(np.stack(rows))
    return out


LENS = np.array([1, 255, 256, 257, 700, 3000], np.int32)


@pytest.mark.parametrize("tau", [1e-2, 1.0])
def test_lamp_decisions_and_output_match_the_oracle(inv, tau):
    Hq, Hkv = 32, 8
    q, oc, gc = _case(inv, LENS)
    slot = np.arange(len(LENS), dtype=np.int32)
    out, rec = inv.attn_decode_lamp(dev(q), gc, dev(slot), dev(LENS), SIGMA, tau, want_recompute=True)
    assert status() == inv.INV_OK
    rec = host(rec)
    crit = _oracle_criterion(q, oc, LENS, Hq, Hkv)
    gpu_sel = []
    for b, L in enumerate(LENS):
        g = rec[b, :, :L].astype(bool)
        o = crit[b] > np.float32(tau)
        far = np.abs(crit[b].astype(np.float64) - tau) > 1e-5 * tau
        assert np.array_equal(g[far], o[far]), (b, int((g[far] != o[far]).sum()))
        gpu_sel.append(g)
    n = sum(int(s.sum()) for s in gpu_sel)
    assert 0 < n < sum(s.size for s in gpu_sel)
    want = ref.attention_decode_lamp(q, oc, slot, LENS, SIGMA, tau, select=gpu_sel)
    err = rowwise_err(host(out).reshape(-1, 128), want.reshape(-1, 128))
    assert err.max() <= TOL, err.max()


def test_lamp_low_precision_scores_match_the_oracle(inv):
    """tau = +inf: only non-finite scores would be recomputed, so the output is
    the softmax of the binary16-accumulated scores themselves."""
    Hq, Hkv = 32, 8
    q, oc, gc = _case(inv, LENS, seed=80)
    slot = np.arange(len(LENS), dtype=np.int32)
    out, rec = inv.attn_decode_lamp(dev(q), gc, dev(slot), dev(LENS), SIGMA, float("inf"), want_recompute=True)
    assert status() == inv.INV_OK
    sel = [host(rec)[b, :, :L].astype(bool) for b, L in enumerate(LENS)]
    assert sum(int(s.sum()) for s in sel) == 0
    want = ref.attention_decode_lamp(q, oc, slot, LENS, SIGMA, 0.0, select=sel)
    full = ref.attention_decode(q, oc, slot, LENS, SIGMA)
    err = rowwise_err(host(out).reshape(-1, 128), want.reshape(-1, 128))
    assert err.max() <= TOL, err.max()
    # and the low-precision softmax is visibly off the plain one
    assert rowwise_err(want.reshape(-1, 128), full.reshape(-1, 128)).max() > 100 * TOL


def test_lamp_recompute_all_is_the_plain_attention_and_batch_invariant(inv):
    q, oc, gc = _case(inv, LENS, seed=90)
    qd = dev(q)
    slot = dev(np.arange(len(LENS), dtype=np.int32))
    ld = dev(LENS)
    plain = inv.attn_decode_fixedsplit(qd, gc, slot, ld, SIGMA)
    every = inv.attn_decode_lamp(qd, gc, slot, ld, SIGMA, -1.0)
    assert torch.equal(every.view(torch.int32), plain.view(torch.int32))
    lamp = inv.attn_decode_lamp(qd, gc, slot, ld, SIGMA, 0.1)
    for b in (0, 3, 5):
        one = inv.attn_decode_lamp(qd[b:b + 1].contiguous(), gc, slot[b:b + 1].contiguous(), ld[b:b + 1].contiguous(),
                                   SIGMA, 0.1)
        assert torch.equal(one[0].view(torch.int32), lamp[b].view(torch.int32))
    r = torch.arange(len(LENS) - 1, -1, -1, device="cuda")
    rev = inv.attn_decode_lamp(qd[r].contiguous(), gc, slot[r].contiguous(), ld[r].contiguous(), SIGMA, 0.1)
    assert torch.equal(rev.view(torch.int32), lamp[r].view(torch.int32))
    assert status() == inv.INV_OK


def test_lamp_reduces_the_low_precision_error(inv):
    """The recompute the criterion selects brings the binary16-accumulated
    attention close to the plain one; as many randomly chosen recomputes
    (evaluated by the oracle) do much less."""
    lens = np.array([700, 1500, 3000, 2048], np.int32)
    q, oc, gc = _case(inv, lens, seed=100)
    slot = np.arange(len(lens), dtype=np.int32)
    full = ref.attention_decode(q, oc, slot, lens, SIGMA)
    none = inv.attn_decode_lamp(dev(q), gc, dev(slot), dev(lens), SIGMA, float("inf"))
    lamp, rec = inv.attn_decode_lamp(dev(q), gc, dev(slot), dev(lens), SIGMA, 0.01, want_recompute=True)
    e = lambda o: float(rowwise_err(np.asarray(o).reshape(-1, 128), full.reshape(-1, 128)).mean())
    sel = [host(rec)[b, :, :L].astype(bool) for b, L in enumerate(lens)]
    g = np.random.Generator(np.random.PCG64(7))
    rnd = []
    for s in sel:
        m = np.zeros(s.size, bool)
        m[g.choice(s.size, int(s.sum()), replace=False)] = True
        rnd.append(m.reshape(s.shape))
    e_rand = e(ref.attention_decode_lamp(q, oc, slot, lens, SIGMA, 0.0, select=rnd))
    rate = sum(int(s.sum()) for s in sel) / sum(s.size for s in sel)
    assert rate < 0.1
    assert e(host(lamp)) < 0.05 * e(host(none)) and e(host(lamp)) < 0.1 * e_rand
    assert status() == inv.INV_OK
