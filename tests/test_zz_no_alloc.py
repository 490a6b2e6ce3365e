"""attn_decode_fixedsplit_noalloc -- the attention entry point for callers that
cannot allocate device memory (an embedding application that owns the whole
device-memory budget, a plug-in without an allocator, a latency-critical path
where an allocation may synchronise the device).  It keeps the split partials
in the library's own fixed device array instead of a caller workspace.

Checked through the C ABI against the workspace entry point on the same
inputs, on two calls in a row (the second call reuses the array the first one
left behind), and for the size limit.  This file is collected last so that a
run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

from invariant_numerics_b200 import synth

from gpu_helpers import TOL, dev, host, rowwise_err, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum
    assert invnum.inv_get_device_status() == invnum.INV_OK
    return invnum


def _case(inv, B, Hq, Hkv, lens, seed, max_len):
    cache = inv.KVCache(n_slots=B, n_kv_heads=Hkv, max_len=max_len)
    c = synth.channel_scale(Hkv, 128, seed=seed)
    for b in range(B):
        L = int(lens[b])
        pos = dev(np.arange(L, dtype=np.int32))
        sl = dev(np.full(L, b, np.int32))
        inv.kv_quant_int16(dev(synth.kv_tensor(L, Hkv, 128, seed=seed + 1, stream=b, scale=c)), sl, pos, cache, "k")
        inv.kv_quant_int16(dev(synth.kv_tensor(L, Hkv, 128, seed=seed + 2, stream=b, scale=c)), sl, pos, cache, "v")
    q = synth.normal((B, Hq, 128), seed=seed + 3)
    return dev(q), cache


def test_noalloc_matches_workspace_entry_point_twice(inv):
    B, Hq, Hkv = 12, 32, 8
    lens = synth.ragged_lengths(B, seed=50, lo=1, hi=3000)
    q, cache = _case(inv, B, Hq, Hkv, lens, seed=51, max_len=3072)
    slot, ld = dev(np.arange(B, dtype=np.int32)), dev(lens)
    sigma = float(np.float32(1 / np.sqrt(128)))
    want, want_hi, _ = inv.attn_decode_fixedsplit(q, cache, slot, ld, sigma, want_split=True)
    first, first_hi, _ = inv.attn_decode_fixedsplit_noalloc(q, cache, slot, ld, sigma, want_split=True)
    # a second, different call in between leaves other partials in the shared array
    q2 = q.flip(0).contiguous()
    inv.attn_decode_fixedsplit_noalloc(q2, cache, slot.flip(0).contiguous(), ld.flip(0).contiguous(), sigma)
    second, second_hi, _ = inv.attn_decode_fixedsplit_noalloc(q, cache, slot, ld, sigma, want_split=True)
    assert status() == inv.INV_OK
    w = host(want).reshape(B * Hq, 128).astype(np.float64)
    for got, got_hi in ((first, first_hi), (second, second_hi)):
        assert rowwise_err(host(got).reshape(B * Hq, 128), w).max() <= TOL
        # the same kernels run on the same inputs: the results are the same bits
        assert torch.equal(got.view(torch.int32), want.view(torch.int32))
        assert torch.equal(got_hi.view(torch.int16), want_hi.view(torch.int16))


def test_noalloc_rejects_sizes_beyond_its_array(inv):
    Hkv, max_len = 8, 8192
    cache = inv.KVCache(n_slots=1, n_kv_heads=Hkv, max_len=max_len)
    B, Hq = 80, 32   # 80 x 32 x 32 splits x 520 B > 34 MiB
    need = inv.attn_decode_workspace_size(B, Hq, max_len)
    assert need > inv.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, 128), device="cuda")
    ones = dev(np.ones(B, np.int32))
    with pytest.raises(inv.InvError) as ei:
        inv.attn_decode_fixedsplit_noalloc(q, cache, dev(np.zeros(B, np.int32)), ones, 0.1)
    assert ei.value.code == inv.INV_ERR_WORKSPACE
    # a bound <= 0 resolves to the cache's max_len, which does not fit either
    with pytest.raises(inv.InvError) as ei:
        inv.attn_decode_fixedsplit_noalloc(q, cache, dev(np.zeros(B, np.int32)), ones, 0.1, max_len_bound=0)
    assert ei.value.code == inv.INV_ERR_WORKSPACE
    # the same call with a smaller length bound fits and runs
    out = inv.attn_decode_fixedsplit_noalloc(q, cache, dev(np.zeros(B, np.int32)), ones, 0.1, max_len_bound=256)
    assert status() == inv.INV_OK
    assert torch.isfinite(out).all()
