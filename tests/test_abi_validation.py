"""Host-side argument validation of the C ABI (CPU only).

Every call below must return its status before touching the GPU: the shape,
range, alignment and workspace checks run first, and an empty call (zero
rows) is a no-op.  Pointers are dummy, 16-byte-aligned addresses that the
library never dereferences on these paths.
"""
import ctypes as C

import pytest

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
PTR = C.c_void_p(0x100000)          # aligned dummy device address
PTR2 = C.c_void_p(0x200000)
MISALIGNED = C.c_void_p(0x100004)


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum  # loads the library and declares the argument types
    return invnum


@pytest.fixture(scope="module")
def L(inv):
    return inv.lib


def cache(inv, head_dim=128, max_len=256, n_slots=2, hkv=8):
    return inv.KVCacheStruct(PTR.value, PTR2.value, PTR.value, PTR2.value, n_slots, hkv, max_len, head_dim)


def test_comp_gemm_validation(L):
    g = L.comp_gemm
    assert g(PTR, PTR, 0, 512, 512, PTR, PTR, 512, PTR, 512, None, 0, None) == OK          # M = 0: no-op
    assert g(PTR, PTR, -1, 512, 512, PTR, PTR, 512, PTR, 512, None, 0, None) == INVALID
    assert g(PTR, PTR, 4, 100, 104, PTR, PTR, 512, PTR, 512, None, 0, None) == UNSUPPORTED  # K % 64
    assert g(PTR, PTR, 4, 512, 512, PTR, PTR, 100, PTR, 100, None, 0, None) == UNSUPPORTED  # N % 64
    assert g(None, PTR, 4, 512, 512, PTR, PTR, 512, PTR, 512, None, 0, None) == INVALID
    assert g(PTR, PTR, 4, 512, 500, PTR, PTR, 512, PTR, 512, None, 0, None) == INVALID      # ld_a < K
    assert g(MISALIGNED, PTR, 4, 512, 512, PTR, PTR, 512, PTR, 512, None, 0, None) == INVALID


def test_split_pack_norm_quant_validation(inv, L):
    assert L.heal_split(PTR, 0, 8, 8, PTR, PTR, 8, None) == OK
    assert L.heal_split(PTR, -1, 8, 8, PTR, PTR, 8, None) == INVALID
    assert L.heal_split(PTR, 4, 8, 4, PTR, PTR, 8, None) == INVALID
    assert L.heal_pack_weight(PTR, 100, 64, PTR, 10 ** 9, PTR, None) == UNSUPPORTED
    assert L.heal_pack_weight(PTR, 64, 64, PTR, 10 ** 9, PTR, None) == UNSUPPORTED       # N % 128
    assert L.heal_pack_weight(PTR, 64, 128, PTR, 10, PTR, None) == WORKSPACE
    assert L.rmsnorm_bi(PTR, PTR, 4, 6, 1e-6, PTR, None, None, None) == UNSUPPORTED
    assert L.rmsnorm_bi(PTR, PTR, 0, 64, 1e-6, PTR, None, None, None) == OK
    assert L.rmsnorm_bi(PTR, PTR, 4, 64, 1e-6, PTR, PTR, None, None) == INVALID          # hi without lo
    c = cache(inv, head_dim=64)
    assert L.kv_quant_int16(PTR, 4, 512, PTR, PTR, C.byref(c), 0, None) == UNSUPPORTED
    c = cache(inv)
    assert L.kv_quant_int16(PTR, 0, 1024, PTR, PTR, C.byref(c), 0, None) == OK
    assert L.kv_quant_int16(PTR, 4, 1024, PTR, PTR, C.byref(c), 2, None) == INVALID    # which
    assert L.kv_quant_int16(PTR, 4, 100, PTR, PTR, C.byref(c), 0, None) == INVALID     # ld_x too small


def test_attention_validation(inv, L):
    a = L.attn_decode_fixedsplit
    c = cache(inv)
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 128, 0.1, PTR, None, None, PTR, 10 ** 9, None) == UNSUPPORTED
    assert a(PTR, 4, 24, C.byref(c), PTR, PTR, 256, 256, 0.1, PTR, None, None, PTR, 10 ** 9, None) == UNSUPPORTED  # G = 3
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, PTR, None, None, PTR, 16, None) == WORKSPACE
    assert a(PTR, 0, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, PTR, None, None, PTR, 16, None) == OK
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, PTR, PTR, None, PTR, 10 ** 9, None) == INVALID  # hi w/o lo
    assert a(MISALIGNED, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, PTR, None, None, PTR, 10 ** 9, None) == INVALID  # q
    need = L.attn_decode_workspace_size(4, 32, 256)
    assert need == 4 * 32 * 1 * 520
    c_big = cache(inv, max_len=8192)
    assert L.attn_decode_fixedsplit_noalloc(PTR, 80, 32, C.byref(c_big), PTR, PTR, 8192, 256, 0.1, PTR, None, None,
                                            None) == WORKSPACE


def test_layer_validation(inv, L):
    Cfg = inv.LayerConfigStruct
    w = inv.LayerWeightsStruct(*([PTR.value] * 12))
    c = cache(inv, hkv=2, max_len=512)
    good = Cfg(256, 8, 2, 128, 512, 512, 1e-6, 0.088)
    d = L.decode_layer
    assert d(C.byref(good), C.byref(w), C.byref(c), PTR, PTR, PTR, 0, 512, PTR2, PTR, 0, None) == OK
    assert d(C.byref(Cfg(256, 8, 2, 64, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 512, PTR2, PTR,
             10 ** 9, None) == UNSUPPORTED
    assert d(C.byref(Cfg(200, 8, 2, 128, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 512, PTR2, PTR,
             10 ** 9, None) == UNSUPPORTED
    assert d(C.byref(Cfg(256, 6, 2, 128, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 512, PTR2, PTR,
             10 ** 9, None) == UNSUPPORTED                                               # G = 3
    assert d(C.byref(good), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 512, PTR, PTR, 10 ** 9, None) == INVALID  # in == out
    assert d(C.byref(good), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 512, PTR2, PTR, 64, None) == WORKSPACE
    pf = L.prefill_layer
    assert pf(C.byref(good), C.byref(w), C.byref(c), PTR, 0, 500, 20, 512, PTR2, PTR, 10 ** 9, None) == INVALID
    assert pf(C.byref(good), C.byref(w), C.byref(c), PTR, 5, 0, 20, 512, PTR2, PTR, 10 ** 9, None) == INVALID  # slot
    assert pf(C.byref(good), C.byref(w), C.byref(c), PTR, 0, 0, 0, 512, PTR2, PTR, 0, None) == OK


def test_helpers_validation(L):
    assert L.embed_gather(PTR, 0, 64, PTR, 4, PTR, None) == INVALID
    assert L.embed_gather(PTR, 10, 64, PTR, 0, PTR, None) == OK
    assert L.argmax_rows(PTR, 4, 100, 50, PTR, None) == INVALID
    assert L.rope_tables(0, 10000.0, PTR, PTR, None) == INVALID
    assert L.rope_tables(16, -1.0, PTR, PTR, None) == INVALID
    events = (C.c_void_p * 4)()
    assert L.inv_trace_events(events, 4) == INVALID
    assert L.inv_trace_events(None, 0) == OK
    assert L.inv_selftest_wait_timeout(0, None) == INVALID
    assert L.inv_selftest_gemm_wait_timeout(PTR, 1 << 20, 0, None) == INVALID
    assert L.inv_selftest_gemm_wait_timeout(None, 1 << 20, 1000, None) == INVALID
    assert L.inv_selftest_gemm_wait_timeout(PTR, 1024, 1000, None) == WORKSPACE


def test_workspace_sizes_use_the_resolved_bound(inv, L):
    """A call with max_len_bound <= 0 resolves its bound to cache->max_len; the
    size functions take that resolved bound and have no size for <= 0."""
    Cfg = inv.LayerConfigStruct
    good = Cfg(256, 8, 2, 128, 512, 512, 1e-6, 0.088)
    assert L.attn_decode_workspace_size(4, 32, 0) == 0
    assert L.decode_layer_workspace_size(C.byref(good), 4, 0) == 0
    assert L.prefill_layer_workspace_size(C.byref(good), 4, -5) == 0
    # a workspace sized with the cache's max_len is accepted by a call that passes bound 0
    w = inv.LayerWeightsStruct(*([PTR.value] * 12))
    c = cache(inv, hkv=2, max_len=512)
    need = L.decode_layer_workspace_size(C.byref(good), 4, 512)
    assert need > L.decode_layer_workspace_size(C.byref(good), 4, 256) > 0
    assert L.decode_layer(C.byref(good), C.byref(w), C.byref(c), PTR, PTR, PTR, 4, 0, PTR2, PTR, need - 1,
                          None) == WORKSPACE
    a = L.attn_decode_fixedsplit
    c8 = cache(inv, max_len=8192)
    need_a = L.attn_decode_workspace_size(4, 32, 8192)
    assert a(PTR, 4, 32, C.byref(c8), PTR, PTR, 0, 256, 0.1, PTR, None, None, PTR, need_a - 1, None) == WORKSPACE
    # the no-alloc variant applies its size limit to the resolved bound too
    c_big = cache(inv, max_len=8192)
    assert L.attn_decode_fixedsplit_noalloc(PTR, 80, 32, C.byref(c_big), PTR, PTR, 0, 256, 0.1, PTR, None, None,
                                            None) == WORKSPACE


def test_lamp_validation(inv, L):
    a = L.attn_decode_lamp
    c = cache(inv)
    nan = float("nan")
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, nan, PTR, None, None, None, 0, PTR, 10 ** 9,
             None) == INVALID                                                     # tau NaN
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 128, 0.1, 0.1, PTR, None, None, None, 0, PTR, 10 ** 9,
             None) == UNSUPPORTED                                                 # split
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, 0.1, PTR, None, None, PTR2, 100, PTR, 10 ** 9,
             None) == INVALID                                                     # recompute_ld < bound
    assert a(PTR, 4, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, 0.1, PTR, None, None, None, 0, PTR, 16,
             None) == WORKSPACE
    assert a(PTR, 0, 32, C.byref(c), PTR, PTR, 256, 256, 0.1, 0.1, PTR, None, None, None, 0, None, 0, None) == OK
