"""Host-side argument validation of the C ABI (CPU only).

Every call below must return its status before touching the GPU: the shape,
range, alignment and workspace checks run first, and an empty call (zero
rows) is a no-op.  Pointers are dummy, 16-byte-aligned addresses that the
library never dereferences on these paths.
"""
import ctypes as C

import pytest

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
P = C.c_void_p(0x100000)          # aligned dummy device address
P2 = C.c_void_p(0x200000)
MISALIGNED = C.c_void_p(0x100004)


@pytest.fixture(scope="module")
def inv():
    from invariant_numerics_b200 import invnum  # loads the library and declares the argument types
    return invnum


@pytest.fixture(scope="module")
def L(inv):
    return inv.lib


def cache(inv, head_dim=128, max_len=256, n_slots=2, hkv=8):
    return inv.KVCacheStruct(P.value, P2.value, P.value, P2.value, n_slots, hkv, max_len, head_dim)


def test_comp_gemm_validation(L):
    g = L.comp_gemm
    assert g(P, P, 0, 512, 512, P, P, 512, P, 512, None, 0, None) == OK          # M = 0: no-op
    assert g(P, P, -1, 512, 512, P, P, 512, P, 512, None, 0, None) == INVALID
    assert g(P, P, 4, 100, 104, P, P, 512, P, 512, None, 0, None) == UNSUPPORTED  # K % 64
    assert g(P, P, 4, 512, 512, P, P, 100, P, 100, None, 0, None) == UNSUPPORTED  # N % 64
    assert g(None, P, 4, 512, 512, P, P, 512, P, 512, None, 0, None) == INVALID
    assert g(P, P, 4, 512, 500, P, P, 512, P, 512, None, 0, None) == INVALID      # ld_a < K
    assert g(MISALIGNED, P, 4, 512, 512, P, P, 512, P, 512, None, 0, None) == INVALID


def test_split_pack_norm_quant_validation(inv, L):
    assert L.heal_split(P, 0, 8, 8, P, P, 8, None) == OK
    assert L.heal_split(P, -1, 8, 8, P, P, 8, None) == INVALID
    assert L.heal_split(P, 4, 8, 4, P, P, 8, None) == INVALID
    assert L.heal_pack_weight(P, 100, 64, P, 10 ** 9, P, None) == UNSUPPORTED
    assert L.heal_pack_weight(P, 64, 64, P, 10 ** 9, P, None) == UNSUPPORTED       # N % 128
    assert L.heal_pack_weight(P, 64, 128, P, 10, P, None) == WORKSPACE
    assert L.rmsnorm_bi(P, P, 4, 6, 1e-6, P, None, None, None) == UNSUPPORTED
    assert L.rmsnorm_bi(P, P, 0, 64, 1e-6, P, None, None, None) == OK
    assert L.rmsnorm_bi(P, P, 4, 64, 1e-6, P, P, None, None) == INVALID          # hi without lo
    c = cache(inv, head_dim=64)
    assert L.kv_quant_int16(P, 4, 512, P, P, C.byref(c), 0, None) == UNSUPPORTED
    c = cache(inv)
    assert L.kv_quant_int16(P, 0, 1024, P, P, C.byref(c), 0, None) == OK
    assert L.kv_quant_int16(P, 4, 1024, P, P, C.byref(c), 2, None) == INVALID    # which
    assert L.kv_quant_int16(P, 4, 100, P, P, C.byref(c), 0, None) == INVALID     # ld_x too small


def test_attention_validation(inv, L):
    a = L.attn_decode_fixedsplit
    c = cache(inv)
    assert a(P, 4, 32, C.byref(c), P, P, 256, 128, 0.1, P, None, None, P, 10 ** 9, None) == UNSUPPORTED
    assert a(P, 4, 24, C.byref(c), P, P, 256, 256, 0.1, P, None, None, P, 10 ** 9, None) == UNSUPPORTED  # G = 3
    assert a(P, 4, 32, C.byref(c), P, P, 256, 256, 0.1, P, None, None, P, 16, None) == WORKSPACE
    assert a(P, 0, 32, C.byref(c), P, P, 256, 256, 0.1, P, None, None, P, 16, None) == OK
    assert a(P, 4, 32, C.byref(c), P, P, 256, 256, 0.1, P, P, None, P, 10 ** 9, None) == INVALID  # hi w/o lo
    assert a(MISALIGNED, 4, 32, C.byref(c), P, P, 256, 256, 0.1, P, None, None, P, 10 ** 9, None) == INVALID  # q
    need = L.attn_decode_workspace_size(4, 32, 256)
    assert need == 4 * 32 * 1 * 520
    c_big = cache(inv, max_len=8192)
    assert L.attn_decode_fixedsplit_noalloc(P, 80, 32, C.byref(c_big), P, P, 8192, 256, 0.1, P, None, None,
                                            None) == WORKSPACE


def test_layer_validation(inv, L):
    Cfg = inv.LayerConfigStruct
    w = inv.LayerWeightsStruct(*([P.value] * 12))
    c = cache(inv, hkv=2, max_len=512)
    good = Cfg(256, 8, 2, 128, 512, 512, 1e-6, 0.088)
    d = L.decode_layer
    assert d(C.byref(good), C.byref(w), C.byref(c), P, P, P, 0, 512, P2, P, 0, None) == OK
    assert d(C.byref(Cfg(256, 8, 2, 64, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), P, P, P, 4, 512, P2, P,
             10 ** 9, None) == UNSUPPORTED
    assert d(C.byref(Cfg(200, 8, 2, 128, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), P, P, P, 4, 512, P2, P,
             10 ** 9, None) == UNSUPPORTED
    assert d(C.byref(Cfg(256, 6, 2, 128, 512, 512, 1e-6, 0.088)), C.byref(w), C.byref(c), P, P, P, 4, 512, P2, P,
             10 ** 9, None) == UNSUPPORTED                                               # G = 3
    assert d(C.byref(good), C.byref(w), C.byref(c), P, P, P, 4, 512, P, P, 10 ** 9, None) == INVALID  # in == out
    assert d(C.byref(good), C.byref(w), C.byref(c), P, P, P, 4, 512, P2, P, 64, None) == WORKSPACE
    pf = L.prefill_layer
    assert pf(C.byref(good), C.byref(w), C.byref(c), P, 0, 500, 20, 512, P2, P, 10 ** 9, None) == INVALID
    assert pf(C.byref(good), C.byref(w), C.byref(c), P, 5, 0, 20, 512, P2, P, 10 ** 9, None) == INVALID  # slot
    assert pf(C.byref(good), C.byref(w), C.byref(c), P, 0, 0, 0, 512, P2, P, 0, None) == OK


def test_helpers_validation(L):
    assert L.embed_gather(P, 0, 64, P, 4, P, None) == INVALID
    assert L.embed_gather(P, 10, 64, P, 0, P, None) == OK
    assert L.argmax_rows(P, 4, 100, 50, P, None) == INVALID
    assert L.rope_tables(0, 10000.0, P, P, None) == INVALID
    assert L.rope_tables(16, -1.0, P, P, None) == INVALID
    events = (C.c_void_p * 4)()
    assert L.inv_trace_events(events, 4) == INVALID
    assert L.inv_trace_events(None, 0) == OK
    assert L.inv_selftest_wait_timeout(0, None) == INVALID
