"""The C-ABI library loads and exports every entry point include/invnum.h
declares (CPU only: no compute call needs a GPU here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "invnum.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"INV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from invariant_numerics_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("heal_split", "heal_pack_weight", "comp_gemm", "kv_quant_int16", "attn_decode_fixedsplit",
              "rmsnorm_bi", "decode_layer", "inv_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    L, path = lib
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_functions()) <= exported
    # nothing but the declared C entry points is exported from the library's own code
    ours = {s for s in exported if not s.startswith("_") and not s.startswith("cu")}
    assert ours <= set(declared_functions()), ours - set(declared_functions())


def test_host_only_entry_points(lib):
    L, _ = lib
    L.inv_status_string.restype = ctypes.c_char_p
    assert L.inv_status_string(0) == b"INV_OK"
    assert L.inv_status_string(6) == b"INV_ERR_TIMEOUT"
    assert L.inv_status_string(99) == b"INV_ERR_UNKNOWN"
    assert L.inv_version() == 1
    L.heal_packed_weight_bytes.restype = ctypes.c_size_t
    assert L.heal_packed_weight_bytes(4096, 11008) == 4096 * 11008 * 4
    assert L.heal_packed_weight_bytes(0, 64) == 0
    L.attn_decode_workspace_size.restype = ctypes.c_size_t
    # (m, l) + o[128] per (row, head, split of 256)
    assert L.attn_decode_workspace_size(2, 32, 257) == 2 * 32 * 2 * (128 * 4 + 8)


def test_binding_module_exposes_the_same_names():
    import invariant_numerics_b200.invnum as inv
    for n in ("heal_split", "heal_pack_weight", "comp_gemm", "kv_quant_int16", "attn_decode_fixedsplit",
              "rmsnorm_bi", "decode_layer", "rope_tables", "embed_gather", "argmax_rows",
              "inv_get_device_status", "inv_set_wait_limit_ns", "inv_selftest_wait_timeout"):
        assert callable(getattr(inv, n)), n


@pytest.fixture(scope="module")
def debug_lib():
    from invariant_numerics_b200 import build
    path = build.build(debug_bounds=True)
    return ctypes.CDLL(path), path


def test_index_checking_build_exports_the_same_symbols(lib, debug_lib):
    L, path = lib
    D, dpath = debug_lib
    nm = lambda p: {ln.split()[-1] for ln in subprocess.run(["nm", "-D", "--defined-only", p], capture_output=True,
                                                             text=True).stdout.splitlines() if " T " in ln}
    assert set(declared_functions()) <= nm(dpath)
    assert {s for s in nm(dpath) if not s.startswith("_") and not s.startswith("cu")} <= set(declared_functions())
    assert L.inv_debug_bounds_enabled() == 0 and D.inv_debug_bounds_enabled() == 1
    L.inv_status_string.restype = ctypes.c_char_p
    assert L.inv_status_string(7) == b"INV_ERR_BOUNDS"
    # the normal build refuses the self-test (its stores would be unchecked) without touching the GPU
    buf = ctypes.c_void_p(16)
    assert L.inv_selftest_bounds(buf, 4, 8, None) == 2  # INV_ERR_UNSUPPORTED_SHAPE
    assert L.inv_selftest_bounds(buf, 8, 4, None) == 1  # n_written < n_declared
    assert D.inv_selftest_bounds(None, 4, 8, None) == 1
