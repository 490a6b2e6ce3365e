"""ctypes binding of libinvnum.so -- argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks tensor dtypes/devices/shapes, passes raw
device pointers and the current CUDA stream, and raises InvError on a non-OK
status.  PyTorch is used for device memory and streams only.  Importing this
module fails loudly (ImportError) if the library has not been built; there is
no fallback path.
"""
from __future__ import annotations

import ctypes as C
import math
import os
from dataclasses import dataclass, field

import torch

# INVNUM_LIBRARY may name another build of the same library (the
# index-checking libinvnum_debug.so); by default the package's libinvnum.so.
_LIB_PATH = os.environ.get("INVNUM_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                              "libinvnum.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m invariant_numerics_b200.build`")
lib = C.CDLL(_LIB_PATH)

INV_OK, INV_ERR_INVALID_ARG, INV_ERR_UNSUPPORTED_SHAPE, INV_ERR_WORKSPACE, INV_ERR_CUDA, INV_ERR_RANGE, \
    INV_ERR_TIMEOUT, INV_ERR_BOUNDS = range(8)
KV_SPLIT = 256
HEAD_DIM = 128

_p, _i, _i64, _sz, _f, _d = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_float, C.c_double


class InvError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {lib.inv_status_string(code).decode()} ({code})")


class KVCacheStruct(C.Structure):
    _fields_ = [("k", _p), ("v", _p), ("k_scale", _p), ("v_scale", _p), ("n_slots", _i), ("n_kv_heads", _i),
                ("max_len", _i), ("head_dim", _i)]


class LayerConfigStruct(C.Structure):
    _fields_ = [("hidden", _i), ("n_heads", _i), ("n_kv_heads", _i), ("head_dim", _i), ("ffn", _i),
                ("max_pos", _i), ("eps", _f), ("softmax_scale", _f)]


class LayerWeightsStruct(C.Structure):
    _fields_ = [("w_qkv", _p), ("e_qkv", _p), ("w_o", _p), ("e_o", _p), ("w_gu", _p), ("e_gu", _p),
                ("w_down", _p), ("e_down", _p), ("g_attn", _p), ("g_mlp", _p), ("rope_cos", _p),
                ("rope_sin", _p)]


_SIGS = {
    "inv_status_string": (C.c_char_p, [_i]),
    "inv_version": (_i, []),
    "inv_get_device_status": (_i, [C.POINTER(_i), _p]),
    "inv_set_wait_limit_ns": (_i, [C.c_longlong]),
    "inv_selftest_wait_timeout": (_i, [C.c_longlong, _p]),
    "inv_debug_bounds_enabled": (_i, []),
    "inv_selftest_bounds": (_i, [_p, _i, _i, _p]),
    "inv_selftest_gemm_wait_timeout": (_i, [_p, _sz, C.c_longlong, _p]),
    "inv_trace_events": (_i, [C.POINTER(C.c_void_p), _i]),
    "heal_split": (_i, [_p, _i64, _i64, _i64, _p, _p, _i64, _p]),
    "heal_packed_weight_bytes": (_sz, [_i, _i]),
    "heal_pack_weight": (_i, [_p, _i, _i, _p, _sz, _p, _p]),
    "comp_gemm": (_i, [_p, _p, _i64, _i, _i64, _p, _p, _i, _p, _i64, _p, _i64, _p]),
    "kv_quant_int16": (_i, [_p, _i, _i64, _p, _p, C.POINTER(KVCacheStruct), _i, _p]),
    "attn_decode_workspace_size": (_sz, [_i, _i, _i]),
    "attn_decode_fixedsplit": (_i, [_p, _i, _i, C.POINTER(KVCacheStruct), _p, _p, _i, _i, _f, _p, _p, _p, _p,
                                    _sz, _p]),
    "attn_decode_fixedsplit_noalloc": (_i, [_p, _i, _i, C.POINTER(KVCacheStruct), _p, _p, _i, _i, _f, _p, _p,
                                            _p, _p]),
    "attn_decode_lamp": (_i, [_p, _i, _i, C.POINTER(KVCacheStruct), _p, _p, _i, _i, _f, _f, _p, _p, _p, _p, _i64,
                              _p, _sz, _p]),
    "rmsnorm_bi": (_i, [_p, _p, _i64, _i, _f, _p, _p, _p, _p]),
    "decode_layer_workspace_size": (_sz, [C.POINTER(LayerConfigStruct), _i, _i]),
    "decode_layer": (_i, [C.POINTER(LayerConfigStruct), C.POINTER(LayerWeightsStruct), C.POINTER(KVCacheStruct),
                          _p, _p, _p, _i, _i, _p, _p, _sz, _p]),
    "prefill_layer_workspace_size": (_sz, [C.POINTER(LayerConfigStruct), _i, _i]),
    "prefill_layer": (_i, [C.POINTER(LayerConfigStruct), C.POINTER(LayerWeightsStruct), C.POINTER(KVCacheStruct),
                           _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "rope_tables": (_i, [_i, _d, _p, _p, _p]),
    "embed_gather": (_i, [_p, _i, _i, _p, _i, _p, _p]),
    "argmax_rows": (_i, [_p, _i, _i, _i64, _p, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def _check(fn: str, rc: int) -> None:
    if rc != INV_OK:
        raise InvError(fn, rc)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _resolved_bound(cache, max_len_bound: int) -> int:
    """The KV length bound a call resolves to (the C entry points' rule): the
    caller's bound clipped to the cache, or the cache's max_len for <= 0."""
    return cache.max_len if max_len_bound <= 0 else min(max_len_bound, cache.max_len)


def _need(t, dtype, name, contiguous=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# --------------------------------------------------------------- status ------

def status_string(code: int) -> str:
    return lib.inv_status_string(code).decode()


def inv_get_device_status(stream=None) -> int:
    out = C.c_int(0)
    _check("inv_get_device_status", lib.inv_get_device_status(C.byref(out), _stream(stream)))
    return out.value


def inv_set_wait_limit_ns(ns: int) -> None:
    _check("inv_set_wait_limit_ns", lib.inv_set_wait_limit_ns(int(ns)))


def inv_selftest_wait_timeout(wait_ns: int, stream=None) -> None:
    _check("inv_selftest_wait_timeout", lib.inv_selftest_wait_timeout(int(wait_ns), _stream(stream)))


SELFTEST_GEMM_WS_BYTES = 40192


def inv_selftest_gemm_wait_timeout(wait_ns: int, workspace=None, stream=None) -> None:
    ws = torch.empty(SELFTEST_GEMM_WS_BYTES, dtype=torch.uint8, device="cuda") if workspace is None else workspace
    _check("inv_selftest_gemm_wait_timeout",
           lib.inv_selftest_gemm_wait_timeout(_ptr(ws), ws.numel(), int(wait_ns), _stream(stream)))


def inv_debug_bounds_enabled() -> bool:
    return bool(lib.inv_debug_bounds_enabled())


def inv_selftest_bounds(buf, n_declared: int, n_written: int, stream=None) -> None:
    _need(buf, torch.float32, "buf")
    if buf.numel() < n_declared:
        raise ValueError("buf must hold n_declared floats")
    _check("inv_selftest_bounds", lib.inv_selftest_bounds(_ptr(buf), int(n_declared), int(n_written), _stream(stream)))


DECODE_LAYER_KERNELS = 8
DECODE_LAYER_KERNEL_NAMES = ("rmsnorm_attn", "gemm_qkv_rope_quant", "attn_split", "attn_combine", "gemm_o",
                             "rmsnorm_mlp", "gemm_gate_up_swiglu", "gemm_down")


def inv_trace_events(events) -> None:
    """Trace decode_layer kernels into torch.cuda.Event objects (2 per kernel), or None to stop."""
    if events is None:
        _check("inv_trace_events", lib.inv_trace_events(None, 0))
        return
    for e in events:  # torch creates the CUDA event lazily, on first record
        if e.cuda_event == 0:
            e.record()
    handles = (C.c_void_p * len(events))(*[C.c_void_p(e.cuda_event) for e in events])
    inv_trace_events._keep = handles  # the library keeps the pointer
    _check("inv_trace_events", lib.inv_trace_events(handles, len(events)))


# ----------------------------------------------------------- operations ------

def heal_split(x, hi=None, lo=None, stream=None):
    """fp32 [rows, cols] -> (hi, lo) binary16 tensors (torch.float16)."""
    _need(x, torch.float32, "x")
    rows, cols = x.shape
    hi = torch.empty((rows, cols), dtype=torch.float16, device=x.device) if hi is None else hi
    lo = torch.empty((rows, cols), dtype=torch.float16, device=x.device) if lo is None else lo
    _need(hi, torch.float16, "hi"), _need(lo, torch.float16, "lo")
    _check("heal_split", lib.heal_split(_ptr(x), rows, cols, cols, _ptr(hi), _ptr(lo), cols, _stream(stream)))
    return hi, lo


def heal_pack_weight(W, stream=None):
    """fp32 W [K, N] (y = x W) -> (packed binary16 [N/128, 2, 128, K], col_exp int8 [N])."""
    _need(W, torch.float32, "W")
    K, N = W.shape
    packed = torch.empty((N // 128, 2, 128, K), dtype=torch.float16, device=W.device)
    col_exp = torch.empty((N,), dtype=torch.int8, device=W.device)
    nbytes = lib.heal_packed_weight_bytes(K, N)
    _check("heal_pack_weight", lib.heal_pack_weight(_ptr(W), K, N, _ptr(packed), nbytes, _ptr(col_exp),
                                                    _stream(stream)))
    return packed, col_exp


def comp_gemm(a_hi, a_lo, packed, col_exp, residual=None, out=None, stream=None):
    """(a_hi, a_lo) binary16 [M, K] x packed weight [K, N] -> fp32 [M, N] (+ residual)."""
    _need(a_hi, torch.float16, "a_hi"), _need(a_lo, torch.float16, "a_lo")
    _need(packed, torch.float16, "packed"), _need(col_exp, torch.int8, "col_exp")
    M, K = a_hi.shape
    N = col_exp.shape[0]
    if packed.numel() != 2 * K * N:
        raise ValueError("packed weight does not match K, N")
    y = torch.empty((M, N), dtype=torch.float32, device=a_hi.device) if out is None else _need(out, torch.float32, "out")
    if residual is not None:
        _need(residual, torch.float32, "residual")
    _check("comp_gemm", lib.comp_gemm(_ptr(a_hi), _ptr(a_lo), M, K, K, _ptr(packed), _ptr(col_exp), N, _ptr(y), N,
                                      _ptr(residual), N if residual is not None else 0, _stream(stream)))
    return y


@dataclass
class KVCache:
    """INT16 KV cache in device memory, layout [slot][kv_head][pos][128]."""
    n_slots: int
    n_kv_heads: int
    max_len: int
    device: str = "cuda"
    k: torch.Tensor = field(init=False)
    v: torch.Tensor = field(init=False)
    k_scale: torch.Tensor = field(init=False)
    v_scale: torch.Tensor = field(init=False)

    def __post_init__(self):
        shape = (self.n_slots, self.n_kv_heads, self.max_len, HEAD_DIM)
        self.k = torch.zeros(shape, dtype=torch.int16, device=self.device)
        self.v = torch.zeros(shape, dtype=torch.int16, device=self.device)
        self.k_scale = torch.zeros(shape[:3], dtype=torch.float32, device=self.device)
        self.v_scale = torch.zeros(shape[:3], dtype=torch.float32, device=self.device)

    def struct(self) -> KVCacheStruct:
        return KVCacheStruct(self.k.data_ptr(), self.v.data_ptr(), self.k_scale.data_ptr(), self.v_scale.data_ptr(),
                             self.n_slots, self.n_kv_heads, self.max_len, HEAD_DIM)


def kv_quant_int16(x, slot, pos, cache: KVCache, which: str, stream=None):
    """fp32 x [T, Hkv, 128] -> cache (which = 'k' or 'v') at (slot[t], :, pos[t])."""
    _need(x, torch.float32, "x"), _need(slot, torch.int32, "slot"), _need(pos, torch.int32, "pos")
    T = x.shape[0]
    cs = cache.struct()
    _check("kv_quant_int16", lib.kv_quant_int16(_ptr(x), T, cache.n_kv_heads * HEAD_DIM, _ptr(slot), _ptr(pos),
                                                C.byref(cs), 0 if which == "k" else 1, _stream(stream)))


def attn_decode_workspace_size(B: int, n_heads: int, max_len_bound: int) -> int:
    return lib.attn_decode_workspace_size(B, n_heads, max_len_bound)


def attn_decode_fixedsplit(q, cache: KVCache, slot, lens, softmax_scale, max_len_bound=None, out=None,
                           want_split=False, workspace=None, stream=None):
    """q fp32 [B, Hq, 128] over the cache -> out fp32 [B, Hq, 128] (and hi/lo if want_split)."""
    _need(q, torch.float32, "q"), _need(slot, torch.int32, "slot"), _need(lens, torch.int32, "lens")
    B, Hq, D = q.shape
    mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
    out = torch.empty_like(q) if out is None else _need(out, torch.float32, "out")
    hi = torch.empty(q.shape, dtype=torch.float16, device=q.device) if want_split else None
    lo = torch.empty(q.shape, dtype=torch.float16, device=q.device) if want_split else None
    nbytes = lib.attn_decode_workspace_size(B, Hq, _resolved_bound(cache, mlb))
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q.device)
    cs = cache.struct()
    _check("attn_decode_fixedsplit",
           lib.attn_decode_fixedsplit(_ptr(q), B, Hq, C.byref(cs), _ptr(slot), _ptr(lens), mlb, KV_SPLIT,
                                      float(softmax_scale), _ptr(out), _ptr(hi), _ptr(lo), _ptr(workspace),
                                      workspace.numel(), _stream(stream)))
    return (out, hi, lo) if want_split else out


def attn_decode_lamp(q, cache: KVCache, slot, lens, softmax_scale, tau, max_len_bound=None, out=None,
                     want_recompute=False, workspace=None, stream=None):
    """LAMP selective-recompute variant of attn_decode_fixedsplit: q fp32
    [B, Hq, 128] -> out fp32 [B, Hq, 128] (and, if want_recompute, the uint8
    recompute flags [B, Hq, L] for L = the resolved length bound)."""
    _need(q, torch.float32, "q"), _need(slot, torch.int32, "slot"), _need(lens, torch.int32, "lens")
    B, Hq, D = q.shape
    mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
    L = _resolved_bound(cache, mlb)
    out = torch.empty_like(q) if out is None else _need(out, torch.float32, "out")
    rec = torch.zeros((B, Hq, L), dtype=torch.uint8, device=q.device) if want_recompute else None
    nbytes = lib.attn_decode_workspace_size(B, Hq, L)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q.device)
    cs = cache.struct()
    _check("attn_decode_lamp",
           lib.attn_decode_lamp(_ptr(q), B, Hq, C.byref(cs), _ptr(slot), _ptr(lens), mlb, KV_SPLIT,
                                float(softmax_scale), float(tau), _ptr(out), None, None, _ptr(rec), L,
                                _ptr(workspace), workspace.numel(), _stream(stream)))
    return (out, rec) if want_recompute else out


NOALLOC_SCRATCH_BYTES = 34 << 20


def attn_decode_fixedsplit_noalloc(q, cache: KVCache, slot, lens, softmax_scale, max_len_bound=None, out=None,
                                   want_split=False, stream=None):
    """attn_decode_fixedsplit without a workspace argument, for callers that
    cannot allocate device memory: the library's own fixed 34 MiB device
    array holds the split partials (see include/invnum.h for the limits).
    `out` (and the hi/lo buffers when want_split) must then be passed in by
    such a caller; this wrapper only allocates them when they are omitted."""
    _need(q, torch.float32, "q"), _need(slot, torch.int32, "slot"), _need(lens, torch.int32, "lens")
    B, Hq, D = q.shape
    mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
    out = torch.empty_like(q) if out is None else _need(out, torch.float32, "out")
    hi = torch.empty(q.shape, dtype=torch.float16, device=q.device) if want_split else None
    lo = torch.empty(q.shape, dtype=torch.float16, device=q.device) if want_split else None
    cs = cache.struct()
    _check("attn_decode_fixedsplit_noalloc",
           lib.attn_decode_fixedsplit_noalloc(_ptr(q), B, Hq, C.byref(cs), _ptr(slot), _ptr(lens), mlb, KV_SPLIT,
                                              float(softmax_scale), _ptr(out), _ptr(hi), _ptr(lo), _stream(stream)))
    return (out, hi, lo) if want_split else out


def rmsnorm_bi(x, gamma, eps, want_y=True, want_split=False, stream=None):
    """fp32 x [rows, hidden] -> y fp32 and/or (hi, lo) binary16."""
    _need(x, torch.float32, "x"), _need(gamma, torch.float32, "gamma")
    rows, hidden = x.shape
    y = torch.empty_like(x) if want_y else None
    hi = torch.empty(x.shape, dtype=torch.float16, device=x.device) if want_split else None
    lo = torch.empty(x.shape, dtype=torch.float16, device=x.device) if want_split else None
    _check("rmsnorm_bi", lib.rmsnorm_bi(_ptr(x), _ptr(gamma), rows, hidden, float(eps), _ptr(y), _ptr(hi), _ptr(lo),
                                        _stream(stream)))
    if want_y and want_split:
        return y, hi, lo
    return y if want_y else (hi, lo)


def rope_tables(max_pos: int, base: float = 10000.0, device="cuda", stream=None):
    cs = torch.empty((max_pos, 64), dtype=torch.float32, device=device)
    sn = torch.empty((max_pos, 64), dtype=torch.float32, device=device)
    _check("rope_tables", lib.rope_tables(max_pos, float(base), _ptr(cs), _ptr(sn), _stream(stream)))
    return cs, sn


def embed_gather(table, ids, out=None, stream=None):
    _need(table, torch.float32, "table"), _need(ids, torch.int32, "ids")
    vocab, hidden = table.shape
    B = ids.shape[0]
    out = torch.empty((B, hidden), dtype=torch.float32, device=table.device) if out is None else out
    _check("embed_gather", lib.embed_gather(_ptr(table), vocab, hidden, _ptr(ids), B, _ptr(out), _stream(stream)))
    return out


def argmax_rows(logits, out=None, stream=None):
    _need(logits, torch.float32, "logits")
    B, n = logits.shape
    out = torch.empty((B,), dtype=torch.int32, device=logits.device) if out is None else out
    _check("argmax_rows", lib.argmax_rows(_ptr(logits), B, n, n, _ptr(out), _stream(stream)))
    return out


# ------------------------------------------------------------ the layer ------

@dataclass
class LayerConfig:
    hidden: int
    n_heads: int
    n_kv_heads: int
    ffn: int
    max_pos: int
    eps: float = 1e-6
    head_dim: int = HEAD_DIM
    rope_base: float = 10000.0

    @property
    def softmax_scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.head_dim), dtype=torch.float32))

    def struct(self) -> LayerConfigStruct:
        return LayerConfigStruct(self.hidden, self.n_heads, self.n_kv_heads, self.head_dim, self.ffn, self.max_pos,
                                 self.eps, self.softmax_scale)


def gate_up_order(F: int, device) -> torch.Tensor:
    """Column order of [gate | up] (2F columns) for the fused SwiGLU epilogue:
    per 32 outputs j and half h, 16 gate columns then the 16 matching up columns."""
    j = torch.arange(F // 32, device=device).view(-1, 1, 1, 1)
    h = torch.arange(2, device=device).view(1, -1, 1, 1)
    part = torch.arange(2, device=device).view(1, 1, -1, 1)
    i = torch.arange(16, device=device).view(1, 1, 1, -1)
    return (part * F + 32 * j + 16 * h + i).reshape(-1)


class LayerWeights:
    """Packed weights of one layer, built on the device by heal_pack_weight.

    Inputs are fp32 CUDA tensors in y = x W orientation: wq [H, Hq*128],
    wk/wv [H, Hkv*128], wo [Hq*128, H], w_gate/w_up [H, F], w_down [F, H],
    g_attn/g_mlp [H].  The fused projections gather columns before packing:
    q | k | v, and gate/up interleaved in groups of 16 (gate 32j+16h..+15,
    then up 32j+16h..+15) as the fused SwiGLU epilogue expects.  Packing is
    per column, so reordering columns does not change any column's numbers.
    """

    def __init__(self, cfg: LayerConfig, wq, wk, wv, wo, w_gate, w_up, w_down, g_attn, g_mlp, rope=None):
        self.w_qkv, self.e_qkv = heal_pack_weight(torch.cat([wq, wk, wv], dim=1).contiguous())
        self.w_o, self.e_o = heal_pack_weight(wo.contiguous())
        F = w_gate.shape[1]
        self.w_gu, self.e_gu = heal_pack_weight(torch.cat([w_gate, w_up], dim=1)[:, gate_up_order(F, w_gate.device)]
                                                .contiguous())
        self.w_down, self.e_down = heal_pack_weight(w_down.contiguous())
        self.g_attn = g_attn.contiguous()
        self.g_mlp = g_mlp.contiguous()
        self.rope_cos, self.rope_sin = rope if rope is not None else rope_tables(cfg.max_pos, cfg.rope_base,
                                                                                  device=wq.device)

    def struct(self) -> LayerWeightsStruct:
        t = lambda x: x.data_ptr()
        return LayerWeightsStruct(t(self.w_qkv), t(self.e_qkv), t(self.w_o), t(self.e_o), t(self.w_gu), t(self.e_gu),
                                  t(self.w_down), t(self.e_down), t(self.g_attn), t(self.g_mlp), t(self.rope_cos),
                                  t(self.rope_sin))


def decode_layer_workspace_size(cfg: LayerConfig, B: int, max_len_bound: int) -> int:
    cs = cfg.struct()
    return lib.decode_layer_workspace_size(C.byref(cs), B, max_len_bound)


def decode_layer(cfg: LayerConfig, w: LayerWeights, cache: KVCache, x, slot, pos, max_len_bound=None, out=None,
                 workspace=None, stream=None):
    """One layer over B rows: fp32 x [B, H] -> fp32 [B, H]; writes the rows' K/V into the cache."""
    _need(x, torch.float32, "x"), _need(slot, torch.int32, "slot"), _need(pos, torch.int32, "pos")
    B = x.shape[0]
    mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
    cs, ws_, cc = cfg.struct(), w.struct(), cache.struct()
    nbytes = lib.decode_layer_workspace_size(C.byref(cs), B, _resolved_bound(cache, mlb))
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=x.device)
    out = torch.empty_like(x) if out is None else _need(out, torch.float32, "out")
    _check("decode_layer", lib.decode_layer(C.byref(cs), C.byref(ws_), C.byref(cc), _ptr(x), _ptr(slot), _ptr(pos), B,
                                            mlb, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def prefill_layer(cfg: LayerConfig, w: LayerWeights, cache: KVCache, x, slot: int, pos0: int, max_len_bound=None,
                  out=None, workspace=None, stream=None):
    """Rows x [T, H] at positions pos0 .. pos0+T-1 of the sequence in `slot`;
    bit-identical per row to decode_layer, with each attention split loaded
    once for the whole chunk."""
    _need(x, torch.float32, "x")
    T = x.shape[0]
    mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
    cs, ws_, cc = cfg.struct(), w.struct(), cache.struct()
    nbytes = lib.prefill_layer_workspace_size(C.byref(cs), T, _resolved_bound(cache, mlb))
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=x.device)
    out = torch.empty_like(x) if out is None else _need(out, torch.float32, "out")
    _check("prefill_layer", lib.prefill_layer(C.byref(cs), C.byref(ws_), C.byref(cc), _ptr(x), int(slot), int(pos0),
                                              T, mlb, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


class DecodeLayerCall:
    """decode_layer with every argument marshalled once: calling it issues one
    C call with fixed device buffers (x, slot, pos, out, workspace)."""

    def __init__(self, cfg: LayerConfig, w: LayerWeights, cache: KVCache, x, slot, pos, out, max_len_bound=None):
        _need(x, torch.float32, "x"), _need(slot, torch.int32, "slot"), _need(pos, torch.int32, "pos")
        _need(out, torch.float32, "out")
        self.B = x.shape[0]
        self.mlb = cache.max_len if max_len_bound is None else int(max_len_bound)
        self._cs, self._ws, self._cc = cfg.struct(), w.struct(), cache.struct()
        nbytes = lib.decode_layer_workspace_size(C.byref(self._cs), self.B, _resolved_bound(cache, self.mlb))
        self.workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=x.device)
        self._keep = (cfg, w, cache, x, slot, pos, out)
        self._args = (C.byref(self._cs), C.byref(self._ws), C.byref(self._cc), _ptr(x), _ptr(slot), _ptr(pos), self.B,
                      self.mlb, _ptr(out), _ptr(self.workspace), self.workspace.numel())

    def __call__(self, stream=None):
        _check("decode_layer", lib.decode_layer(*self._args, _stream(stream)))
