"""Plain float64 definitions of what the decode step computes (oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Everything here is the mathematical definition evaluated in float64 from the
fp32 inputs: no blocking, no splitting, no fixed-split softmax.  The fixed
reduction orders of the batch-invariant kernels [BI] are GPU strategies for
reproducing *one* rounding of these definitions; the oracle instead computes
the exact-as-possible value the method approximates.  The only encodings used
are the KV-cache quantiser (the cache is INT16 by definition [HEAL, section
"1. 「スマート・パッキング」のトリック"]) from `oracle.encodings`.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import encodings as enc


def f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# matrix product  [HEAL, section "2. 「誤差補償」のトリック（計算用）": the
# compensated GEMM targets FP32-grade accuracy of y = x W]
# ----------------------------------------------------------------------------

def gemm(A, W) -> np.ndarray:
    """y = A W in float64 (fp32 products are exact in float64)."""
    return f64(A) @ f64(W)


def gemm_fp16_only(A, W) -> np.ndarray:
    """Diagnostic: the uncompensated 16-bit product rn16(A) rn16(W), float64 sums."""
    a = enc.f16_bits_to_f64(enc.rn16_bits(f64(np.asarray(A, np.float32))))
    w = enc.f16_bits_to_f64(enc.rn16_bits(f64(np.asarray(W, np.float32))))
    return a @ w


def gemm_split3(A, W) -> np.ndarray:
    """Diagnostic: the three-product algebra A_hi B_hi + 2^-11 (A_hi B_lo + A_lo B_hi),
    rescaled by 2^-e_n, summed in float64 (isolates truncation from rounding)."""
    a_hi, a_lo, _ = enc.heal_split(A, 0)
    e = enc.column_exponents(W).astype(np.int64)
    w_hi, w_lo, _ = enc.heal_split(W, e[None, :])
    ah, al = enc.f16_bits_to_f64(a_hi), enc.f16_bits_to_f64(a_lo)
    wh, wl = enc.f16_bits_to_f64(w_hi), enc.f16_bits_to_f64(w_lo)
    y = ah @ wh + np.ldexp(ah @ wl + al @ wh, -enc.LO_SCALE_LOG2)
    return np.ldexp(y, -e[None, :])


# ----------------------------------------------------------------------------
# RMSNorm  [BI, table row "RMSNorm"]
# ----------------------------------------------------------------------------

def rmsnorm(x, gamma, eps) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * gamma, per row, float64."""
    x = f64(x)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + float(eps))
    return x * r * f64(gamma)


# ----------------------------------------------------------------------------
# rotary position embedding (rotate-half pairing (i, i + D/2), theta_i = base^(-2i/D))
# ----------------------------------------------------------------------------

def rope_angles(pos, head_dim: int, base: float = 10000.0) -> np.ndarray:
    """angle[p, i] = pos_p * base^(-2 i / D), float64 [len(pos), D/2]."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / head_dim)
    return f64(pos)[:, None] * theta[None, :]


def apply_rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate x[T, H, D] by the angles of positions pos[T] (float64)."""
    x = f64(x)
    D = x.shape[-1]
    ang = rope_angles(pos, D, base)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# ----------------------------------------------------------------------------
# KV cache (INT16 codes + fp32 scales, layout [slot][kv_head][pos][D])
# ----------------------------------------------------------------------------

@dataclass
class KVCache:
    k: np.ndarray        # int16 [S, Hkv, Lmax, D]
    ks: np.ndarray       # fp32  [S, Hkv, Lmax]
    v: np.ndarray
    vs: np.ndarray

    @staticmethod
    def empty(n_slots: int, n_kv: int, max_len: int, head_dim: int) -> "KVCache":
        return KVCache(np.zeros((n_slots, n_kv, max_len, head_dim), np.int16),
                       np.zeros((n_slots, n_kv, max_len), np.float32),
                       np.zeros((n_slots, n_kv, max_len, head_dim), np.int16),
                       np.zeros((n_slots, n_kv, max_len), np.float32))

    def write(self, which: str, x, slot, pos) -> None:
        """Quantise fp32 x[T, Hkv, D] and store it at (slot[t], :, pos[t])."""
        q, s = enc.kv_quant_int16(np.asarray(x, np.float32))
        codes, scales = (self.k, self.ks) if which == "k" else (self.v, self.vs)
        for t in range(q.shape[0]):
            codes[slot[t], :, pos[t]] = q[t]
            scales[slot[t], :, pos[t]] = s[t]


# ----------------------------------------------------------------------------
# decode attention over the dequantised cache  [BI, table row "Attention";
# HEAL, section "1. 「スマート・パッキング」のトリック"]
# ----------------------------------------------------------------------------

def attention_decode(q, cache: KVCache, slot, length, softmax_scale, return_probs=False):
    """One query row per sequence: out[b, h] = sum_j p_j V~_j with
    p = softmax_j(sigma q_h . K~_j) over the first length[b] keys of slot[b].

    q: [B, Hq, D]; K~/V~ are the exact float64 dequantised cache values; query
    head h reads kv head h // (Hq / Hkv).  softmax_scale is taken as the fp32
    value the caller passes, promoted to float64.  The softmax is one pass over
    all keys (the definition), not the GPU's fixed 256-key splits.
    """
    q = f64(q)
    B, Hq, D = q.shape
    Hkv = cache.k.shape[1]
    G = Hq // Hkv
    sigma = float(np.float32(softmax_scale))
    out = np.zeros((B, Hq, D), np.float64)
    probs = []
    for b in range(B):
        L = int(length[b])
        s = int(slot[b])
        Kt = enc.kv_dequant(cache.k[s, :, :L], cache.ks[s, :, :L])   # [Hkv, L, D]
        Vt = enc.kv_dequant(cache.v[s, :, :L], cache.vs[s, :, :L])
        qb = q[b].reshape(Hkv, G, D)
        t = sigma * np.einsum("hgd,hld->hgl", qb, Kt)                # [Hkv, G, L]
        t = t - t.max(axis=-1, keepdims=True)
        p = np.exp(t)
        p = p / p.sum(axis=-1, keepdims=True)
        out[b] = np.einsum("hgl,hld->hgd", p, Vt).reshape(Hq, D)
        if return_probs:
            probs.append(p.reshape(Hq, L))
    return (out, probs) if return_probs else out


# ----------------------------------------------------------------------------
# LAMP-style selective recompute of the attention scores  [LAMP summary
# ("LAMP", gist.science), section "Fondement théorique", item 3 (softmax: the l1
# objective and the condition 2 z_j (1 - z_j) |y_j| > tau for recomputing the
# KQ product y_j), section "Stratégie d'implémentation" (evaluate in low
# precision, select from the low-precision result, recompute the selected
# components in higher precision) and the relaxed relative-threshold variant of
# "Résultats expérimentaux" (no dependence on the normalisation constant, for
# single-pass softmax kernels)]
# ----------------------------------------------------------------------------

def softmax_l1_sensitivity(y) -> np.ndarray:
    """2 z_j (1 - z_j) |y_j| with z = softmax(y): the l1 change of the softmax
    output, to first order, per unit relative error in the score y_j."""
    y = f64(y)
    z = np.exp(y - y.max())
    z = z / z.sum()
    return 2.0 * z * (1.0 - z) * np.abs(y)


def lamp_relaxed_criterion(y, split: int = 256) -> np.ndarray:
    """The relaxed criterion 2 exp(y_j - m_s) |y_j|, m_s the largest score of
    the fixed `split`-key block (absolute positions split*s ..) that holds key
    j: no normalisation constant is needed, and since z_j <= exp(y_j - m_s)
    and 1 - z_j <= 1 it bounds the strict 2 z_j (1 - z_j) |y_j| from above, so
    it selects every score the strict rule selects (and some more)."""
    y = f64(y)
    out = np.empty_like(y)
    for s0 in range(0, y.shape[-1], split):
        ys = y[..., s0:s0 + split]
        zh = np.exp(ys - ys.max(axis=-1, keepdims=True))
        out[..., s0:s0 + split] = 2.0 * zh * np.abs(ys)
    return out


def lamp_low_precision_scores(q16_bits, codes, scales, softmax_scale) -> np.ndarray:
    """Scores y_lo_j accumulated in binary16 (the low-precision evaluation).

    With code = 256 h + l (h the signed high byte, l the low byte, both exact
    in binary16 as h and l/256), two binary16 accumulators run over
    d = 0, 1, ..., D-1 in order, each step one fused multiply-add rounded once
    to binary16 (round half to even):
        a_h <- rn16(q16_d h_jd + a_h),   a_l <- rn16(q16_d (l_jd / 256) + a_l)
    (a sum that leaves the binary16 range becomes +-inf).  Then, in fp32 and in
    this order, y_lo_j = ((256 a_h + 256 a_l) s_j) sigma.
      q16_bits : uint16 [D] binary16 bits of the query head
      codes    : int16 [L, D] INT16 codes of the keys;  scales : fp32 [L]
    Returns fp32 [L]."""
    q16 = enc.f16_bits_to_f64(np.asarray(q16_bits, np.uint16))
    c = np.asarray(codes, np.int64)
    h = (c >> 8).astype(np.float64)                 # arithmetic shift: the signed high byte
    l = (c & 255).astype(np.float64) / 256.0
    a_h = np.zeros(c.shape[0], np.float64)
    a_l = np.zeros(c.shape[0], np.float64)
    for d in range(c.shape[1]):                     # products and sums exact in float64
        a_h = enc.f16_bits_to_f64(enc.rn16_bits(q16[d] * h[:, d] + a_h))
        a_l = enc.f16_bits_to_f64(enc.rn16_bits(q16[d] * l[:, d] + a_l))
    with np.errstate(invalid="ignore", over="ignore"):
        t = np.float32(256.0) * a_h.astype(np.float32) + np.float32(256.0) * a_l.astype(np.float32)
        return (t * np.asarray(scales, np.float32)) * np.float32(softmax_scale)


def lamp_criterion_f32(y_lo, split: int = 256) -> np.ndarray:
    """The relaxed criterion of fp32 low-precision scores y_lo [L] (keys at
    absolute positions 0..L-1) evaluated in fp32:
        zh = fl32(exp(y - m_s)),  c = (2 zh) |y|,
    m_s the largest finite score of the key's 256-key block; +inf for a
    non-finite score (always recomputed)."""
    y = np.asarray(y_lo, np.float32)
    c = np.full(y.shape, np.inf, np.float32)
    for s0 in range(0, y.shape[-1], split):
        ys = y[s0:s0 + split]
        fin = np.isfinite(ys)
        if not fin.any():
            continue
        m = ys[fin].max()
        with np.errstate(invalid="ignore", over="ignore"):
            zh = np.exp((ys - m).astype(np.float64)).astype(np.float32)
            c[s0:s0 + split] = np.where(fin, (np.float32(2.0) * zh) * np.abs(ys), np.inf)
    return c


def lamp_select(y_lo, tau, split: int = 256) -> np.ndarray:
    """The recompute decision: lamp_criterion_f32(y_lo) > tau (fp32)."""
    return lamp_criterion_f32(y_lo, split) > np.float32(tau)


def attention_decode_lamp(q, cache: KVCache, slot, length, softmax_scale, tau, split: int = 256,
                          return_selection=False, select=None):
    """Decode attention with LAMP selective recompute of the scores.

    Every score is first evaluated in low precision (lamp_low_precision_scores:
    binary16 accumulation of q16 . code, q16 = rn16(q)); the scores that
    lamp_select picks are recomputed in full precision, y_j = sigma q . K~_j
    (the definition, float64), the others keep y_lo.  The output is the
    softmax of these mixed scores over all keys times V~ (as attention_decode).
    With tau < 0 everything is recomputed (attention_decode itself).
    `select`, if given, replaces the decision: select[b] is a boolean [Hq, L]
    mask (for comparing other selection rules, or for evaluating a decision
    taken elsewhere)."""
    q32 = np.asarray(q, np.float32)
    q = f64(q32)
    q16_bits = enc.rn16_bits(q)
    B, Hq, D = q.shape
    Hkv = cache.k.shape[1]
    G = Hq // Hkv
    sigma = np.float32(softmax_scale)
    out = np.zeros((B, Hq, D), np.float64)
    selection = []
    for b in range(B):
        L = int(length[b])
        s = int(slot[b])
        Kt = enc.kv_dequant(cache.k[s, :, :L], cache.ks[s, :, :L])
        Vt = enc.kv_dequant(cache.v[s, :, :L], cache.vs[s, :, :L])
        sel_b = np.zeros((Hq, L), bool)
        y = np.zeros((Hq, L), np.float64)
        for h in range(Hq):
            kh = h // G
            y_lo = lamp_low_precision_scores(q16_bits[b, h], cache.k[s, kh, :L], cache.ks[s, kh, :L], sigma)
            y_hi = float(sigma) * (Kt[kh] @ q[b, h])
            sel = lamp_select(y_lo, tau, split) if select is None else np.asarray(select[b][h], bool)
            sel_b[h] = sel
            y[h] = np.where(sel, y_hi, y_lo.astype(np.float64))
        y = y - y.max(axis=-1, keepdims=True)
        p = np.exp(y)
        p = p / p.sum(axis=-1, keepdims=True)
        for h in range(Hq):
            out[b, h] = p[h] @ Vt[h // G]
        selection.append(sel_b)
    return (out, selection) if return_selection else out


# ----------------------------------------------------------------------------
# decode layer and layer stack (LLaMA-style block: RMSNorm -> GQA attention with
# rotary embedding over the INT16 cache -> residual -> RMSNorm -> SwiGLU MLP ->
# residual)
# ----------------------------------------------------------------------------

@dataclass
class LayerParams:
    wq: np.ndarray        # fp32 [H, Hq*D]
    wk: np.ndarray        # fp32 [H, Hkv*D]
    wv: np.ndarray        # fp32 [H, Hkv*D]
    wo: np.ndarray        # fp32 [Hq*D, H]
    w_gate: np.ndarray    # fp32 [H, F]
    w_up: np.ndarray      # fp32 [H, F]
    w_down: np.ndarray    # fp32 [F, H]
    g_attn: np.ndarray    # fp32 [H]
    g_mlp: np.ndarray     # fp32 [H]
    n_heads: int
    n_kv_heads: int
    head_dim: int
    eps: float = 1e-6
    rope_base: float = 10000.0


def silu(x) -> np.ndarray:
    x = f64(x)
    return x / (1.0 + np.exp(-x))


def decode_layer(p: LayerParams, cache: KVCache, x, slot, pos, softmax_scale=None,
                 return_intermediates=False):
    """One layer over B token rows; row b belongs to cache slot slot[b] at position
    pos[b].  The K/V of every row are quantised into the cache before any row
    attends, and row b attends over positions 0..pos[b] of its slot.  Returns the
    float64 output rows (and optionally the intermediates)."""
    x = f64(np.asarray(x, np.float32))
    B = x.shape[0]
    Hq, Hkv, D = p.n_heads, p.n_kv_heads, p.head_dim
    sigma = np.float32(1.0 / np.sqrt(D)) if softmax_scale is None else np.float32(softmax_scale)
    slot = np.asarray(slot, np.int64)
    pos = np.asarray(pos, np.int64)

    h = rmsnorm(x, p.g_attn, p.eps)
    q = (h @ f64(p.wq)).reshape(B, Hq, D)
    k = (h @ f64(p.wk)).reshape(B, Hkv, D)
    v = (h @ f64(p.wv)).reshape(B, Hkv, D)
    q = apply_rope(q, pos, p.rope_base)
    k = apply_rope(k, pos, p.rope_base)
    cache.write("k", k.astype(np.float32), slot, pos)
    cache.write("v", v.astype(np.float32), slot, pos)
    o = attention_decode(q, cache, slot, pos + 1, sigma).reshape(B, Hq * D)
    x1 = x + o @ f64(p.wo)
    h2 = rmsnorm(x1, p.g_mlp, p.eps)
    a = silu(h2 @ f64(p.w_gate)) * (h2 @ f64(p.w_up))
    out = x1 + a @ f64(p.w_down)
    if return_intermediates:
        return out, dict(h=h, q=q, k=k, v=v, o=o, x1=x1, h2=h2, a=a)
    return out


def decode_layer_at(p: LayerParams, cache: KVCache, x, slot, pos, rows, softmax_scale=None):
    """decode_layer evaluated at the chosen `rows` only.

    The K/V of EVERY input row are computed (RMSNorm, the K and V projections,
    rotary embedding of K) and quantised into the cache first, exactly as
    decode_layer does; the query, attention, output projection and MLP are
    then evaluated for the rows listed in `rows` alone.  Row r of the result
    is decode_layer's row rows[r] (same float64 operations on the same values;
    only the set of rows each product runs over differs).  Used for checks at
    sampled positions of long prompts, where the whole layer at every position
    would be too slow."""
    x = f64(np.asarray(x, np.float32))
    B = x.shape[0]
    Hq, Hkv, D = p.n_heads, p.n_kv_heads, p.head_dim
    sigma = np.float32(1.0 / np.sqrt(D)) if softmax_scale is None else np.float32(softmax_scale)
    slot = np.asarray(slot, np.int64)
    pos = np.asarray(pos, np.int64)
    rows = np.asarray(rows, np.int64)

    h = rmsnorm(x, p.g_attn, p.eps)
    k = apply_rope((h @ f64(p.wk)).reshape(B, Hkv, D), pos, p.rope_base)
    v = (h @ f64(p.wv)).reshape(B, Hkv, D)
    cache.write("k", k.astype(np.float32), slot, pos)
    cache.write("v", v.astype(np.float32), slot, pos)
    n = len(rows)
    q = apply_rope((h[rows] @ f64(p.wq)).reshape(n, Hq, D), pos[rows], p.rope_base)
    o = attention_decode(q, cache, slot[rows], pos[rows] + 1, sigma).reshape(n, Hq * D)
    x1 = x[rows] + o @ f64(p.wo)
    h2 = rmsnorm(x1, p.g_mlp, p.eps)
    a = silu(h2 @ f64(p.w_gate)) * (h2 @ f64(p.w_up))
    return x1 + a @ f64(p.w_down)


@dataclass
class StackParams:
    embed: np.ndarray      # fp32 [V, H]
    layers: list           # [LayerParams]
    g_final: np.ndarray    # fp32 [H]
    lm_head: np.ndarray    # fp32 [H, V]
    eps: float = 1e-6


def argmax_lowest(logits) -> np.ndarray:
    """Index of the maximum per row; ties go to the lowest index (np.argmax)."""
    return np.argmax(f64(logits), axis=-1).astype(np.int64)


def stack_forward(sp: StackParams, caches, tokens, slot, pos, return_hidden=False):
    """Token ids -> embedding -> every layer -> final RMSNorm -> LM head ->
    (logits, greedy ids).  Hidden states between layers are rounded to fp32,
    the container every inter-layer tensor uses."""
    x = np.asarray(sp.embed, np.float32)[np.asarray(tokens, np.int64)]
    hidden = []
    for li, lp in enumerate(sp.layers):
        x = decode_layer(lp, caches[li], x, slot, pos).astype(np.float32)
        hidden.append(x)
    hf = rmsnorm(x, sp.g_final, sp.eps)
    logits = hf @ f64(sp.lm_head)
    ids = argmax_lowest(logits)
    if return_hidden:
        return logits, ids, hidden
    return logits, ids
