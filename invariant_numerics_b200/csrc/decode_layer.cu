// decode_layer: one LLaMA-style block over B token rows, composed from the
// library's kernels and nothing else (stream-ordered, no host synchronisation).
//
// HEAL explainer, section "真の犯人（「カーネル境界」）": precision is lost at kernel
// boundaries when intermediates are stored in smaller containers.  Here every
// tensor crossing a kernel boundary is either fp32 or an exact binary16 hi/lo
// pair; the only lossy store is the INT16 KV cache the method prescribes.
#include "common.cuh"
#include "internal.h"

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct LayerWs {
  uint16_t *h_hi, *h_lo;
  float* q_rot;
  int32_t* lens;
  int32_t* rows_slot;  // prefill_layer: per-row slot / position arrays
  int32_t* rows_pos;
  void* attn;
  float* o;
  uint16_t *o_hi, *o_lo;
  float* x1;
  uint16_t *h2_hi, *h2_lo;
  uint16_t *a_hi, *a_lo;
  int* ready;          // gate/up tiles published to the down GEMM
  size_t bytes;
};

LayerWs carve(const inv_layer_config& c, int B, int mlb, uint8_t* base) {
  LayerWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    uint8_t* p = base ? base + off : nullptr;
    off += align256(n);
    return p;
  };
  const size_t H = c.hidden, F = c.ffn, QD = (size_t)c.n_heads * 128;
  w.h_hi = reinterpret_cast<uint16_t*>(take(B * H * 2));
  w.h_lo = reinterpret_cast<uint16_t*>(take(B * H * 2));
  w.q_rot = reinterpret_cast<float*>(take(B * QD * 4));
  w.lens = reinterpret_cast<int32_t*>(take(B * 4));
  w.rows_slot = reinterpret_cast<int32_t*>(take(B * 4));
  w.rows_pos = reinterpret_cast<int32_t*>(take(B * 4));
  w.attn = take(inv::attn_workspace_bytes(B, c.n_heads, mlb));
  w.o = reinterpret_cast<float*>(take(B * QD * 4));
  w.o_hi = reinterpret_cast<uint16_t*>(take(B * QD * 2));
  w.o_lo = reinterpret_cast<uint16_t*>(take(B * QD * 2));
  w.x1 = reinterpret_cast<float*>(take(B * H * 4));
  w.h2_hi = reinterpret_cast<uint16_t*>(take(B * H * 2));
  w.h2_lo = reinterpret_cast<uint16_t*>(take(B * H * 2));
  w.a_hi = reinterpret_cast<uint16_t*>(take(B * F * 2));
  w.a_lo = reinterpret_cast<uint16_t*>(take(B * F * 2));
  w.ready = reinterpret_cast<int*>(take(inv::gemm_ready_bytes(B, (int)(2 * F))));
  w.bytes = off;
  return w;
}

int validate(const inv_layer_config* cfg, const inv_kv_cache* cache) {
  if (!cfg || !cache) return INV_ERR_INVALID_ARG;
  if (cfg->head_dim != INV_HEAD_DIM || cache->head_dim != INV_HEAD_DIM) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cfg->hidden <= 0 || cfg->ffn <= 0 || cfg->n_heads <= 0 || cfg->n_kv_heads <= 0 || cfg->max_pos <= 0)
    return INV_ERR_INVALID_ARG;
  if (cfg->hidden % INV_GEMM_BN != 0 || cfg->ffn % 64 != 0) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cfg->n_heads % cfg->n_kv_heads != 0) return INV_ERR_UNSUPPORTED_SHAPE;
  const int G = cfg->n_heads / cfg->n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->n_kv_heads != cfg->n_kv_heads || cache->max_len <= 0 || cache->max_len % 64 != 0 ||
      cache->n_slots <= 0)
    return INV_ERR_INVALID_ARG;
  if ((uint64_t)cache->n_slots * cache->n_kv_heads * cache->max_len >= (1ull << 31)) return INV_ERR_UNSUPPORTED_SHAPE;
  return INV_OK;
}

int bound_of(const inv_kv_cache* cache, int max_len_bound) {
  return max_len_bound > 0 ? (max_len_bound < cache->max_len ? max_len_bound : cache->max_len) : cache->max_len;
}

__global__ void fill_rows_kernel(int32_t* slot_out, int32_t* pos_out, int T, int slot, int pos0) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    slot_out[t] = slot;
    pos_out[t] = pos0 + t;
  }
}

#define INV_TRY(expr)          \
  do {                         \
    const int rc_ = (expr);    \
    if (rc_ != INV_OK) return rc_; \
  } while (0)

// The layer's launches.  prefill_slot < 0: arbitrary rows (slot[b], pos[b]);
// otherwise rows are positions prefill_pos0 + b of the sequence in
// prefill_slot and the attention loads each split once for all of them.
int run_layer(const inv_layer_config* cfg, const inv_layer_weights* w, const inv_kv_cache* cache, const float* x_in,
              const int32_t* slot, const int32_t* pos, int B, int mlb, float* x_out, const LayerWs& ws,
              cudaStream_t s, int prefill_slot, int prefill_pos0) {
  const int H = cfg->hidden, F = cfg->ffn, Hq = cfg->n_heads, Hkv = cfg->n_kv_heads;
  const int QD = Hq * 128, NQKV = (Hq + 2 * Hkv) * 128;

  // Kernel i is bracketed by trace slots 2i and 2i+1 (inv_trace_events).
#define INV_TRACED(i, expr)         \
  do {                              \
    inv::trace_record(2 * (i), s);  \
    INV_TRY(expr);                  \
    inv::trace_record(2 * (i) + 1, s); \
  } while (0)
  // 1. h = rmsnorm(x) -> hi/lo
  INV_TRACED(0, inv::launch_rmsnorm(x_in, w->g_attn, B, H, cfg->eps, nullptr, ws.h_hi, ws.h_lo, s));
  // 2. [q | k | v] = h W_qkv with, in the GEMM's epilogue, the rotary
  //    embedding of q and k, k and v INT16-quantised into the cache, q to
  //    q_rot, len = pos + 1 (and the gate/up tile counters of this layer
  //    cleared; the previous layer has finished with them)
  {
    inv::AttnInputs ai;
    ai.slot = slot;
    ai.pos = pos;
    ai.rope_cos = w->rope_cos;
    ai.rope_sin = w->rope_sin;
    ai.max_pos = cfg->max_pos;
    ai.q_out = ws.q_rot;
    ai.Hq = Hq;
    ai.cache = *cache;
    ai.len_out = ws.lens;
    ai.zero_a = ws.ready;
    ai.n_a = (int64_t)(inv::gemm_ready_bytes(B, 2 * F) / 4);
    INV_TRACED(1, inv::launch_qkv_attn_inputs(ws.h_hi, ws.h_lo, B, H, H, w->w_qkv, w->e_qkv, NQKV, ai, s));
  }
  // 3-4. fixed-split attention + ordered combine -> o hi/lo (kernels 2 and 3)
  if (prefill_slot < 0) {
    INV_TRY(inv::launch_attention(ws.q_rot, B, Hq, *cache, slot, ws.lens, mlb, cfg->softmax_scale, ws.o, ws.o_hi,
                                  ws.o_lo, ws.attn, s, 2));
  } else {
    INV_TRY(inv::launch_attention_prefill(ws.q_rot, B, Hq, *cache, prefill_slot, prefill_pos0, ws.lens, mlb,
                                          cfg->softmax_scale, ws.o, ws.o_hi, ws.o_lo, ws.attn, s, 2));
  }
  // 5. x1 = x + o W_o
  INV_TRACED(4, inv::launch_comp_gemm(ws.o_hi, ws.o_lo, B, QD, QD, w->w_o, w->e_o, H, ws.x1, H, x_in, H, s));
  // 6. h2 = rmsnorm(x1) -> hi/lo
  INV_TRACED(5, inv::launch_rmsnorm(ws.x1, w->g_mlp, B, H, cfg->eps, nullptr, ws.h2_hi, ws.h2_lo, s));
  // 7. [gate | up] = h2 W_gu with the SwiGLU a = silu(gate) * up fused in the epilogue -> hi/lo
  // 8. out = x1 + a W_down.  The down GEMM starts while the gate/up GEMM's
  // last tiles (a partial wave) run, loading each 64-column K block of a as
  // soon as the gate/up tile that stores it has published it.
  INV_TRACED(6, inv::launch_comp_gemm_ex(ws.h2_hi, ws.h2_lo, B, H, H, w->w_gu, w->e_gu, 2 * F, nullptr, 0, nullptr, 0,
                                         ws.a_hi, ws.a_lo, F, ws.ready, nullptr, s));
  INV_TRACED(7, inv::launch_comp_gemm_ex(ws.a_hi, ws.a_lo, B, F, F, w->w_down, w->e_down, H, x_out, H, ws.x1, H,
                                         nullptr, nullptr, 0, nullptr, ws.ready, s));
#undef INV_TRACED
  return INV_OK;
}

}  // namespace

extern "C" {

size_t decode_layer_workspace_size(const inv_layer_config* cfg, int B, int max_len_bound) {
  // The bound must be the one the call resolves to (a positive bound, or the
  // cache's max_len when the call passes <= 0); <= 0 here has no size.
  if (!cfg || B <= 0 || max_len_bound <= 0 || cfg->hidden <= 0 || cfg->ffn <= 0 || cfg->n_heads <= 0 ||
      cfg->n_kv_heads <= 0)
    return 0;
  return carve(*cfg, B, max_len_bound, nullptr).bytes;
}

int decode_layer(const inv_layer_config* cfg, const inv_layer_weights* w, const inv_kv_cache* cache,
                 const float* x_in, const int32_t* slot, const int32_t* pos, int B, int max_len_bound, float* x_out,
                 void* workspace, size_t ws_bytes, inv_stream stream) {
  INV_TRY(validate(cfg, cache));
  if (!w || B < 0) return INV_ERR_INVALID_ARG;
  if (B == 0) return INV_OK;
  if (B > 65535) return INV_ERR_UNSUPPORTED_SHAPE;
  if (!x_in || !x_out || !slot || !pos || !workspace || x_in == x_out) return INV_ERR_INVALID_ARG;
  if (!w->w_qkv || !w->e_qkv || !w->w_o || !w->e_o || !w->w_gu || !w->e_gu || !w->w_down || !w->e_down ||
      !w->g_attn || !w->g_mlp || !w->rope_cos || !w->rope_sin)
    return INV_ERR_INVALID_ARG;
  if (!cache->k || !cache->v || !cache->k_scale || !cache->v_scale) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(x_in) || !inv::aligned16(x_out) || !inv::aligned16(workspace) || !inv::aligned16(w->rope_cos) ||
      !inv::aligned16(w->rope_sin) || !inv::aligned16(w->g_attn) || !inv::aligned16(w->g_mlp) ||
      !inv::aligned16(cache->k) || !inv::aligned16(cache->v))
    return INV_ERR_INVALID_ARG;
  const int mlb = bound_of(cache, max_len_bound);
  const LayerWs ws = carve(*cfg, B, mlb, static_cast<uint8_t*>(workspace));
  if (ws_bytes < ws.bytes) return INV_ERR_WORKSPACE;

  return run_layer(cfg, w, cache, x_in, slot, pos, B, mlb, x_out, ws, static_cast<cudaStream_t>(stream), -1, 0);
}

size_t prefill_layer_workspace_size(const inv_layer_config* cfg, int T, int max_len_bound) {
  return decode_layer_workspace_size(cfg, T, max_len_bound);
}

int prefill_layer(const inv_layer_config* cfg, const inv_layer_weights* w, const inv_kv_cache* cache,
                  const float* x_in, int slot, int pos0, int T, int max_len_bound, float* x_out, void* workspace,
                  size_t ws_bytes, inv_stream stream) {
  INV_TRY(validate(cfg, cache));
  if (!w || T < 0 || slot < 0 || slot >= cache->n_slots || pos0 < 0) return INV_ERR_INVALID_ARG;
  if (T == 0) return INV_OK;
  if (T > 65535) return INV_ERR_UNSUPPORTED_SHAPE;
  if (!x_in || !x_out || !workspace || x_in == x_out) return INV_ERR_INVALID_ARG;
  if (!w->w_qkv || !w->e_qkv || !w->w_o || !w->e_o || !w->w_gu || !w->e_gu || !w->w_down || !w->e_down ||
      !w->g_attn || !w->g_mlp || !w->rope_cos || !w->rope_sin)
    return INV_ERR_INVALID_ARG;
  if (!cache->k || !cache->v || !cache->k_scale || !cache->v_scale) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(x_in) || !inv::aligned16(x_out) || !inv::aligned16(workspace) || !inv::aligned16(w->rope_cos) ||
      !inv::aligned16(w->rope_sin) || !inv::aligned16(w->g_attn) || !inv::aligned16(w->g_mlp) ||
      !inv::aligned16(cache->k) || !inv::aligned16(cache->v))
    return INV_ERR_INVALID_ARG;
  const int mlb = bound_of(cache, max_len_bound);
  if ((int64_t)pos0 + T > mlb || (int64_t)pos0 + T > cfg->max_pos) return INV_ERR_INVALID_ARG;
  const LayerWs ws = carve(*cfg, T, mlb, static_cast<uint8_t*>(workspace));
  if (ws_bytes < ws.bytes) return INV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fill_rows_kernel<<<(T + 255) / 256, 256, 0, s>>>(ws.rows_slot, ws.rows_pos, T, slot, pos0);
  INV_CHECK_LAUNCH();
  return run_layer(cfg, w, cache, x_in, ws.rows_slot, ws.rows_pos, T, mlb, x_out, ws, s, slot, pos0);
}

}  // extern "C"
