// Internal launchers shared between translation units (no validation: the
// public entry points and decode_layer validate before calling these).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "invnum.h"

namespace inv {

int launch_rmsnorm(const float* x, const float* gamma, int64_t rows, int hidden, float eps, float* y,
                   uint16_t* yh, uint16_t* yl, cudaStream_t s);

// Where the QKV GEMM's epilogue puts the attention inputs of its M rows
// (row t at position pos[t] of sequence slot[t]): query heads rotated into
// q_out [M][Hq][128], key heads rotated and value heads as they are,
// INT16-quantised into the cache; len_out[t] = pos[t] + 1 (0 and
// INV_ERR_INVALID_ARG for a slot or position out of range, whose row is then
// skipped).  zero_a[0 .. n_a) is cleared on the way (counters a later kernel
// of the layer needs zero; may be null).  q_out == nullptr: no fusion.
struct AttnInputs {
  const int32_t* slot = nullptr;
  const int32_t* pos = nullptr;
  const float* rope_cos = nullptr;  // [max_pos][64]
  const float* rope_sin = nullptr;
  int max_pos = 0;
  float* q_out = nullptr;
  int Hq = 0;
  inv_kv_cache cache = {};
  int32_t* len_out = nullptr;
  int* zero_a = nullptr;
  int64_t n_a = 0;
};


// Panel width (output columns per GEMM tile and per packed panel) of a weight
// with N output columns: a function of N alone, so every M uses the same tile.
int gemm_panel_width(int N);

int launch_comp_gemm(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                     const uint16_t* w_packed, const int8_t* col_exp, int N, float* y, int64_t ld_y,
                     const float* residual, int64_t ld_r, cudaStream_t s);

// comp_gemm with the fused SwiGLU epilogue: the packed weight holds gate/up
// columns interleaved in groups of 16 ([gate 16 | up 16] per 32 columns);
// writes the hi/lo split of silu(gate) * up to gate_hi/gate_lo [M][ld_g]
// (N/2 outputs per row) instead of y.
// Producer/consumer pair (both nullable): a producer given ready_out
// ([tiles_m][N/128] ints, zero before the launch) adds 1 per epilogue warp to
// ready_out[mt][nt] once that warp has stored its part of tile (mt, nt); a
// consumer given ready_in (the producer's array; the producer's N/128 must
// equal the consumer's K/64) is launched as a programmatic dependent of the
// producer launched just before it on the same stream and loads K block kb of
// row tile mt only once ready_in[mt][kb] is complete.  Neither changes the
// arithmetic.  wait_ns < 0: the library-wide wait bound.
int launch_comp_gemm_ex(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                        const uint16_t* w_packed, const int8_t* col_exp, int N, float* y, int64_t ld_y,
                        const float* residual, int64_t ld_r, uint16_t* gate_hi, uint16_t* gate_lo, int64_t ld_g,
                        int* ready_out, const int* ready_in, cudaStream_t s, long long wait_ns = -1);
// The QKV projection with the rotary embedding and the KV quantiser in its
// epilogue (one 128-wide head per tile; N = (Hq + 2 Hkv) 128): writes the
// attention inputs described by `ai` instead of the GEMM's output.
int launch_qkv_attn_inputs(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                           const uint16_t* w_packed, const int8_t* col_exp, int N, const AttnInputs& ai,
                           cudaStream_t s);
// Bytes of the ready array of a producer GEMM with M rows and N columns.
inline size_t gemm_ready_bytes(int64_t M, int N) { return (size_t)((M + 127) / 128) * (size_t)(N / 128) * 4; }

// Workspace layout of the attention: partial o and partial (m, l) per
// (row, head, split).
size_t attn_workspace_bytes(int B, int Hq, int max_len_bound);
// Decode attention: split kernel, then the ascending fold of each row's
// splits (combine kernel).  trace_base < 0: no tracing.
int launch_attention(const float* q, int B, int Hq, const inv_kv_cache& c, const int32_t* slot, const int32_t* len,
                     int max_len_bound, float sigma, float* out, uint16_t* out_hi, uint16_t* out_lo, void* ws,
                     cudaStream_t s, int trace_base);

// Prefill form: rows t = 0..T-1 are consecutive positions pos0 + t of the
// sequence in `slot`; each split's K/V is loaded once for all rows that reach
// it, and every (row, split) runs the decode kernel's per-row code.
int launch_attention_prefill(const float* q, int T, int Hq, const inv_kv_cache& c, int slot, int pos0,
                             const int32_t* len, int max_len_bound, float sigma, float* out, uint16_t* out_hi,
                             uint16_t* out_lo, void* ws, cudaStream_t s, int trace_base);

}  // namespace inv
