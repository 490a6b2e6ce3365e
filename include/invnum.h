/*
 * invnum.h -- C ABI of libinvnum.so, a batch-invariant, error-compensated
 * transformer decode step for NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow:
 *   [HEAL] "Demystifying Numerical Instability in LLM Inference: Achieving
 *          Reproducible Inference for Mission-Critical Tasks with HEAL"
 *          (gist.science explainer of arXiv 2606.21023), sections
 *          "1. 「スマート・パッキング」のトリック（アテンション用）" (INT16 K/V,
 *          dual-FP16 unpack) and "2. 「誤差補償」のトリック（計算用）" (main
 *          product plus clean-up product on 16-bit units).
 *   [BI]   Blog summary of Thinking Machines Lab, "Defeating Nondeterminism in
 *          LLM Inference", sections "バッチ不変性とは何か？" (definition of
 *          batch invariance) and "解決へのアプローチ：3種の主要演算の再設計"
 *          (table rows RMSNorm, MatMul, Attention).
 *
 * Conventions (all entry points)
 *   - Every pointer is caller-owned DEVICE memory unless stated otherwise; the
 *     library never allocates or frees memory.  Its only global state is one
 *     device status word per GPU (see inv_get_device_status).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work and return without synchronising.
 *   - Return value: INV_OK after a successful enqueue; otherwise an inv_status
 *     code from host-side validation, in which case NOTHING was launched.
 *   - Errors found on the device (binary16 overflow in a split, an index out
 *     of range, a bounded wait that expired) are recorded in the status word.
 *   - fp16 buffers are IEEE binary16 bit patterns stored as uint16_t.
 *   - Batch invariance [BI]: every result row depends only on that row's own
 *     inputs (and, for attention, its own cache slot and length), never on how
 *     many rows are in the call, which other rows are present, or where a row
 *     sits in the batch.  Tile shapes, reduction orders and the KV split size
 *     are compile-time constants, not functions of the call's shape.
 *   - Inputs are assumed finite; non-finite inputs give unspecified values but
 *     never a hang or a fault.
 */
#ifndef INVNUM_H
#define INVNUM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define INV_API __attribute__((visibility("default")))
#else
#define INV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  INV_OK = 0,
  INV_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad index, misalignment */
  INV_ERR_UNSUPPORTED_SHAPE = 2, /* a dimension the fixed kernel configuration cannot take */
  INV_ERR_WORKSPACE = 3,         /* workspace or output buffer smaller than required */
  INV_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
  INV_ERR_RANGE = 5,             /* a value outside the binary16 range (|x| >= 65520) was split */
  INV_ERR_TIMEOUT = 6,           /* a bounded wait inside a kernel expired */
  INV_ERR_BOUNDS = 7             /* a kernel computed an index outside the buffer its caller
                                    passed (recorded by the INV_DEBUG_BOUNDS build only) */
} inv_status;

/* Fixed algorithm constants (part of the numerics; not tunable). */
#define INV_KV_SPLIT 256        /* keys per attention split, at absolute positions 256*s */
#define INV_GEMM_BM 128         /* rows per compensated-GEMM tile */
#define INV_GEMM_BN 128         /* output columns per tile (= packed panel width) */
#define INV_GEMM_BK 64          /* K per pipeline stage; K must be a multiple of it */
#define INV_GEMM_KGROUP 256     /* K per tensor-memory accumulation group */
#define INV_HEAD_DIM 128        /* the only supported attention head size */

typedef void* inv_stream;

/* Human-readable name of a status code (static string, never NULL). */
INV_API const char* inv_status_string(int status);

/* Library ABI version (increments on incompatible change). */
INV_API int inv_version(void);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  *status_out receives INV_OK or the first device-side error recorded
 * since the last call.  Returns INV_ERR_CUDA if the synchronisation or copy
 * fails (e.g. a sticky context error), else INV_OK.
 */
INV_API int inv_get_device_status(int* status_out, inv_stream stream);

/*
 * Upper bound, in nanoseconds of GPU global time, on every barrier wait inside
 * the library's kernels (default 2e9).  A wait that exceeds it records
 * INV_ERR_TIMEOUT, releases what the kernel holds and returns.  Values <= 0
 * restore the default.  Host-global setting, read at each launch.
 */
INV_API int inv_set_wait_limit_ns(long long ns);

/*
 * Self-test of the bounded-wait path: launches one CTA that waits on a
 * shared-memory barrier nothing ever arrives at, with a limit of `wait_ns`
 * nanoseconds.  The kernel must give up, record INV_ERR_TIMEOUT in the status
 * word and exit; no GPU state is left behind.  For failure-detection tests.
 */
INV_API int inv_selftest_wait_timeout(long long wait_ns, inv_stream stream);

/*
 * Self-test of the bounded wait of a GEMM consumer (the W_down GEMM of
 * decode_layer waits on per-tile counters of the gate/up GEMM): launches a
 * small consumer GEMM whose one input block is never published, with a limit
 * of `wait_ns` nanoseconds.  It must give up, record INV_ERR_TIMEOUT and exit.
 * `workspace`: >= INV_SELFTEST_GEMM_WS_BYTES of caller device memory, 16-byte
 * aligned (cleared and used for the operands).  For failure-detection tests.
 * Errors: INV_ERR_INVALID_ARG (wait_ns <= 0, null or misaligned workspace),
 * INV_ERR_WORKSPACE.
 */
#define INV_SELFTEST_GEMM_WS_BYTES 40192u
INV_API int inv_selftest_gemm_wait_timeout(void* workspace, size_t ws_bytes, long long wait_ns,
                                           inv_stream stream);

/*
 * Index checks.  A library built with -DINV_DEBUG_BOUNDS (build option
 * --debug-bounds, file libinvnum_debug.so) checks, in every kernel, each
 * global-memory index it computes -- or, for a contiguous or strided block it
 * accesses as a whole (a TMA tile, a split's scales, a row's partials), the
 * block's first and last index -- against the extent of the buffer the
 * caller passed, as stated by that call's contract.  An index outside it
 * records INV_ERR_BOUNDS in the status word and the access is skipped (a
 * block is skipped whole, before any of its loads is issued).  The normal
 * build compiles the checks out.
 * inv_debug_bounds_enabled: 1 in the checking build, 0 otherwise.
 * inv_selftest_bounds: self-test of the check itself.  A kernel stores the
 * value i to buf[i] for i = 0 .. n_written-1 while declaring the extent
 * n_declared <= n_written (buf must hold n_declared floats): the stores
 * i >= n_declared fail the check, are skipped and INV_ERR_BOUNDS is recorded.
 * Errors: INV_ERR_UNSUPPORTED_SHAPE in the normal build (nothing launched, as
 * the unchecked stores would leave the buffer); INV_ERR_INVALID_ARG for a null
 * buf, n_declared < 0 or n_written < n_declared.
 */
INV_API int inv_debug_bounds_enabled(void);
INV_API int inv_selftest_bounds(float* buf, int n_declared, int n_written, inv_stream stream);

/*
 * Kernel tracing for decode_layer (profiling aid; off by default).  With
 * events != NULL and n_events >= 2 * INV_DECODE_LAYER_KERNELS, every later
 * decode_layer call records events[2i] before and events[2i+1] after its i-th
 * kernel launch, on the call's stream (i: 0 rmsnorm, 1 qkv GEMM with the
 * rotary embedding and the KV quantiser in its epilogue, 2 attention splits,
 * 3 attention combine, 4 output GEMM, 5 rmsnorm, 6 gate/up GEMM with fused
 * SwiGLU, 7 down GEMM).  events are cudaEvent_t handles the caller created
 * and keeps alive.  NULL / 0 switches tracing off.  Host-global.
 */
#define INV_DECODE_LAYER_KERNELS 8
INV_API int inv_trace_events(void** events, int n_events);

/* ------------------------------------------------------------------------
 * heal_split -- [HEAL] section 2: split fp32 activations into the binary16
 * (hi, lo) pair used by the compensated product:
 *     hi = rn16(x),   lo = rn16((x - hi) * 2^11)     (round half to even)
 * so that x ~= hi + 2^-11 lo with |error| <= 2^-22 |x| for 2^-14 <= |x| < 65520.
 *   x   : fp32 [rows][ld_x], first `cols` entries of each row used.
 *   hi, lo : binary16 [rows][ld_out].
 * Errors: INV_ERR_INVALID_ARG (null, negative sizes, ld < cols);
 *         device status INV_ERR_RANGE when some |x| >= 65520.
 * ------------------------------------------------------------------------ */
INV_API int heal_split(const float* x, int64_t rows, int64_t cols, int64_t ld_x,
               uint16_t* hi, uint16_t* lo, int64_t ld_out, inv_stream stream);

/* ------------------------------------------------------------------------
 * heal_pack_weight -- offline, once per weight: [HEAL] section 2 applied to a
 * weight matrix W fp32 [K][N] (row-major, y = x W).  For every output column
 * n a static exponent e_n makes max_k |W[k][n]| 2^e_n fall in [2^14, 2^15)
 * (0 for an all-zero column; clamped to [-120, 120]); then W 2^e_n is split
 * like heal_split.  The packed image is binary16 [N/128][2][128][K]: panel j
 * holds the hi rows of its 128 columns, then their lo rows, each contiguous in
 * K.  Needs heal_packed_weight_bytes(K, N) bytes at `packed`; col_exp is int8 [N].
 * Errors: INV_ERR_INVALID_ARG; INV_ERR_UNSUPPORTED_SHAPE unless K % 64 == 0
 * and N % 128 == 0; INV_ERR_WORKSPACE if packed_bytes is too small.
 * ------------------------------------------------------------------------ */
INV_API size_t heal_packed_weight_bytes(int K, int N);
INV_API int heal_pack_weight(const float* W, int K, int N, uint16_t* packed, size_t packed_bytes,
                     int8_t* col_exp, inv_stream stream);

/* ------------------------------------------------------------------------
 * comp_gemm -- [HEAL] section 2 error-compensated GEMM on 16-bit tensor cores,
 * batch-invariant per [BI] table row "MatMul" (one tile, one K order, no
 * split-K, for every M):
 *   y[m][n] = ((sum_k hh) + 2^-11 (sum_k cross)) * 2^-e_n  (+ residual[m][n])
 *   hh    = a_hi[m][k] * w_hi[k][n]
 *   cross = a_hi[m][k] * w_lo[k][n] + a_lo[m][k] * w_hi[k][n]
 * with fp32 accumulation.  K is consumed in ascending 64-wide blocks; each
 * group of 256 K values accumulates in tensor memory and groups are added in
 * ascending order with fp32 round-to-nearest adds.
 *   a_hi, a_lo : binary16 [M][ld_a] (from heal_split or a fused producer);
 *                ld_a % 8 == 0 and both base pointers 16-byte aligned.
 *   w_packed, col_exp : from heal_pack_weight for this K, N.
 *   y          : fp32 [M][ld_y].   residual : fp32 [M][ld_r] or NULL.
 *                y may alias residual exactly (same pointer and ld).
 * Errors: INV_ERR_INVALID_ARG; INV_ERR_UNSUPPORTED_SHAPE unless K % 64 == 0,
 * N % 128 == 0, K >= 64; M == 0 is a no-op.  Device: INV_ERR_TIMEOUT.
 * ------------------------------------------------------------------------ */
INV_API int comp_gemm(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
              const uint16_t* w_packed, const int8_t* col_exp, int N,
              float* y, int64_t ld_y, const float* residual, int64_t ld_r, inv_stream stream);

/* ------------------------------------------------------------------------
 * INT16 KV cache ([HEAL] section 1).  Layout: codes int16
 * [n_slots][n_kv_heads][max_len][head_dim], scales fp32
 * [n_slots][n_kv_heads][max_len], separately for K and V.  A sequence owns a
 * slot; its token at position p lives at [slot][h][p].  max_len % 64 == 0.
 * ------------------------------------------------------------------------ */
typedef struct {
  int16_t* k;
  int16_t* v;
  float* k_scale;
  float* v_scale;
  int n_slots;
  int n_kv_heads;
  int max_len;
  int head_dim;
} inv_kv_cache;

/*
 * kv_quant_int16 -- quantise fp32 x[T][ld_x] (token t's heads at
 * x[t*ld_x + h*head_dim + d]) into the cache at (slot[t], h, pos[t]):
 *   s = fl32(max_d |x_d| / 32767),  q_d = clamp(rint_even(fl32(x_d / s)), +-32767)
 * with IEEE fp32 division; max == 0 (or s underflowing to 0) stores s = 0, q = 0.
 * which: 0 = K, 1 = V.  slot/pos: int32 [T] device arrays.
 * Errors: INV_ERR_INVALID_ARG; INV_ERR_UNSUPPORTED_SHAPE unless head_dim == 128.
 * Device: INV_ERR_INVALID_ARG for a slot/pos out of range (that token is skipped).
 */
INV_API int kv_quant_int16(const float* x, int T, int64_t ld_x, const int32_t* slot, const int32_t* pos,
                   const inv_kv_cache* cache, int which, inv_stream stream);

/*
 * attn_decode_fixedsplit -- decode attention over the INT16 cache, one query
 * row per sequence ([BI] table row "Attention": unified cache layout and
 * fixed-size splits; [HEAL] section 1: codes unpacked to dual-FP16).
 * For row b, query head h (kv head h / (n_heads / n_kv_heads)) and the keys
 * 0..len[b]-1 of slot[b]:
 *   out = sum_j softmax_j(sigma * q . K~_j) V~_j,  K~_j = s_K,j * code_j.
 * Keys are processed in splits of INV_KV_SPLIT at absolute positions 256*s;
 * each split forms its scores with 16-bit tensor-core products of the
 * dual-FP16 unpacked codes (code = 256 h + l, both exact in binary16) and the
 * hi/lo split of q, its own max, exp-sum and value sum; the splits are then
 * folded in ascending s.  Nothing depends on other rows or on len beyond the
 * row's own split count.  Two kernels on `stream`: the split kernel, then the
 * ordered combine as its programmatic dependent.
 *   q        : fp32 [B][n_heads][128], 16-byte aligned.
 *   len      : int32 [B], 1 <= len[b] <= cache->max_len.
 *   max_len_bound : host upper bound on every len[b] (<= 0: cache->max_len);
 *                   only sizes the launch grid.
 *   split    : must equal INV_KV_SPLIT.
 *   out      : fp32 [B][n_heads][128]; out_hi/out_lo: binary16 split of out
 *              (both NULL or both non-NULL).
 *   workspace: >= attn_decode_workspace_size(B, n_heads, L) bytes, where L is
 *              the bound the call resolves to: min(max_len_bound,
 *              cache->max_len), or cache->max_len when max_len_bound <= 0.
 *              The size function itself needs L > 0 (it returns 0 otherwise).
 * Errors: INV_ERR_INVALID_ARG; INV_ERR_UNSUPPORTED_SHAPE unless head_dim == 128
 * and n_heads / n_kv_heads is 1, 2 or 4; INV_ERR_WORKSPACE.
 * Device: INV_ERR_INVALID_ARG for a len/slot out of range (row skipped),
 * INV_ERR_TIMEOUT, INV_ERR_RANGE (out split overflow).
 */
INV_API size_t attn_decode_workspace_size(int B, int n_heads, int max_len_bound);
INV_API int attn_decode_fixedsplit(const float* q, int B, int n_heads, const inv_kv_cache* cache,
                           const int32_t* slot, const int32_t* len, int max_len_bound, int split,
                           float softmax_scale, float* out, uint16_t* out_hi, uint16_t* out_lo,
                           void* workspace, size_t ws_bytes, inv_stream stream);

/*
 * attn_decode_fixedsplit_noalloc -- the same attention, numerically identical,
 * for callers that cannot allocate device memory or pass a workspace (an
 * embedding application that owns the whole device-memory budget, a plug-in
 * without an allocator, a latency-critical path where an allocation may
 * synchronise the device).  No counterpart on the pages: it is an interface
 * variant only.  The split partials live in a file-scope device array of
 * INV_NOALLOC_SCRATCH_BYTES on every GPU that loads the library, held until
 * exit.  Calls needing more than that return INV_ERR_WORKSPACE and launch
 * nothing: the test is attn_decode_workspace_size(B, n_heads, L) >
 * INV_NOALLOC_SCRATCH_BYTES with the resolved bound L = min(max_len_bound,
 * cache->max_len), or L = cache->max_len when max_len_bound <= 0.  The first call on a device looks the array's address up
 * (with that device current); make it before any stream capture.  All calls on
 * a device share the array, so calls that overlap on the GPU race; calls
 * ordered on one stream do not.  Allocates nothing; arguments and other errors
 * as attn_decode_fixedsplit.
 */
#define INV_NOALLOC_SCRATCH_BYTES (34u << 20)
INV_API int attn_decode_fixedsplit_noalloc(const float* q, int B, int n_heads, const inv_kv_cache* cache,
                                           const int32_t* slot, const int32_t* len, int max_len_bound, int split,
                                           float softmax_scale, float* out, uint16_t* out_hi, uint16_t* out_lo,
                                           inv_stream stream);

/*
 * attn_decode_lamp -- attn_decode_fixedsplit with LAMP-style selective
 * recompute of the scores (LAMP summary, gist.science: section "Fondement
 * théorique", item 3, the softmax condition 2 z_j (1 - z_j) |y_j| > tau for
 * recomputing a KQ product; section "Stratégie d'implémentation", evaluate in
 * low precision, select, recompute the selected in high precision; the
 * relaxed threshold of "Résultats expérimentaux", free of the softmax
 * normalisation).  Opt-in precision variant; its results are NOT those of
 * attn_decode_fixedsplit.  Per (row, query head, key j):
 *   low precision : y_lo_j from binary16 accumulation of q16 . code_j, q16 =
 *                   rn16(q): with code = 256 h + l, two binary16 accumulators
 *                   a_h <- rn16(q16_d h + a_h), a_l <- rn16(q16_d (l/256) + a_l)
 *                   over d = 0..127 in order (one rounding per multiply-add),
 *                   then in fp32 y_lo = ((256 a_h + 256 a_l) s_K,j) sigma;
 *   decision      : recompute iff y_lo_j is not finite or
 *                   (2 fl32(exp(y_lo_j - m_s))) |y_lo_j| > tau (fp32), m_s the
 *                   largest finite y_lo of the key's 256-key split -- an upper
 *                   bound of the strict criterion, evaluated per split;
 *   score         : recomputed keys take the full-precision score of
 *                   attn_decode_fixedsplit, the others keep y_lo; the softmax,
 *                   values and split fold are attn_decode_fixedsplit's.
 * The decision depends only on the row's own keys and split boundaries, so the
 * variant is batch-invariant like the plain call.
 *   tau        : threshold (not NaN); tau < 0 recomputes every score.
 *   recompute  : uint8 [B][n_heads][recompute_ld] or NULL; byte (b, h, j) of
 *                every key j < len[b] is set to 1 if its score was recomputed,
 *                else 0 (bytes past len[b] are not written).  recompute_ld >=
 *                the resolved length bound.
 *   other arguments and errors as attn_decode_fixedsplit (same workspace size).
 */
INV_API int attn_decode_lamp(const float* q, int B, int n_heads, const inv_kv_cache* cache, const int32_t* slot,
                             const int32_t* len, int max_len_bound, int split, float softmax_scale, float tau,
                             float* out, uint16_t* out_hi, uint16_t* out_lo, uint8_t* recompute,
                             int64_t recompute_ld, void* workspace, size_t ws_bytes, inv_stream stream);

/* ------------------------------------------------------------------------
 * rmsnorm_bi -- [BI] table row "RMSNorm": always the data-parallel strategy,
 * one CTA per row and one fixed reduction order per row:
 *   r = 1 / sqrt(sum_i x_i^2 / hidden + eps),   y_i = (x_i r) gamma_i
 * Thread t of 256 accumulates the float4 chunks i4 = t, t+256, ... in
 * ascending order (x.x, x.y, x.z, x.w within a chunk, fused multiply-adds),
 * then a fixed xor-shuffle tree inside each warp, then warps 0..7 in order.
 *   x : fp32 [rows][hidden];  gamma : fp32 [hidden];  hidden % 4 == 0.
 *   y : fp32 [rows][hidden] or NULL;  y_hi, y_lo : binary16 [rows][hidden]
 *       (both NULL or both non-NULL), the heal_split of y.
 * Errors: INV_ERR_INVALID_ARG; INV_ERR_UNSUPPORTED_SHAPE if hidden % 4 != 0.
 * ------------------------------------------------------------------------ */
INV_API int rmsnorm_bi(const float* x, const float* gamma, int64_t rows, int hidden, float eps,
               float* y, uint16_t* y_hi, uint16_t* y_lo, inv_stream stream);

/* ------------------------------------------------------------------------
 * decode_layer -- one LLaMA-style block over B token rows, every step a
 * library kernel ([HEAL] section 2 compensated GEMMs, [HEAL] section 1 INT16
 * cache, [BI] batch-invariant RMSNorm / MatMul / Attention):
 *   h  = rmsnorm_bi(x, g_attn)                       -> hi/lo
 *   qkv = comp_gemm(h, W_qkv)                         (N = (Hq + 2 Hkv) 128)
 *   q, k <- rotary embedding (rotate-half, pairs (i, i+64), tables below)
 *   k, v -> kv_quant_int16 into (slot[b], pos[b])     (all rows before any attention)
 *        (these three run as one kernel: the GEMM's epilogue rotates and
 *        quantises each 128-wide head tile in fp32, the same operations in
 *        the same order as the separate steps)
 *   o  = attn_decode_fixedsplit(q, len = pos + 1)    -> hi/lo
 *   x1 = x + comp_gemm(o, W_o)
 *   h2 = rmsnorm_bi(x1, g_mlp)                       -> hi/lo
 *   a  = silu(gate) * up, gate/up = h2 W_gu: one comp_gemm over N = 2 F whose
 *        epilogue applies silu(g) * u = g / (1 + exp(-g)) * u  -> hi/lo
 *   out = x1 + comp_gemm(a, W_down)
 * Rows of one sequence at consecutive positions (a prefill chunk) are legal:
 * every row's K/V is in the cache before any row attends.
 *   x_in, x_out : fp32 [B][hidden] (may not alias).
 *   slot, pos   : int32 [B]; 0 <= pos[b] < min(cache->max_len, cfg->max_pos).
 *   rope_cos, rope_sin : fp32 [max_pos][64], cos/sin(p * base^(-2i/128)).
 *   workspace   : >= decode_layer_workspace_size(cfg, B, L) bytes, L the
 *                 resolved bound: min(max_len_bound, cache->max_len), or
 *                 cache->max_len when max_len_bound <= 0 (the size function
 *                 returns 0 for L <= 0).  Calls that overlap on the GPU need
 *                 separate workspaces.
 * Stream work: the layer's kernels only, all on `stream` (the QKV GEMM also
 * clears the workspace's gate/up tile counters).  The W_down GEMM is launched
 * as a programmatic dependent of the gate/up GEMM and starts during its last
 * partial wave, loading each K block of a once the gate/up tile that stores it
 * has published it (no change to any product or sum).  The attention combine
 * is a programmatic dependent of the split kernel and waits for that grid
 * before its first load.  All of this may be captured into a CUDA graph.
 * Errors: as the component calls; INV_ERR_WORKSPACE.
 * ------------------------------------------------------------------------ */
typedef struct {
  int hidden;          /* H, multiple of 128 */
  int n_heads;         /* Hq */
  int n_kv_heads;      /* Hkv; Hq / Hkv in {1, 2, 4} */
  int head_dim;        /* must be 128 */
  int ffn;             /* F, multiple of 64 */
  int max_pos;         /* rows of the rotary tables */
  float eps;           /* RMSNorm epsilon */
  float softmax_scale; /* sigma, e.g. fl32(1/sqrt(128)) */
} inv_layer_config;

typedef struct {
  const uint16_t* w_qkv;  const int8_t* e_qkv;   /* packed [H x (Hq+2Hkv)128] */
  const uint16_t* w_o;    const int8_t* e_o;     /* packed [Hq 128 x H] */
  const uint16_t* w_gu;   const int8_t* e_gu;    /* packed [H x 2F], columns interleaved in
                                                    groups of 16: for j < F/32, h in {0, 1}:
                                                    gate 32j+16h .. +15, then up 32j+16h .. +15 */
  const uint16_t* w_down; const int8_t* e_down;  /* packed [F x H] */
  const float* g_attn;    /* [H] */
  const float* g_mlp;     /* [H] */
  const float* rope_cos;  /* [max_pos][64] */
  const float* rope_sin;  /* [max_pos][64] */
} inv_layer_weights;

INV_API size_t decode_layer_workspace_size(const inv_layer_config* cfg, int B, int max_len_bound);
INV_API int decode_layer(const inv_layer_config* cfg, const inv_layer_weights* w, const inv_kv_cache* cache,
                 const float* x_in, const int32_t* slot, const int32_t* pos, int B, int max_len_bound,
                 float* x_out, void* workspace, size_t ws_bytes, inv_stream stream);

/* ------------------------------------------------------------------------
 * prefill_layer -- decode_layer for T rows that are consecutive positions
 * pos0 .. pos0+T-1 of the one sequence in `slot` (a prefill chunk).  Same
 * steps and same per-row arithmetic as decode_layer; the attention loads each
 * 256-key split once for every row that reaches it and runs the decode
 * kernel's per-row code on it, so every output row (and the cache) is
 * bit-identical to decode_layer on the same rows ([BI] table row "Attention":
 * chunked prefill and decode must not change a row's reduction).
 *   x_in, x_out : fp32 [T][hidden].  0 <= slot < n_slots; 0 <= pos0;
 *   pos0 + T <= min(max_len_bound (or cache->max_len), cfg->max_pos).
 *   workspace : >= prefill_layer_workspace_size(cfg, T, L) bytes, L resolved
 *               as for decode_layer.
 * Errors: as decode_layer.
 * ------------------------------------------------------------------------ */
INV_API size_t prefill_layer_workspace_size(const inv_layer_config* cfg, int T, int max_len_bound);
INV_API int prefill_layer(const inv_layer_config* cfg, const inv_layer_weights* w, const inv_kv_cache* cache,
                          const float* x_in, int slot, int pos0, int T, int max_len_bound, float* x_out,
                          void* workspace, size_t ws_bytes, inv_stream stream);

/* ------------------------------------------------------------------------
 * rope_tables -- model constants for the rotary embedding of decode_layer:
 *   cos_out[p][i] = fl32(cos(p theta_i)), sin_out[p][i] = fl32(sin(p theta_i)),
 *   theta_i = base^(-2i/128), i < 64, 0 <= p < max_pos, evaluated in double
 *   precision on the device.  cos_out, sin_out: fp32 [max_pos][64].
 * Errors: INV_ERR_INVALID_ARG (null, max_pos <= 0, base <= 0).
 * ------------------------------------------------------------------------ */
INV_API int rope_tables(int max_pos, double base, float* cos_out, float* sin_out, inv_stream stream);

/* ------------------------------------------------------------------------
 * Stack helpers (embedding, greedy head) for running a layer stack.
 * embed_gather: x[b][:] = table[ids[b]][:] (fp32 [vocab][hidden]); an id
 *   outside [0, vocab) records INV_ERR_INVALID_ARG and writes zeros.
 * argmax_rows: ids[b] = index of the largest logits[b][j] (fp32 [B][ld]),
 *   lowest index on ties; NaNs are ignored.
 * ------------------------------------------------------------------------ */
INV_API int embed_gather(const float* table, int vocab, int hidden, const int32_t* ids, int B,
                 float* x, inv_stream stream);
INV_API int argmax_rows(const float* logits, int B, int n, int64_t ld, int32_t* ids, inv_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* INVNUM_H */
