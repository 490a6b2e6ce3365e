// Error-compensated GEMM on 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// HEAL explainer, section "2. 「誤差補償」のトリック（計算用）": a main product in
// 16-bit containers plus a clean-up product that catches what it spilled.
// With a = a_hi + 2^-11 a_lo and w 2^e = w_hi + 2^-11 w_lo (binary16 pairs):
//   y = ( sum a_hi w_hi  +  2^-11 sum (a_hi w_lo + a_lo w_hi) ) 2^-e   [+ residual]
// Batch invariance ("Defeating Nondeterminism" summary, table row MatMul):
// ONE tile (128 x 128), ONE K order, no split-K, whatever M is.
//
// Per 128 x 128 output tile and per 64-wide K block, the MMA thread issues for
// each 16-wide K step:
//   MMA1  D[0:256)   (+)= A_hi * [W_hi ; W_lo]^T  (N = 256: columns 0..127 "hh",
//                                                  128..255 the first cross term)
//   MMA2  D[128:256) += A_lo * W_hi^T              (N = 128: second cross term)
// The tile is 128 wide because a tcgen05.mma costs the issuing thread about the
// same whatever its N up to 256: with N = 256 + 128 per K step the tensor pipe,
// not the issue loop, sets the pace.  Accumulation runs in tensor memory over a
// group of 256 K values (4 blocks), then the epilogue warps read the group
// (tcgen05.ld) and add it to fp32 registers with round-to-nearest adds, groups
// in ascending K.  Restarting the tensor-memory accumulator every 256 K bounds
// the error of the tensor core's internal accumulation, whatever K is.  Two
// group buffers (2 x 256 TMEM columns, all of tensor memory) let the MMAs of
// group g+1 overlap the drain of group g.
//
// Warp roles (320 threads): warp 0 = TMA producer (a 192 KB ring of stages of
// A_hi, A_lo and the 256-row weight panel: 3 stages at 128 A rows, up to 5 for
// small M), warp 1 = TMEM allocator + MMA issuer, warps 2..9 =
// epilogue (warp w reads TMEM lanes 32*(w%4).., output columns 64*((w-2)/4)..).
// For M < 128 only round_up(M, 8) A rows are loaded (the MMA's other rows hold
// stale data and produce output rows that are never stored).  Persistent grid over tiles ordered
// N-panel-major so a wave of CTAs shares weight panels and A stays in L2.
//
// Two entry points share this body: comp_gemm_kernel (y, optional residual,
// or the fused SwiGLU epilogue, optionally one side of a producer/consumer
// pair) and qkv_attn_kernel, the QKV projection whose epilogue applies the
// rotary embedding and the INT16 KV quantiser to each 128-wide head tile and
// writes the attention's inputs instead of y (its epilogue warps take column
// quarters {0, 2} / {1, 3} so that rotate-half partners meet in one thread).
#include "common.cuh"
#include "internal.h"

namespace {

constexpr int BM = INV_GEMM_BM;            // 128
constexpr int BK = INV_GEMM_BK;            // 64
constexpr int MAX_STAGES = 8;
constexpr int RING_BYTES = 3 * (2 * BM * INV_GEMM_BK * 2 + 2 * 128 * INV_GEMM_BK * 2);  // 192 KB
constexpr int GROUP_KB = INV_GEMM_KGROUP / BK;  // 4
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;

// Everything that depends on the panel width BN (output columns per tile).
template <int BN>
struct Tile {
  static_assert(BN == 32 || BN == 64 || BN == 128, "panel widths 32, 64, 128");
  static constexpr int W_BYTES = 2 * BN * BK * 2;   // BN hi rows then BN lo rows, 64 K each
  static constexpr int ACC_COLS = 2 * BN;           // hh | cross
  static constexpr int TMEM_COLS = 2 * ACC_COLS;    // two group buffers
  static constexpr int EPI_COLS = BN / 2;           // output columns per epilogue thread
  static constexpr uint32_t IDESC_HILO = inv::idesc_f16_f32(128, 2 * BN);
  static constexpr uint32_t IDESC_HI = inv::idesc_f16_f32(128, BN);
  static_assert(TMEM_COLS <= 512, "tensor memory holds 512 columns");
};

struct __align__(1024) GemmSmem {
  uint8_t ring[RING_BYTES];  // n_stages stages of [A_hi | A_lo | weight panel], each 1024-aligned
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;
// The fused attention-input epilogue also needs, after GemmSmem, the per-row
// max |x| of each half of a head: [2][BM] floats.  (Measured: 198.7 KB of
// dynamic shared memory plus the 1 KB each CTA reserves fills the 196 KB
// shared-memory configuration exactly; 1 KB more still fits it, while 2 KB
// more moved every GEMM to the next configuration and made it 1-2 us slower.)
constexpr size_t kRowMaxBytes = 2 * BM * sizeof(float);
template <bool kAttnIn>
constexpr size_t smem_bytes() { return kSmemBytes + (kAttnIn ? kRowMaxBytes : 0); }

// Consumer side of a producer/consumer GEMM pair: ready_row[kb] counts the
// epilogue warps of the producing grid that have stored (and released) the
// 64 A columns of K block kb of this row tile; EPI_WARPS means complete.
// Scans forward from kb, a window of 64 counters per memory round trip, as
// far as the blocks are complete; on success *upto is the end of that run
// (> kb) and the acquire and async-proxy fences that make the data visible to
// this thread's TMA loads have been executed once for the whole run.  Gives
// up like mbar_wait (time limit or *abort).
__device__ bool wait_published(const int* ready_row, int kb, int nkb, int* upto, long long limit_ns,
                               volatile int* abort, int* status) {
  constexpr int WIN = 64;
  const unsigned long long t0 = inv::global_ns();
  for (uint32_t i = 0;; ++i) {
    int end = kb;  // first block not seen complete
    for (;;) {
      uint64_t done = 0;
#pragma unroll
      for (int j = 0; j < WIN; ++j) {
        const int v = end + j < nkb ? inv::ld_relaxed_gpu(ready_row + end + j) : 0;
        done |= (uint64_t)(v == EPI_WARPS) << j;
      }
      const int run = ~done == 0 ? WIN : __ffsll((long long)~done) - 1;
      end += run;
      if (run < WIN || end >= nkb) break;
    }
    if (end > kb) {
      inv::fence_acquire_gpu();
      inv::fence_proxy_async_global();
      *upto = end;
      return true;
    }
    if (abort != nullptr && *abort) return false;
    if ((i & 15u) == 15u && (long long)(inv::global_ns() - t0) > limit_ns) {
      inv::record_status(status, INV_ERR_TIMEOUT);
      if (abort != nullptr) *abort = 1;
      return false;
    }
  }
}

// AND of v over the 64 threads (two warps) at named barrier `id`.
__device__ __forceinline__ bool pair_all(bool v, int id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

// The kernel body; comp_gemm_kernel and qkv_attn_kernel (the fused
// attention-input epilogue, kAttnIn) are its two entry points, so that the
// plain GEMM's parameter list carries nothing it does not use.
template <int BN, bool kAttnIn>
__device__ __forceinline__ void gemm_body(const CUtensorMap& tm_ahi, const CUtensorMap& tm_alo,
                                          const CUtensorMap& tm_w, const int8_t* __restrict__ col_exp, float* y,
                                          int64_t ld_y, const float* residual, int64_t ld_r, __half* gate_hi,
                                          __half* gate_lo, int64_t ld_g, int M, int N, int K, int box_rows,
                                          int a_stride, int n_stages, int* ready_out, const int* ready_in,
                                          int* status, long long wait_ns, const inv::AttnInputs& ai) {
  using T = Tile<BN>;
  constexpr int W_BYTES = T::W_BYTES, ACC_COLS = T::ACC_COLS, TMEM_COLS = T::TMEM_COLS, EPI_COLS = T::EPI_COLS;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A grid that publishes its tiles lets its consumer grid start as soon as
  // every one of its own CTAs is resident (the consumer waits per K block).
  if (ready_out != nullptr) inv::grid_launch_dependents();
  const int tiles_m = (M + BM - 1) / BM;
  const int n_tiles = tiles_m * (N / BN);
  const int nkb = K / BK;
  const int ngroups = (nkb + GROUP_KB - 1) / GROUP_KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      inv::mbar_init(&sm.full[s], 1);
      inv::mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      inv::mbar_init(&sm.tfull[b], 1);
      inv::mbar_init(&sm.tempty[b], EPI_WARPS);
    }
    inv::mbar_init(&sm.done, 1);
    sm.abort = 0;
    inv::fence_mbar_init();
  }
  if (warp == 1) {
    inv::tmem_alloc(&sm.tmem_base, TMEM_COLS);
    inv::tmem_relinquish();
  }
  inv::tc_fence_before();
  __syncthreads();
  inv::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const uint32_t a_bytes = (uint32_t)box_rows * (BK * 2);  // one of A_hi / A_lo
      uint32_t stage = 0, phase = 0;
      uint32_t issued_mask = 0, last_phase_mask = 0;
      int ready_mt = -1, ready_upto = 0;  // K blocks [0, ready_upto) of row tile ready_mt seen published
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int nt = tile / tiles_m, mt = tile - nt * tiles_m;
        if (mt != ready_mt) {
          ready_mt = mt;
          ready_upto = 0;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!inv::mbar_wait(&sm.empty[stage], phase ^ 1u, wait_ns, abort_flag, status)) goto producer_done;
          if (ready_in != nullptr && kb >= ready_upto &&
              (!INV_SPAN_IN_BOUNDS(status, (int64_t)mt * nkb, (int64_t)mt * nkb + nkb - 1, (int64_t)tiles_m * nkb) ||
               !wait_published(ready_in + (int64_t)mt * nkb, kb, nkb, &ready_upto, wait_ns, abort_flag, status)))
            goto producer_done;
          uint8_t* st = sm.ring + stage * (2 * a_stride + W_BYTES);
          inv::mbar_arrive_expect_tx(&sm.full[stage], 2 * a_bytes + W_BYTES);
          inv::tma_load_2d(st, &tm_ahi, &sm.full[stage], kb * BK, mt * BM);
          inv::tma_load_2d(st + a_stride, &tm_alo, &sm.full[stage], kb * BK, mt * BM);
          inv::tma_load_2d(st + 2 * a_stride, &tm_w, &sm.full[stage], kb * BK, nt * 2 * BN);
          issued_mask |= 1u << stage;
          last_phase_mask = (last_phase_mask & ~(1u << stage)) | (phase << stage);
          if (++stage == (uint32_t)n_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      // Every load issued must have landed before the CTA may exit.
      for (int s = 0; s < n_stages; ++s)
        if (issued_mask & (1u << s))
          inv::mbar_wait(&sm.full[s], (last_phase_mask >> s) & 1u, wait_ns, nullptr, status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, g = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        for (int grp = 0; grp < ngroups; ++grp, ++g) {
          const uint32_t buf = g & 1u, tph = (g >> 1) & 1u;
          if (!inv::mbar_wait(&sm.tempty[buf], tph ^ 1u, wait_ns, abort_flag, status)) goto mma_done;
          inv::tc_fence_after();
          const uint32_t d = tmem + buf * ACC_COLS;
          const int kb0 = grp * GROUP_KB;
          const int kb1 = min(nkb, kb0 + GROUP_KB);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!inv::mbar_wait(&sm.full[stage], phase, wait_ns, abort_flag, status)) goto mma_done;
            inv::tc_fence_after();
            const uint32_t base = inv::smem_u32(sm.ring + stage * (2 * a_stride + W_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ahi = inv::sw128_kmajor_desc(base + kk * 32);
              const uint64_t alo = inv::sw128_kmajor_desc(base + a_stride + kk * 32);
              const uint64_t bw = inv::sw128_kmajor_desc(base + 2 * a_stride + kk * 32);
              inv::umma_f16(d, ahi, bw, T::IDESC_HILO, (kb > kb0 || kk > 0) ? 1u : 0u);
              inv::umma_f16(d + BN, alo, bw, T::IDESC_HI, 1u);
            }
            inv::umma_commit(&sm.empty[stage]);
            if (++stage == (uint32_t)n_stages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          inv::umma_commit(&sm.tfull[buf]);
        }
      }
    mma_done:
      // Every MMA issued must have completed before TMEM is released.
      inv::umma_commit(&sm.done);
      inv::mbar_wait(&sm.done, 0, wait_ns, nullptr, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    // Warp w drains TMEM lanes 32*(w%4).. (its 32 rows) and half of the tile's
    // columns: half = (w-2)/4 takes [half EPI_COLS, +EPI_COLS); with the fused
    // attention inputs (the second loop below) instead [half BN/4, +BN/4) and
    // [BN/2 + half BN/4, +BN/4), so that a thread holds columns j and j + BN/2
    // of its row (the rotate-half partners of a 128-wide head); there local
    // column c < EPI_COLS maps to tile column tcol(c).
    if constexpr (!kAttnIn) {
      const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
      const int half = (warp - 2) >> 2;      // output columns EPI_COLS*half .. +EPI_COLS-1
      uint32_t g = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int nt = tile / tiles_m, mt = tile - nt * tiles_m;
        float acc_h[EPI_COLS], acc_x[EPI_COLS];
#pragma unroll
        for (int i = 0; i < EPI_COLS; ++i) acc_h[i] = acc_x[i] = 0.0f;
        for (int grp = 0; grp < ngroups; ++grp, ++g) {
          const uint32_t buf = g & 1u, tph = (g >> 1) & 1u;
          int okw = 1;
          if (lane == 0) okw = inv::mbar_wait(&sm.tfull[buf], tph, wait_ns, abort_flag, status) ? 1 : 0;
          okw = __shfl_sync(0xffffffffu, okw, 0);  // keep the warp converged for tcgen05.ld
          if (!okw) goto epi_done;
          inv::tc_fence_after();
          const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * ACC_COLS + half * EPI_COLS;
#pragma unroll
          for (int c = 0; c < EPI_COLS; c += 16) {
            uint32_t rh[16], rx[16];
            inv::tmem_ld_32x16(ta + c, rh);
            inv::tmem_ld_32x16(ta + BN + c, rx);
            inv::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc_h[c + i] = __fadd_rn(acc_h[c + i], __uint_as_float(rh[i]));
              acc_x[c + i] = __fadd_rn(acc_x[c + i], __uint_as_float(rx[i]));
            }
          }
          inv::tc_fence_before();
          __syncwarp();
          if (lane == 0) inv::mbar_arrive(&sm.tempty[buf]);
        }
        {
          const int row = mt * BM + quarter * 32 + lane;
          const int col0 = nt * BN + half * EPI_COLS;
          if (row < M && gate_hi != nullptr) {
            // Fused SwiGLU: each 32 packed columns are 16 gate columns then the
            // 16 matching up columns of outputs f0 .. f0+15, f0 = column / 2
            // (a panel of BN >= 64 columns; the host never asks for less).
#pragma unroll
            for (int c = 0; c < (EPI_COLS % 32 == 0 ? EPI_COLS : 0); c += 32) {
              const int f0 = (col0 + c) / 2;
              // index checks: 32 column exponents, 16 outputs of gate_hi/lo [M][ld_g] (N / 2 used)
              if (!INV_SPAN_IN_BOUNDS(status, col0 + c, col0 + c + 31, N) ||
                  !INV_SPAN_IN_BOUNDS(status, (int64_t)row * ld_g + f0, (int64_t)row * ld_g + f0 + 15,
                                      (int64_t)(M - 1) * ld_g + N / 2))
                continue;
              float v[32];
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const char4 e4 = *reinterpret_cast<const char4*>(col_exp + col0 + c + i);
                const int ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float t = __fadd_rn(acc_h[c + i + j], __fmul_rn(acc_x[c + i + j], 0x1p-11f));
                  v[i + j] = __fmul_rn(t, inv::pow2f(-ev[j]));
                }
              }
              uint32_t hw[8], lw[8];
              bool bad = false;
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                __half h0, l0, h1, l1;
                const float a0 = __fmul_rn(__fdiv_rn(v[i], __fadd_rn(1.0f, expf(-v[i]))), v[16 + i]);
                const float a1 = __fmul_rn(__fdiv_rn(v[i + 1], __fadd_rn(1.0f, expf(-v[i + 1]))), v[17 + i]);
                bad |= inv::f16_overflow(a0) | inv::f16_overflow(a1);
                inv::split_hi_lo(a0, h0, l0);
                inv::split_hi_lo(a1, h1, l1);
                hw[i / 2] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
                lw[i / 2] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
              }
              if (bad) inv::record_status(status, INV_ERR_RANGE);
              uint4* gh = reinterpret_cast<uint4*>(gate_hi + (int64_t)row * ld_g + f0);
              uint4* gl = reinterpret_cast<uint4*>(gate_lo + (int64_t)row * ld_g + f0);
              gh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              gh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
              gl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
              gl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
            }
          } else if (row < M &&
                     INV_SPAN_IN_BOUNDS(status, col0, col0 + EPI_COLS - 1, N) &&
                     INV_SPAN_IN_BOUNDS(status, (int64_t)row * ld_y + col0, (int64_t)row * ld_y + col0 + EPI_COLS - 1,
                                        (int64_t)(M - 1) * ld_y + N) &&
                     (residual == nullptr ||
                      INV_SPAN_IN_BOUNDS(status, (int64_t)row * ld_r + col0, (int64_t)row * ld_r + col0 + EPI_COLS - 1,
                                         (int64_t)(M - 1) * ld_r + N))) {
            // (index checks above: column exponents, y [M][ld_y] and residual [M][ld_r], N columns used)
            float* yr = y + (int64_t)row * ld_y + col0;
            const float* rr = residual ? residual + (int64_t)row * ld_r + col0 : nullptr;
#pragma unroll
            for (int i = 0; i < EPI_COLS; i += 4) {
              const char4 e4 = *reinterpret_cast<const char4*>(col_exp + col0 + i);
              const int ev[4] = {e4.x, e4.y, e4.z, e4.w};
              float o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float t = __fadd_rn(acc_h[i + j], __fmul_rn(acc_x[i + j], 0x1p-11f));
                o[j] = __fmul_rn(t, inv::pow2f(-ev[j]));
              }
              if (rr) {
                const float4 r4 = *reinterpret_cast<const float4*>(rr + i);
                o[0] = __fadd_rn(o[0], r4.x);
                o[1] = __fadd_rn(o[1], r4.y);
                o[2] = __fadd_rn(o[2], r4.z);
                o[3] = __fadd_rn(o[3], r4.w);
              }
              *reinterpret_cast<float4*>(yr + i) = make_float4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        if (ready_out != nullptr) {
          // publish: this warp's stores of the tile, then one release add per
          // warp; the tile is complete when all EPI_WARPS warps have added
          __threadfence();
          __syncwarp();
          if (lane == 0 && INV_IN_BOUNDS(status, (int64_t)mt * (N / BN) + nt, (int64_t)tiles_m * (N / BN)))
            inv::red_release_gpu_add(ready_out + (int64_t)mt * (N / BN) + nt, 1);
        }
      }
    } else {
      const int quarter = warp & 3;
      const int half = (warp - 2) >> 2;
      constexpr int QC = BN / 4;
      const auto tcol = [half](int c) { return c < QC ? half * QC + c : 2 * QC + half * QC + (c - QC); };
      if (ai.zero_a != nullptr)  // counters of a later kernel, cleared here (any CTA, any order)
        for (int64_t i = (int64_t)blockIdx.x * (THREADS - 64) + (threadIdx.x - 64); i < ai.n_a;
             i += (int64_t)gridDim.x * (THREADS - 64))
          if (INV_IN_BOUNDS(status, i, ai.n_a)) ai.zero_a[i] = 0;
      uint32_t g = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int nt = tile / tiles_m, mt = tile - nt * tiles_m;
        float acc_h[EPI_COLS], acc_x[EPI_COLS];
#pragma unroll
        for (int i = 0; i < EPI_COLS; ++i) acc_h[i] = acc_x[i] = 0.0f;
        for (int grp = 0; grp < ngroups; ++grp, ++g) {
          const uint32_t buf = g & 1u, tph = (g >> 1) & 1u;
          int okw = 1;
          if (lane == 0) okw = inv::mbar_wait(&sm.tfull[buf], tph, wait_ns, abort_flag, status) ? 1 : 0;
          okw = __shfl_sync(0xffffffffu, okw, 0);  // keep the warp converged for tcgen05.ld
          // with the fused attention inputs the two warps of a row block meet
          // at a barrier later on: they leave (after a failed wait) together
          okw = pair_all(okw != 0, 1 + quarter) ? 1 : 0;
          if (!okw) goto epi_done;
          inv::tc_fence_after();
          const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * ACC_COLS;
#pragma unroll
          for (int c = 0; c < EPI_COLS; c += 16) {
            uint32_t rh[16], rx[16];
            inv::tmem_ld_32x16(ta + tcol(c), rh);
            inv::tmem_ld_32x16(ta + BN + tcol(c), rx);
            inv::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc_h[c + i] = __fadd_rn(acc_h[c + i], __uint_as_float(rh[i]));
              acc_x[c + i] = __fadd_rn(acc_x[c + i], __uint_as_float(rx[i]));
            }
          }
          inv::tc_fence_before();
          __syncwarp();
          if (lane == 0) inv::mbar_arrive(&sm.tempty[buf]);
        }
        {
          const int row = mt * BM + quarter * 32 + lane;
          const int col0 = nt * BN;  // first column of the tile
          // y = (hh + 2^-11 cross) 2^-e_n per column, into acc_h
          auto scale_cols = [&]() {
#pragma unroll
            for (int c = 0; c < EPI_COLS; c += 4) {
              const char4 e4 = *reinterpret_cast<const char4*>(col_exp + col0 + tcol(c));
              const int ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
              for (int j = 0; j < 4; ++j)
                acc_h[c + j] = __fmul_rn(__fadd_rn(acc_h[c + j], __fmul_rn(acc_x[c + j], 0x1p-11f)), inv::pow2f(-ev[j]));
            }
          };
          {
            // Fused attention inputs (one 128-wide head per tile): rotary
            // embedding of query and key heads, then query heads to q_out and
            // key/value heads INT16-quantised into the cache at (slot, pos) of
            // the row; len = pos + 1.  Same arithmetic, in the same order, as
            // the rotary and quantiser definitions on the stored fp32 values.
            const bool in_row = row < M;
            int sl = 0, p = 0;
            bool ok = false;
            if (in_row) {
              sl = ai.slot[row];
              p = ai.pos[row];
              ok = sl >= 0 && sl < ai.cache.n_slots && p >= 0 && p < ai.cache.max_len && p < ai.max_pos;
              if (nt == 0 && half == 0) {
                if (INV_IN_BOUNDS(status, row, M)) ai.len_out[row] = ok ? p + 1 : 0;
                if (!ok) inv::record_status(status, INV_ERR_INVALID_ARG);
              }
            }
            const int Hkv = ai.cache.n_kv_heads;
            const bool is_q = nt < ai.Hq, is_k = !is_q && nt < ai.Hq + Hkv;
            if (ok && (!INV_IN_BOUNDS(status, col0 + BN - 1, N) ||
                       !INV_SPAN_IN_BOUNDS(status, (int64_t)p * 64, (int64_t)p * 64 + 63, (int64_t)ai.max_pos * 64)))
              ok = false;
            if (ok) {
              scale_cols();
              if (is_q || is_k) {
                // rotate-half: columns j and j + 64 (local c and c + QC), frequency j
                const float* cs = ai.rope_cos + (int64_t)p * 64 + half * QC;
                const float* sn = ai.rope_sin + (int64_t)p * 64 + half * QC;
#pragma unroll
                for (int c = 0; c < QC; c += 4) {
                  const float4 c4 = *reinterpret_cast<const float4*>(cs + c);
                  const float4 s4 = *reinterpret_cast<const float4*>(sn + c);
                  const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const float lo = acc_h[c + j], hi = acc_h[QC + c + j];
                    acc_h[c + j] = __fsub_rn(__fmul_rn(lo, cv[j]), __fmul_rn(hi, sv[j]));
                    acc_h[QC + c + j] = __fadd_rn(__fmul_rn(hi, cv[j]), __fmul_rn(lo, sv[j]));
                  }
                }
              }
            }
            if (is_q) {
              const int64_t qb = ((int64_t)row * ai.Hq + nt) * 128;
              if (ok && INV_SPAN_IN_BOUNDS(status, qb, qb + 127, (int64_t)M * ai.Hq * 128)) {
#pragma unroll
                for (int c = 0; c < EPI_COLS; c += 4)
                  *reinterpret_cast<float4*>(ai.q_out + qb + tcol(c)) =
                      make_float4(acc_h[c], acc_h[c + 1], acc_h[c + 2], acc_h[c + 3]);
              }
            } else {
              // max |x| over the row's 128 values: this thread's EPI_COLS, then
              // the partner warp's (same rows, other half) through shared memory;
              // NaN is ignored by fmaxf as in the quantiser's definition
              float m = fabsf(acc_h[0]);
#pragma unroll
              for (int c = 1; c < EPI_COLS; ++c) m = fmaxf(m, fabsf(acc_h[c]));
              // exchange with the partner warp (same rows, other half); the
              // second barrier keeps the next tile's write after both reads
              float* rm = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(&sm) + sizeof(GemmSmem));
              rm[half * BM + quarter * 32 + lane] = m;
              asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");  // the warp pair of these rows
              m = fmaxf(m, rm[(half ^ 1) * BM + quarter * 32 + lane]);
              asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
              const int h = is_k ? nt - ai.Hq : nt - ai.Hq - Hkv;
              const int64_t rowi = ((int64_t)sl * Hkv + h) * ai.cache.max_len + p;
              if (ok && INV_IN_BOUNDS(status, rowi, (int64_t)ai.cache.n_slots * Hkv * ai.cache.max_len)) {
                const float sc = __fdiv_rn(m, 32767.0f);
                int16_t* codes = (is_k ? ai.cache.k : ai.cache.v) + rowi * 128;
#pragma unroll
                for (int c = 0; c < EPI_COLS; c += 8) {
                  uint32_t w4[4];
#pragma unroll
                  for (int j = 0; j < 8; j += 2) {
                    int q2[2] = {0, 0};
                    if (sc != 0.0f)
#pragma unroll
                      for (int u = 0; u < 2; ++u) {
                        const int t = __float2int_rn(__fdiv_rn(acc_h[c + j + u], sc));  // round half to even
                        q2[u] = t > 32767 ? 32767 : (t < -32767 ? -32767 : t);
                      }
                    w4[j / 2] = (uint32_t)(uint16_t)q2[0] | ((uint32_t)(uint16_t)q2[1] << 16);
                  }
                  *reinterpret_cast<uint4*>(codes + tcol(c)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                if (half == 0) (is_k ? ai.cache.k_scale : ai.cache.v_scale)[rowi] = sc;
              }
            }
          }
        }
        if (ready_out != nullptr) {
          // publish: this warp's stores of the tile, then one release add per
          // warp; the tile is complete when all EPI_WARPS warps have added
          __threadfence();
          __syncwarp();
          if (lane == 0 && INV_IN_BOUNDS(status, (int64_t)mt * (N / BN) + nt, (int64_t)tiles_m * (N / BN)))
            inv::red_release_gpu_add(ready_out + (int64_t)mt * (N / BN) + nt, 1);
        }
      }
    }
  epi_done:;
  }

  inv::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    inv::tc_fence_after();
    inv::tmem_dealloc(tmem, TMEM_COLS);
  }
  // a consumer grid completes only after its producer grid has
  if (ready_in != nullptr) inv::grid_wait_prerequisites();
}

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
    comp_gemm_kernel(const __grid_constant__ CUtensorMap tm_ahi, const __grid_constant__ CUtensorMap tm_alo,
                     const __grid_constant__ CUtensorMap tm_w, const int8_t* __restrict__ col_exp, float* y,
                     int64_t ld_y, const float* residual, int64_t ld_r, __half* gate_hi, __half* gate_lo,
                     int64_t ld_g, int M, int N, int K, int box_rows, int a_stride, int n_stages, int* ready_out,
                     const int* ready_in, int* status, long long wait_ns) {
  gemm_body<BN, false>(tm_ahi, tm_alo, tm_w, col_exp, y, ld_y, residual, ld_r, gate_hi, gate_lo, ld_g, M, N, K,
                       box_rows, a_stride, n_stages, ready_out, ready_in, status, wait_ns, inv::AttnInputs{});
}

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
    qkv_attn_kernel(const __grid_constant__ CUtensorMap tm_ahi, const __grid_constant__ CUtensorMap tm_alo,
                    const __grid_constant__ CUtensorMap tm_w, const int8_t* __restrict__ col_exp, int M, int N, int K,
                    int box_rows, int a_stride, int n_stages, int* status, long long wait_ns,
                    const inv::AttnInputs ai) {
  gemm_body<BN, true>(tm_ahi, tm_alo, tm_w, col_exp, nullptr, 0, nullptr, 0, nullptr, nullptr, 0, M, N, K, box_rows,
                      a_stride, n_stages, nullptr, nullptr, status, wait_ns, ai);
}

// One launch of the BN-wide kernel (arguments validated by the caller).
template <int BN, bool kAttnIn>
int launch_tiles(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a, const uint16_t* w_packed,
                 const int8_t* col_exp, int N, float* y, int64_t ld_y, const float* residual, int64_t ld_r,
                 uint16_t* gate_hi, uint16_t* gate_lo, int64_t ld_g, int* ready_out, const int* ready_in,
                 cudaStream_t s, long long wait_ns, const inv::AttnInputs& ai) {
  static bool attr_set[64] = {};
  // A rows per load: the whole 128-row tile, or only round_up(M, 8) when M < 128
  const int box_rows = M < BM ? (int)((M + 7) / 8 * 8) : BM;
  // Stage = [A_hi | A_lo | weight panel]; with fewer A rows the same ring holds
  // more stages (more weight bytes in flight).  The MMA still reads 128 A rows
  // from each A base: rows past box_rows hold other data of the stage and
  // only feed output rows that are never stored.
  const int a_stride = (box_rows * BK * 2 + 1023) / 1024 * 1024;
  const int stage_bytes = 2 * a_stride + Tile<BN>::W_BYTES;
  const int n_stages = RING_BYTES / stage_bytes < MAX_STAGES ? RING_BYTES / stage_bytes : MAX_STAGES;
  CUtensorMap ta, tl, tw;
  int rc = inv::make_tensor_map_2d(&ta, a_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)M,
                                   (uint64_t)ld_a * 2, BK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  rc = inv::make_tensor_map_2d(&tl, a_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)M,
                               (uint64_t)ld_a * 2, BK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  rc = inv::make_tensor_map_2d(&tw, w_packed, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)K, (uint64_t)N * 2,
                               (uint64_t)K * 2, BK, 2 * BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t ea =
        kAttnIn ? cudaFuncSetAttribute(qkv_attn_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_bytes<true>())
                : cudaFuncSetAttribute(comp_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_bytes<false>());
    if (ea != cudaSuccess) return INV_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int64_t tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = (int)(tiles < inv::sm_count() ? tiles : inv::sm_count());
  // A consumer (ready_in) is launched as a programmatic dependent of the
  // producer launched just before it on the stream, so it may start while the
  // producer's last tiles are still running; it waits per K block instead.
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(THREADS);
  lc.dynamicSmemBytes = smem_bytes<kAttnIn>();
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = ready_in != nullptr ? 1 : 0;
  const long long wl = wait_ns < 0 ? inv::wait_limit_ns() : wait_ns;
  const cudaError_t e =
      kAttnIn ? cudaLaunchKernelEx(&lc, qkv_attn_kernel<BN>, ta, tl, tw, col_exp, (int)M, N, K, box_rows, a_stride,
                                   n_stages, inv::status_ptr(), wl, ai)
              : cudaLaunchKernelEx(&lc, comp_gemm_kernel<BN>, ta, tl, tw, col_exp, y, ld_y, residual, ld_r,
                                   reinterpret_cast<__half*>(gate_hi), reinterpret_cast<__half*>(gate_lo), ld_g,
                                   (int)M, N, K, box_rows, a_stride, n_stages, ready_out, ready_in,
                                   inv::status_ptr(), wl);
  if (e != cudaSuccess) return INV_ERR_CUDA;
  INV_CHECK_LAUNCH();
  return INV_OK;
}

}  // namespace

namespace inv {

int gemm_panel_width(int N) {
  (void)N;
  return INV_GEMM_BN;
}

int launch_comp_gemm(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                     const uint16_t* w_packed, const int8_t* col_exp, int N, float* y, int64_t ld_y,
                     const float* residual, int64_t ld_r, cudaStream_t s) {
  return launch_comp_gemm_ex(a_hi, a_lo, M, K, ld_a, w_packed, col_exp, N, y, ld_y, residual, ld_r, nullptr, nullptr,
                             0, nullptr, nullptr, s);
}

int launch_comp_gemm_ex(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                        const uint16_t* w_packed, const int8_t* col_exp, int N, float* y, int64_t ld_y,
                        const float* residual, int64_t ld_r, uint16_t* gate_hi, uint16_t* gate_lo, int64_t ld_g,
                        int* ready_out, const int* ready_in, cudaStream_t s, long long wait_ns) {
  if (M == 0) return INV_OK;
  if (gemm_panel_width(N) != INV_GEMM_BN) return INV_ERR_UNSUPPORTED_SHAPE;
  return launch_tiles<INV_GEMM_BN, false>(a_hi, a_lo, M, K, ld_a, w_packed, col_exp, N, y, ld_y, residual, ld_r, gate_hi,
                                   gate_lo, ld_g, ready_out, ready_in, s, wait_ns, AttnInputs{});
}

int launch_qkv_attn_inputs(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                           const uint16_t* w_packed, const int8_t* col_exp, int N, const AttnInputs& ai,
                           cudaStream_t s) {
  if (M == 0) return INV_OK;
  if (gemm_panel_width(N) != INV_GEMM_BN || N != (ai.Hq + 2 * ai.cache.n_kv_heads) * INV_HEAD_DIM)
    return INV_ERR_UNSUPPORTED_SHAPE;
  return launch_tiles<INV_GEMM_BN, true>(a_hi, a_lo, M, K, ld_a, w_packed, col_exp, N, nullptr, 0, nullptr, 0, nullptr,
                                   nullptr, 0, nullptr, nullptr, s, -1, ai);
}

}  // namespace inv

extern "C" int comp_gemm(const uint16_t* a_hi, const uint16_t* a_lo, int64_t M, int K, int64_t ld_a,
                         const uint16_t* w_packed, const int8_t* col_exp, int N, float* y, int64_t ld_y,
                         const float* residual, int64_t ld_r, inv_stream stream) {
  if (M < 0 || K <= 0 || N <= 0) return INV_ERR_INVALID_ARG;
  if (K % BK != 0 || N % inv::gemm_panel_width(N) != 0) return INV_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return INV_OK;
  if (M > 0x7fffffffLL) return INV_ERR_UNSUPPORTED_SHAPE;
  if (!a_hi || !a_lo || !w_packed || !col_exp || !y) return INV_ERR_INVALID_ARG;
  if (ld_a < K || ld_a % 8 != 0 || ld_y < N || ld_y % 4 != 0) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(a_hi) || !inv::aligned16(a_lo) || !inv::aligned16(w_packed) || !inv::aligned16(y))
    return INV_ERR_INVALID_ARG;
  if (residual && (ld_r < N || ld_r % 4 != 0 || !inv::aligned16(residual))) return INV_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(col_exp) & 3u) != 0) return INV_ERR_INVALID_ARG;
  return inv::launch_comp_gemm(a_hi, a_lo, M, K, ld_a, w_packed, col_exp, N, y, ld_y, residual, ld_r,
                               static_cast<cudaStream_t>(stream));
}

// Self-test of the consumer side of a GEMM pair: a small consumer GEMM (M = 8,
// K = 64, N = 128) whose one K block is never published (its counter is
// zeroed and no producer runs) must give up after wait_ns, record
// INV_ERR_TIMEOUT and exit.  The operands live in the caller's workspace;
// their values do not matter (nothing is loaded).
extern "C" int inv_selftest_gemm_wait_timeout(void* workspace, size_t ws_bytes, long long wait_ns,
                                              inv_stream stream) {
  if (wait_ns <= 0 || workspace == nullptr || !inv::aligned16(workspace)) return INV_ERR_INVALID_ARG;
  if (ws_bytes < INV_SELFTEST_GEMM_WS_BYTES) return INV_ERR_WORKSPACE;
  constexpr int M = 8, K = 64, N = 128;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  uint16_t* a_hi = reinterpret_cast<uint16_t*>(p);                 // [8][64] binary16
  uint16_t* a_lo = reinterpret_cast<uint16_t*>(p + 1024);
  uint16_t* w = reinterpret_cast<uint16_t*>(p + 2048);             // [1][2][128][64] binary16
  int8_t* e = reinterpret_cast<int8_t*>(p + 2048 + 32768);         // [128]
  float* y = reinterpret_cast<float*>(p + 2048 + 32768 + 256);     // [8][128]
  int* ready = reinterpret_cast<int*>(p + 2048 + 32768 + 256 + 4096);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, INV_SELFTEST_GEMM_WS_BYTES, s) != cudaSuccess) return INV_ERR_CUDA;
  return inv::launch_comp_gemm_ex(a_hi, a_lo, M, K, K, w, e, N, y, N, nullptr, 0, nullptr, nullptr, 0, nullptr, ready,
                                  s, wait_ns);
}
