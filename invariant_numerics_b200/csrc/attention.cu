// Batch-invariant decode attention over the INT16 KV cache.
//
// "Defeating Nondeterminism" summary, table row Attention: one unified cache
// layout and FIXED-SIZE splits, so a row's reduction never depends on batch
// size, sequence length beyond its own, or prefill/decode chunking.  Splits are
// 256 keys at absolute positions [256 s, 256 s + 256).
// HEAL explainer, section "1. 「スマート・パッキング」のトリック": the INT16 codes
// are unpacked into two 16-bit values for the arithmetic.  Here a code is
// q = 256 h + l (h the signed high byte, l the low byte); h and l/256 are
// exact binary16 numbers, so two 16-bit tensor-core products recover q/256
// exactly before fp32 accumulation.
//
// Split kernel: one CTA (4 warps) per (row b, kv head, split s); every warp
// owns 64 keys and stages them by TMA (2-D, 128-byte swizzle) as two halves of
// 32 keys in its own 8 KB slot, so a CTA needs ~40 KB of shared memory and 5
// CTAs share an SM.  Scores S^T = K Q^T use mma.m16n8k16 with the 16 keys of
// an m-tile as rows and the 8 columns [q_hi, q_lo] x 4 query heads of the GQA
// group (q split like heal_split) as N.  The split max, exp, sum and a
// per-(split, head) power-of-two scaling of w = p s_V follow; the V halves
// then take the K slots and O^T = V^T W runs with d as rows and [w_hi, w_lo] x
// 4 heads as columns.  Warps' partial sums are added in warp order.  Output per
// (row, head, split): (m, l, o[128]).
// Combine kernel: one warp per (row, head) folds the splits s = 0, 1, ... in
// order, o / l, and writes fp32 plus the binary16 hi/lo split.
//
// This is a bandwidth-bound kernel (520 bytes of codes and scales per key and
// kv head); the warp-level MMAs only keep the 16-bit products exact at the
// rate HBM delivers the codes.
#include "common.cuh"
#include "internal.h"

namespace {

using inv::record_status;

constexpr int SPLIT = INV_KV_SPLIT;          // 256
constexpr int THREADS = 128;                 // 4 warps x 64 keys
constexpr int BOX_BYTES = 64 * 64 * 2;       // 64 keys x 64 d x int16
constexpr int CODE_BYTES = 8 * BOX_BYTES;    // 256 keys x 128 d

// Per-CTA scratch for the reductions of one row of one split.
struct RowScratch {
  float red_m[4][4];
  float red_l[4][4];
  float red_w[4][4];
  float red_mlo[4][4];  // LAMP: per-warp max of the low-precision scores
};

// LAMP selective recompute (decode, one row per call; see attn_decode_lamp).
struct LampArgs {
  float tau;                 // recompute threshold
  const float* q;            // fp32 q of the row's heads in shared memory, [head][128]
  uint8_t* sel;              // recompute flags of head 0 of the group at this split's first key, or null
  int64_t sel_head_stride;
};

// The decode kernel stages each warp's 64 keys as two halves of 32 keys in one
// 8 KB slot (K first half, second half, then V likewise), so that a CTA needs
// ~39 KB of shared memory and 5 CTAs fit on an SM.
constexpr int HALF_KEYS = 32;
constexpr int HBOX_BYTES = HALF_KEYS * 64 * 2;  // 32 keys x 64 d x int16
constexpr int WARP_SLOT = 2 * HBOX_BYTES;       // 32 keys x 128 d

struct __align__(1024) DecodeSmem {
  uint8_t codes[4 * WARP_SLOT];  // per warp: K halves, then V halves; then the warp exchange of O
  float qs[4 * 128];             // q of the row's G query heads (bulk copy with K)
  uint32_t qfrag[512];           // their hi/lo MMA fragments
  float ks[SPLIT];
  float vs[SPLIT];
  RowScratch rs;
  uint64_t bar_k, bar_q, bar_k2[4], bar_v[4], bar_v2[4];  // K first halves (all warps); per warp the rest
  int abort;
};
constexpr size_t kDecodeSmem = sizeof(DecodeSmem) + 1024;
static_assert(4 * 4 * 128 * sizeof(float) <= sizeof(DecodeSmem::codes), "the O exchange aliases the codes");

// Prefill: PF_GROUPS groups of 128 threads each run the per-row code on PF_R
// rows at a time of the block (every unpacked K/V fragment feeds PF_R rows'
// MMAs), so one SM keeps PF_GROUPS x PF_R rows in flight on the same resident
// K and V.
constexpr int PF_GROUPS = 3;
constexpr int PF_R = 3;
constexpr int PF_THREADS = PF_GROUPS * THREADS;

struct __align__(1024) PrefillSmem {
  uint8_t kcodes[CODE_BYTES];  // K and V of one split stay resident for every row
  uint8_t vcodes[CODE_BYTES];
  float xo[PF_GROUPS][PF_R][4 * 4 * 128];  // per group and row: warp exchange of O
  float ks[SPLIT];
  float vs[SPLIT];
  RowScratch rs[PF_GROUPS][PF_R];
  uint64_t bar_kv;
  int abort;
};
constexpr size_t kPrefillSmem = sizeof(PrefillSmem) + 1024;

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Dual-FP16 unpack of two INT16 codes (low half = first).  Returns the pair of
// high bytes h as binary16 and the pair of low bytes as l/256 in binary16:
// (1024 + (h + 128)) - 1152 = h and (4 + l/256) - 4 = l/256, all exact.
__device__ __forceinline__ void unpack_dual(uint32_t x, uint32_t& hpart, uint32_t& lpart) {
  const uint32_t xs = x ^ 0x80008000u;  // biased high byte h + 128; low byte unchanged
  const uint32_t hb = __byte_perm(xs, 0x64646464u, 0x4341);
  const uint32_t lb = __byte_perm(xs, 0x44444444u, 0x4240);
  const __half2 hv = __hsub2(*reinterpret_cast<const __half2*>(&hb), __halves2half2(__ushort_as_half(0x6480),
                                                                                     __ushort_as_half(0x6480)));
  const __half2 lv = __hsub2(*reinterpret_cast<const __half2*>(&lb), __halves2half2(__ushort_as_half(0x4400),
                                                                                     __ushort_as_half(0x4400)));
  hpart = *reinterpret_cast<const uint32_t*>(&hv);
  lpart = *reinterpret_cast<const uint32_t*>(&lv);
}

// Shared address of code (key kk of the split, d0 multiple of 8) in the
// 128-byte-swizzled TMA layout: box kk/64, d half d0/64, row kk%64, 16-byte
// chunk ((d0%64)/8) xor (row%8).
__device__ __forceinline__ uint32_t code_addr(uint32_t base, int kk, int d0) {
  const int r = kk & 63;
  return base + (kk >> 6) * (2 * BOX_BYTES) + (d0 >> 6) * BOX_BYTES + r * 128 +
         ((((d0 & 63) >> 3) ^ (r & 7)) << 4);
}

// The same for the decode kernel's half staging: warp slot kk/64, d half d0/64
// (a 32-row box), row kk%32, 16-byte chunk ((d0%64)/8) xor (row%8); each
// warp's two 32-key halves share its slot one after the other.
__device__ __forceinline__ uint32_t code_addr_half(uint32_t base, int kk, int d0) {
  const int r = kk & 31;
  return base + (kk >> 6) * WARP_SLOT + (d0 >> 6) * HBOX_BYTES + r * 128 + ((((d0 & 63) >> 3) ^ (r & 7)) << 4);
}

template <bool kHalf>
__device__ __forceinline__ uint32_t caddr(uint32_t base, int kk, int d0) {
  if constexpr (kHalf)
    return code_addr_half(base, kk, d0);
  else
    return code_addr(base, kk, d0);
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// The query rows one call of split_rows works on: R rows of the same kv head
// and split.  n[r] = 0 marks an absent row (nothing computed or written; its
// q pointer must still be a readable row).
template <int R>
struct RowSet {
  const float* q[R];      // fp32 q of the row's G query heads ([G][128])
  int n[R];               // valid keys of the row in the split (0..256)
  float* out_o[R];        // partial o of head 0 of the group, split s
  float2* out_ml[R];      // partial (m, l) of head 0 of the group, split s
};

// R query rows of one split: the whole per-row computation shared by the
// decode (R = 1) and prefill (R = PF_R) kernels.  Each unpacked K or V fragment
// feeds the MMAs of all R rows, and every row's accumulators receive exactly
// the MMAs, in exactly the order, that they receive with R = 1 (an m-tile
// beyond a row's n is skipped for that row), so a (row, split) gives the same
// bits in both kernels.
//   tid  : thread index within the rows' 128-thread group.
//   sync : barrier over exactly that group (__syncthreads in the decode kernel,
//          a named barrier per group in the prefill kernel).
//   kbase/vbase : shared addresses of the split's K / V codes (swizzled layout).
//   ks/vs : shared scales (zero beyond the keys that were loaded).
//   rs   : R scratch records, one per row.
//   xo   : R shared [4 warps][4 heads][128] exchange buffers (in the decode
//          kernel the one buffer aliases the codes: it is written only after
//          the last V read).
//   issue_v / wait_v : hooks around the first V access.  issue_v runs in every
//          thread once its warp has finished reading K (a warp reads and later
//          overwrites only the codes of its own 64 keys); the decode kernel
//          loads the first half of that warp's V codes into its slot there.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// The B fragments of S^T = K Q^T for R rows: column g is query head g/2 of
// the group, its hi part for even g and lo part for odd g; rows k = d.  Every
// warp needs the same fragments, so the group splits each q value once: pair
// p = (row r, k-step ks, i, head, c) holds d = 16 ks + 2 c + 8 i and d + 1, and
// its hi and lo words go to lanes 4 (2 head) + c and 4 (2 head + 1) + c at
// qfrag[((r 4 + j) 32 + lane) 4 + e] for ks 2 + i = 4 j + e, so that each lane
// later reads its 16 words as 4 conflict-free 128-bit loads.
template <int R>
__device__ __forceinline__ void write_q_fragments(int tid, const RowSet<R>& rows, int G, uint32_t* qfrag,
                                                  int* status) {
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 2 * R; ++k) {
    const int r = k >> 1, rem = (tid + THREADS * k) & 255;
    const int cc = rem & 3, head = (rem >> 2) & 3, q16 = rem >> 4;  // q16 = ks 2 + i
    const int d = 16 * (q16 >> 1) + 2 * cc + 8 * (q16 & 1);
    const bool valid = head < G && rows.n[r] > 0;
    const float2 x = valid ? *reinterpret_cast<const float2*>(rows.q[r] + head * 128 + d) : make_float2(0.f, 0.f);
    __half h0, l0, h1, l1;
    inv::split_hi_lo(x.x, h0, l0);
    inv::split_hi_lo(x.y, h1, l1);
    bad |= inv::f16_overflow(x.x) | inv::f16_overflow(x.y);
    uint32_t* dst = qfrag + ((r * 4 + (q16 >> 2)) * 32 + 8 * head + cc) * 4 + (q16 & 3);
    dst[0] = pack_half2(h0, h1);
    dst[16] = pack_half2(l0, l1);  // lane + 4
  }
  if (bad) record_status(status, INV_ERR_RANGE);
}

// kQReady: the caller has already written the rows' q fragments into qfrag
// (write_q_fragments) and synchronised the group.
// kLamp (R = 1 only): each score is also evaluated in low precision -- q16 .
// code accumulated in binary16, one rounding per multiply-add, over d in
// ascending order, the high and low code bytes in two accumulators -- and the
// scores whose relaxed criterion 2 exp(y_lo - m_lo) |y_lo| exceeds tau (m_lo
// the split's largest finite low-precision score; non-finite ones always)
// keep the full-precision value; the others continue with y_lo.
// kHalf: the codes are staged in 32-key halves (code_addr_half); mid_k and
// mid_v run in every thread of a warp before its third m-tile of the scores
// and of P.V, once the warp has read its first half: they bring the second
// half of the warp's K or V codes into its slot and return the warp's ok.
template <int R, bool kReuse, bool kLamp, bool kQReady, bool kHalf, class Sync, class IssueV, class WaitV, class MidK,
          class MidV>
__device__ __forceinline__ void split_rows(int tid, Sync sync, const RowSet<R>& rows, int G, uint32_t kbase,
                                           uint32_t vbase, const float* ks, const float* vs, RowScratch* rs,
                                           float* xo, uint32_t* qfrag, float sigma, int64_t head_stride_o,
                                           int64_t head_stride_ml,
                                           bool ok, int* status, const LampArgs& lamp, IssueV issue_v,
                                           WaitV wait_v, MidK mid_k, MidV mid_v) {
  static_assert(!kLamp || R == 1, "the low-precision pass is per row");
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  int n_max = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) n_max = max(n_max, rows.n[r]);

  // B fragments of S^T = K Q^T (write_q_fragments' layout)
  uint32_t qf[R][8][2];
  {
    if constexpr (!kQReady) {
      write_q_fragments<R>(tid, rows, G, qfrag, status);
      sync();
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w4 = lds128(inv::smem_u32(qfrag + ((r * 4 + j) * 32 + lane) * 4));
        qf[r][2 * j][0] = w4.x;
        qf[r][2 * j][1] = w4.y;
        qf[r][2 * j + 1][0] = w4.z;
        qf[r][2 * j + 1][1] = w4.w;
      }
  }

  // ---------------------------------------------------------------- scores --
  float tsc[R][4][2];
  float mx[R];
  float tlo[4][2];          // kLamp: low-precision scores of this thread's keys
  float mlo = -INFINITY;    // kLamp: their largest finite value
#pragma unroll
  for (int r = 0; r < R; ++r) mx[r] = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int kb = warp * 64 + mt * 16;
    if constexpr (kHalf) {
      if (mt == 2) ok = mid_k(ok);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) tsc[r][mt][0] = tsc[r][mt][1] = -INFINITY;
    if constexpr (kLamp) tlo[mt][0] = tlo[mt][1] = -INFINITY;
    if constexpr (kLamp) {
      if (ok && kb < n_max) {
        // keys kb + g and kb + g + 8 of head c, side by side in one half2
        __half2 ah = __float2half2_rn(0.0f), al = ah;
        const float* qh = lamp.q + c * 128;
#pragma unroll 2
        for (int d0 = 0; d0 < 128; d0 += 8) {
          const uint4 c1 = lds128(caddr<kHalf>(kbase, kb + g, d0));
          const uint4 c2 = lds128(caddr<kHalf>(kbase, kb + g + 8, d0));
          const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w}, w2[4] = {c2.x, c2.y, c2.z, c2.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t a = (w1[j >> 1] >> (16 * (j & 1))) & 0xFFFFu, b = (w2[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
            uint32_t hp, lp;
            unpack_dual(a | (b << 16), hp, lp);
            const __half2 q2 = __float2half2_rn(qh[d0 + j]);
            ah = __hfma2(q2, *reinterpret_cast<const __half2*>(&hp), ah);
            al = __hfma2(q2, *reinterpret_cast<const __half2*>(&lp), al);
          }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int key = kb + g + 8 * i;
          const float h = __half2float(i ? __high2half(ah) : __low2half(ah));
          const float l = __half2float(i ? __high2half(al) : __low2half(al));
          const float y = __fmul_rn(__fmul_rn(__fadd_rn(__fmul_rn(256.0f, h), __fmul_rn(256.0f, l)), ks[key]), sigma);
          if (key < rows.n[0]) {
            tlo[mt][i] = y;
            if (isfinite(y)) mlo = fmaxf(mlo, y);
          }
        }
      }
    }
    if (ok && kb < n_max) {
      float acc[R][4];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.0f;
      const int lkey = kb + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks_ = 0; ks_ < 8; ++ks_) {
        uint32_t a[4], ah[4], al[4];
        ldsm_x4(caddr<kHalf>(kbase, lkey, 16 * ks_ + (lane >> 4) * 8), a);
#pragma unroll
        for (int i = 0; i < 4; ++i) unpack_dual(a[i], ah[i], al[i]);
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (kb < rows.n[r]) mma16816(acc[r], ah, qf[r][ks_][0], qf[r][ks_][1]);
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (kb < rows.n[r]) mma16816(acc[r], al, qf[r][ks_][0], qf[r][ks_][1]);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (kb >= rows.n[r]) continue;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int key = kb + g + 8 * i;
          // acc[2i] = q_hi . code / 256, acc[2i+1] = q_lo . code / 256 (head c)
          const float dot = __fmul_rn(__fadd_rn(acc[r][2 * i], __fmul_rn(acc[r][2 * i + 1], 0x1p-11f)), 256.0f);
          const float t = __fmul_rn(__fmul_rn(dot, ks[key]), sigma);
          tsc[r][mt][i] = key < rows.n[r] ? t : -INFINITY;
          mx[r] = fmaxf(mx[r], tsc[r][mt][i]);
        }
      }
    }
  }
  if constexpr (kLamp) {
    // the split's largest finite low-precision score of head c, then the
    // recompute decision of every key
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 4));
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 8));
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 16));
    if (g == 0) rs[0].red_mlo[warp][c] = mlo;
    sync();
    const float Mlo = fmaxf(fmaxf(rs[0].red_mlo[0][c], rs[0].red_mlo[1][c]),
                            fmaxf(rs[0].red_mlo[2][c], rs[0].red_mlo[3][c]));
    mx[0] = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int key = warp * 64 + mt * 16 + g + 8 * i;
        if (ok && key < rows.n[0]) {
          const float y = tlo[mt][i];
          const bool sel =
              !isfinite(y) || __fmul_rn(__fmul_rn(2.0f, expf(__fsub_rn(y, Mlo))), fabsf(y)) > lamp.tau;
          if (!sel) tsc[0][mt][i] = y;
          if (lamp.sel != nullptr && c < G) lamp.sel[c * lamp.sel_head_stride + key] = sel ? 1 : 0;
        }
        mx[0] = fmaxf(mx[0], tsc[0][mt][i]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 4));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 8));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 16));
    if (g == 0) rs[r].red_m[warp][c] = mx[r];
  }
  inv::fence_proxy_async_smem();  // this warp's K reads (generic proxy) before the TMA overwrite (async proxy)
  __syncwarp();
  issue_v();
  sync();

  // ---------------------------------------------------------------- softmax --
  float w[R][4][2];
  int E[R];
  {
    float lsum[R], wmax[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float M = fmaxf(fmaxf(rs[r].red_m[0][c], rs[r].red_m[1][c]), fmaxf(rs[r].red_m[2][c], rs[r].red_m[3][c]));
      lsum[r] = 0.0f;
      wmax[r] = 0.0f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int key = warp * 64 + mt * 16 + g + 8 * i;
          const float p = tsc[r][mt][i] == -INFINITY ? 0.0f : expf(__fsub_rn(tsc[r][mt][i], M));
          lsum[r] = __fadd_rn(lsum[r], p);
          w[r][mt][i] = (key < rows.n[r] && p != 0.0f) ? __fmul_rn(p, vs[key]) : 0.0f;
          wmax[r] = fmaxf(wmax[r], w[r][mt][i]);
        }
      }
      lsum[r] = __fadd_rn(lsum[r], __shfl_xor_sync(0xffffffffu, lsum[r], 4));
      lsum[r] = __fadd_rn(lsum[r], __shfl_xor_sync(0xffffffffu, lsum[r], 8));
      lsum[r] = __fadd_rn(lsum[r], __shfl_xor_sync(0xffffffffu, lsum[r], 16));
      wmax[r] = fmaxf(wmax[r], __shfl_xor_sync(0xffffffffu, wmax[r], 4));
      wmax[r] = fmaxf(wmax[r], __shfl_xor_sync(0xffffffffu, wmax[r], 8));
      wmax[r] = fmaxf(wmax[r], __shfl_xor_sync(0xffffffffu, wmax[r], 16));
      if (g == 0) {
        rs[r].red_l[warp][c] = lsum[r];
        rs[r].red_w[warp][c] = wmax[r];
      }
    }
  }
  sync();
  // per-(split, head) exponent E: max_j w_j 2^E in [2^14, 2^15); packed
  // (hi, lo) of w 2^E for keys g and g+8 of every m-tile
  uint32_t pw_hi[R][4], pw_lo[R][4];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    E[r] = 0;
    const float wm = fmaxf(fmaxf(rs[r].red_w[0][c], rs[r].red_w[1][c]), fmaxf(rs[r].red_w[2][c], rs[r].red_w[3][c]));
    if (wm > 0.0f) {
      int ex;
      frexpf(wm, &ex);
      E[r] = 15 - ex;
      E[r] = E[r] < -120 ? -120 : (E[r] > 120 ? 120 : E[r]);
    }
    const float scaleE = inv::pow2f(E[r]);
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      __half h0, l0, h1, l1;
      inv::split_hi_lo(__fmul_rn(w[r][mt][0], scaleE), h0, l0);
      inv::split_hi_lo(__fmul_rn(w[r][mt][1], scaleE), h1, l1);
      pw_hi[r][mt] = pack_half2(h0, h1);
      pw_lo[r][mt] = pack_half2(l0, l1);
    }
  }

  ok = wait_v(ok);

  // --------------------------------------------------------------- values --
  float o[R][8][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int dt = 0; dt < 8; ++dt) o[r][dt][0] = o[r][dt][1] = o[r][dt][2] = o[r][dt][3] = 0.0f;
  const int src1 = 4 * (2 * c) + (g >> 1), src2 = 4 * (2 * c + 1) + (g >> 1);
  const bool want_lo = (g & 1) != 0;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int kb = warp * 64 + mt * 16;
    if constexpr (kHalf) {
      if (mt == 2) ok = mid_v(ok);
    }
    // B fragment of O^T = V^T W: rows k = keys, column g = head g/2 (hi/lo)
    uint32_t b0[R], b1[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint32_t x1h = __shfl_sync(0xffffffffu, pw_hi[r][mt], src1);
      const uint32_t x1l = __shfl_sync(0xffffffffu, pw_lo[r][mt], src1);
      const uint32_t x2h = __shfl_sync(0xffffffffu, pw_hi[r][mt], src2);
      const uint32_t x2l = __shfl_sync(0xffffffffu, pw_lo[r][mt], src2);
      const uint32_t x1 = want_lo ? x1l : x1h, x2 = want_lo ? x2l : x2h;
      b0[r] = __byte_perm(x1, x2, 0x5410);  // keys 2c, 2c+1
      b1[r] = __byte_perm(x1, x2, 0x7632);  // keys 2c+8, 2c+9
    }
    if (ok && kb < n_max) {
      const int lkey = kb + (lane >> 4) * 8 + (lane & 7);
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        uint32_t a[4], ah[4], al[4];
        ldsm_x4_t(caddr<kHalf>(vbase, lkey, 16 * dt + ((lane >> 3) & 1) * 8), a);
#pragma unroll
        for (int i = 0; i < 4; ++i) unpack_dual(a[i], ah[i], al[i]);
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (kb < rows.n[r]) mma16816(o[r][dt], ah, b0[r], b1[r]);
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (kb < rows.n[r]) mma16816(o[r][dt], al, b0[r], b1[r]);
      }
    }
  }
  // o[r][dt]: (d = 16dt + g, col 2c = w_hi head c), (d, col 2c+1 = w_lo), (d+8, ...)
  sync();  // every warp is done reading V codes (xo may alias them)
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float unscale = inv::pow2f(-E[r]);
    float* xr = xo + r * (4 * 4 * 128);
#pragma unroll
    for (int dt = 0; dt < 8; ++dt) {
      const float v0 =
          __fmul_rn(__fmul_rn(__fadd_rn(o[r][dt][0], __fmul_rn(o[r][dt][1], 0x1p-11f)), 256.0f), unscale);
      const float v1 =
          __fmul_rn(__fmul_rn(__fadd_rn(o[r][dt][2], __fmul_rn(o[r][dt][3], 0x1p-11f)), 256.0f), unscale);
      xr[(warp * 4 + c) * 128 + 16 * dt + g] = v0;
      xr[(warp * 4 + c) * 128 + 16 * dt + g + 8] = v1;
    }
  }
  sync();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (rows.n[r] <= 0) continue;
    const float* xr = xo + r * (4 * 4 * 128);
    {
      // thread t: head t / 32, d = 4 (t % 32) .. +3; the warps' partials are
      // added in warp order 0, 1, 2, 3
      const int head = tid >> 5, d = (tid & 31) * 4;
      if (head < G) {
        float4 v = *reinterpret_cast<const float4*>(xr + (0 * 4 + head) * 128 + d);
#pragma unroll
        for (int w = 1; w < 4; ++w) {
          const float4 u = *reinterpret_cast<const float4*>(xr + (w * 4 + head) * 128 + d);
          v.x = __fadd_rn(v.x, u.x);
          v.y = __fadd_rn(v.y, u.y);
          v.z = __fadd_rn(v.z, u.z);
          v.w = __fadd_rn(v.w, u.w);
        }
        *reinterpret_cast<float4*>(rows.out_o[r] + head * head_stride_o + d) = v;
      }
    }
    if (tid < G) {
      const RowScratch& sr = rs[r];
      const float Mh = fmaxf(fmaxf(sr.red_m[0][tid], sr.red_m[1][tid]), fmaxf(sr.red_m[2][tid], sr.red_m[3][tid]));
      float l = sr.red_l[0][tid];
      l = __fadd_rn(l, sr.red_l[1][tid]);
      l = __fadd_rn(l, sr.red_l[2][tid]);
      l = __fadd_rn(l, sr.red_l[3][tid]);
      rows.out_ml[r][tid * head_stride_ml] = make_float2(Mh, l);
    }
  }
  if (kReuse) sync();  // the scratch and xo are reused by the next rows
}

// Decode: one CTA per (row b, kv head h, split s).  kLamp: the LAMP variant
// (tau, and the recompute flags sel [B][Hq][sel_ld] or null).
template <bool kLamp>
__global__ void __launch_bounds__(THREADS, 5)
    attn_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const float* __restrict__ q, const float* __restrict__ kscale, const float* __restrict__ vscale,
                      const int32_t* __restrict__ slot, const int32_t* __restrict__ len, int Hq, int Hkv,
                      int n_slots, int max_len, int len_limit, int S_max, float sigma, float* __restrict__ part_o,
                      float2* __restrict__ part_ml, int* status, long long wait_ns, float tau, uint8_t* sel,
                      int64_t sel_ld) {
  inv::grid_launch_dependents();  // the combine kernel may be scheduled once every CTA has started
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int L = len[b], sl = slot[b];
  if (L < 1 || L > len_limit || sl < 0 || sl >= n_slots) {
    if (s == 0 && h == 0 && threadIdx.x == 0) record_status(status, INV_ERR_INVALID_ARG);
    return;
  }
  const int key0 = s * SPLIT;
  if (key0 >= L) return;
  const int n = min(SPLIT, L - key0);
  const int nbox = (n + 63) >> 6;
  const int row0 = (int)(((int64_t)sl * Hkv + h) * max_len + key0);
  const int64_t obase = (int64_t)b * Hq + (int64_t)h * G;
  {
    // index checks: the split's scales, the row's G query heads, their partials
    // (part_o [B][Hq][S_max][128], part_ml [B][Hq][S_max]) and recompute flags
    [[maybe_unused]] const int64_t BHq = (int64_t)gridDim.z * Hq;
    if (!INV_SPAN_IN_BOUNDS(status, row0, row0 + n - 1, (int64_t)n_slots * Hkv * max_len) ||
        !INV_SPAN_IN_BOUNDS(status, obase * 128, (obase + G) * 128 - 1, BHq * 128) ||
        !INV_SPAN_IN_BOUNDS(status, (obase * S_max + s) * 128, ((obase + G - 1) * S_max + s) * 128 + 127,
                            BHq * S_max * 128) ||
        !INV_SPAN_IN_BOUNDS(status, obase * S_max + s, (obase + G - 1) * S_max + s, BHq * S_max) ||
        (sel != nullptr &&
         !INV_SPAN_IN_BOUNDS(status, obase * sel_ld + key0, (obase + G - 1) * sel_ld + key0 + n - 1, BHq * sel_ld)))
      return;
  }

  extern __shared__ uint8_t smem_raw[];
  DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t cbase = inv::smem_u32(sm.codes);

  if (tid == 0) {
    inv::mbar_init(&sm.bar_k, 1);
    inv::mbar_init(&sm.bar_q, 1);
    for (int w = 0; w < 4; ++w) {
      inv::mbar_init(&sm.bar_k2[w], 1);
      inv::mbar_init(&sm.bar_v[w], 1);
      inv::mbar_init(&sm.bar_v2[w], 1);
    }
    sm.abort = 0;
    inv::fence_mbar_init();
  }
  __syncthreads();
  // warp w holds keys 64 w .. 64 w + 63 of the split: its first half exists
  // when 64 w < n (w < nbox), its second half when 64 w + 32 < n
  if (tid == 0) {
    // q on its own barrier: its fragments are split while the codes land
    inv::mbar_arrive_expect_tx(&sm.bar_q, G * 128 * 4);
    inv::bulk_load(sm.qs, q + obase * 128, (uint32_t)(G * 128 * 4), &sm.bar_q);
    inv::mbar_arrive_expect_tx(&sm.bar_k, nbox * WARP_SLOT);
    for (int w = 0; w < nbox; ++w) {
      inv::tma_load_2d(sm.codes + w * WARP_SLOT, &tm_k, &sm.bar_k, 0, row0 + 64 * w);
      inv::tma_load_2d(sm.codes + w * WARP_SLOT + HBOX_BYTES, &tm_k, &sm.bar_k, 64, row0 + 64 * w);
    }
  }
  // the scales go to registers first (stored after the q fragments are done)
  constexpr int SPT = SPLIT / THREADS;
  float ksr[SPT], vsr[SPT];
#pragma unroll
  for (int i = 0; i < SPT; ++i) {
    const int j = tid + i * THREADS;
    ksr[i] = j < n ? kscale[(int64_t)row0 + j] : 0.0f;
    vsr[i] = j < n ? vscale[(int64_t)row0 + j] : 0.0f;
  }
  const RowSet<1> rows = {{sm.qs}, {n}, {part_o + (obase * S_max + s) * 128}, {part_ml + obase * S_max + s}};
  bool ok = true;
  if (lane == 0) ok = inv::mbar_wait(&sm.bar_q, 0, wait_ns, &sm.abort, status);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) write_q_fragments<1>(tid, rows, G, sm.qfrag, status);
#pragma unroll
  for (int i = 0; i < SPT; ++i) {
    sm.ks[tid + i * THREADS] = ksr[i];
    sm.vs[tid + i * THREADS] = vsr[i];
  }
  __syncthreads();  // scales and q fragments visible

  if (lane == 0 && ok) ok = inv::mbar_wait(&sm.bar_k, 0, wait_ns, &sm.abort, status);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;

  const int warp = tid >> 5;
  const bool has_first = warp < nbox, has_second = 64 * warp + HALF_KEYS < n;
  uint8_t* slot_ptr = sm.codes + warp * WARP_SLOT;
  // one bounded load of 32 keys x 128 d into this warp's slot, after every
  // lane's reads of the slot (generic proxy) are ordered before the copy
  bool issued_k2 = false, issued_v = false, issued_v2 = false;
  const auto reload = [&](bool okr, const CUtensorMap* tm, uint64_t* bar, int key_row, bool& issued) {
    inv::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && okr) {
      issued = true;
      inv::mbar_arrive_expect_tx(bar, WARP_SLOT);
      inv::tma_load_2d(slot_ptr, tm, bar, 0, key_row);
      inv::tma_load_2d(slot_ptr + HBOX_BYTES, tm, bar, 64, key_row);
    }
  };
  const auto await = [&](bool okw, uint64_t* bar) {
    if (lane == 0 && okw) okw = inv::mbar_wait(bar, 0, wait_ns, &sm.abort, status);
    return __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
  };
  const LampArgs lamp = {tau, sm.qs, sel != nullptr ? sel + obase * sel_ld + key0 : nullptr, sel_ld};
  split_rows<1, false, kLamp, true, true>(
      tid, []() { __syncthreads(); }, rows, G, cbase, cbase, sm.ks, sm.vs, &sm.rs,
      reinterpret_cast<float*>(sm.codes), sm.qfrag, sigma, (int64_t)S_max * 128, (int64_t)S_max, ok, status, lamp,
      [&]() {  // this warp is done with its K codes: bring its first V half into the same slot
        if (has_first) reload(ok, &tm_v, &sm.bar_v[warp], row0 + 64 * warp, issued_v);
      },
      [&](bool okv) { return has_first ? await(okv, &sm.bar_v[warp]) : okv; },
      [&](bool okk) {  // scores of the first K half done: the second K half
        if (!has_second) return okk;
        reload(okk, &tm_k, &sm.bar_k2[warp], row0 + 64 * warp + HALF_KEYS, issued_k2);
        return await(okk, &sm.bar_k2[warp]);
      },
      [&](bool okv) {  // P.V of the first V half done: the second V half
        if (!has_second) return okv;
        reload(okv, &tm_v, &sm.bar_v2[warp], row0 + 64 * warp + HALF_KEYS, issued_v2);
        return await(okv, &sm.bar_v2[warp]);
      });
  // No copy may still be landing in this CTA's shared memory when it exits
  // (only possible after a timed-out wait; immediate otherwise).
  if (tid == 0) {
    inv::mbar_wait(&sm.bar_q, 0, wait_ns, nullptr, status);
    inv::mbar_wait(&sm.bar_k, 0, wait_ns, nullptr, status);
  }
  if (lane == 0) {
    if (issued_k2) inv::mbar_wait(&sm.bar_k2[warp], 0, wait_ns, nullptr, status);
    if (issued_v) inv::mbar_wait(&sm.bar_v[warp], 0, wait_ns, nullptr, status);
    if (issued_v2) inv::mbar_wait(&sm.bar_v2[warp], 0, wait_ns, nullptr, status);
  }
}

// Prefill: rows r = 0..T-1 of one sequence (slot sl) at positions p0 + r.
// One CTA per (kv head h, split s, block of ROWS_PER_CTA rows): the split's K
// and V are loaded once and every row of the block that reaches split s runs
// split_rows -- the decode kernel's per-row code, with the same thread-to-data
// mapping inside its 128-thread group -- on them, PF_GROUPS x PF_R rows at a
// time.
constexpr int ROWS_PER_CTA = 72;  // a multiple of PF_GROUPS x PF_R

__global__ void __launch_bounds__(PF_THREADS, 1)
    attn_prefill_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                              const float* __restrict__ q, const float* __restrict__ kscale,
                              const float* __restrict__ vscale, int sl, int p0, int T, int Hq, int Hkv, int max_len,
                              int S_max, float sigma, float* __restrict__ part_o, float2* __restrict__ part_ml,
                              int* status, long long wait_ns, int n_slots) {
  inv::grid_launch_dependents();  // the combine kernel may be scheduled once every CTA has started
  const int s = blockIdx.x, h = blockIdx.y, rb = blockIdx.z;
  const int G = Hq / Hkv;
  const int key0 = s * SPLIT;
  // rows of this block that reach split s: p0 + r + 1 > key0
  const int r_first = max(rb * ROWS_PER_CTA, key0 - p0);
  const int r_last = min(T, (rb + 1) * ROWS_PER_CTA) - 1;
  if (r_first > r_last) return;
  const int n_max = min(SPLIT, p0 + r_last + 1 - key0);
  const int nbox = (n_max + 63) >> 6;
  const int row0 = (int)(((int64_t)sl * Hkv + h) * max_len + key0);
  // index check of the split's scales (the rows' q and partials: per row below)
  if (!INV_SPAN_IN_BOUNDS(status, row0, row0 + n_max - 1, (int64_t)n_slots * Hkv * max_len)) return;

  extern __shared__ uint8_t smem_raw[];
  PrefillSmem& sm = *reinterpret_cast<PrefillSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31;

  if (tid == 0) {
    inv::mbar_init(&sm.bar_kv, 1);
    sm.abort = 0;
    inv::fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    inv::mbar_arrive_expect_tx(&sm.bar_kv, 2 * nbox * 2 * BOX_BYTES);
    for (int bx = 0; bx < nbox; ++bx) {
      inv::tma_load_2d(sm.kcodes + bx * 2 * BOX_BYTES, &tm_k, &sm.bar_kv, 0, row0 + 64 * bx);
      inv::tma_load_2d(sm.kcodes + bx * 2 * BOX_BYTES + BOX_BYTES, &tm_k, &sm.bar_kv, 64, row0 + 64 * bx);
      inv::tma_load_2d(sm.vcodes + bx * 2 * BOX_BYTES, &tm_v, &sm.bar_kv, 0, row0 + 64 * bx);
      inv::tma_load_2d(sm.vcodes + bx * 2 * BOX_BYTES + BOX_BYTES, &tm_v, &sm.bar_kv, 64, row0 + 64 * bx);
    }
  }
  for (int j = tid; j < SPLIT; j += PF_THREADS) {
    sm.ks[j] = j < n_max ? kscale[(int64_t)row0 + j] : 0.0f;
    sm.vs[j] = j < n_max ? vscale[(int64_t)row0 + j] : 0.0f;
  }
  __syncthreads();
  bool ok = true;
  if (lane == 0) ok = inv::mbar_wait(&sm.bar_kv, 0, wait_ns, &sm.abort, status);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;

  const uint32_t kbase = inv::smem_u32(sm.kcodes), vbase = inv::smem_u32(sm.vcodes);
  // group grp takes the rows r0 .. r0 + PF_R - 1 for r0 = r_first + grp PF_R,
  // then + PF_GROUPS PF_R, ...; its barrier is named barrier 1 + grp over its
  // own 128 threads.  A row past r_last is absent (n = 0).
  const int grp = tid / THREADS, gtid = tid % THREADS;
  const auto group_sync = [grp]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(THREADS) : "memory"); };
  for (int r0 = r_first + grp * PF_R; r0 <= r_last; r0 += PF_GROUPS * PF_R) {
    RowSet<PF_R> rows;
#pragma unroll
    for (int i = 0; i < PF_R; ++i) {
      const int r = r0 + i <= r_last ? r0 + i : r0;
      const int64_t obase = (int64_t)r * Hq + (int64_t)h * G;
      rows.q[i] = q + obase * 128;
      rows.n[i] = r0 + i <= r_last ? min(SPLIT, p0 + r + 1 - key0) : 0;
      rows.out_o[i] = part_o + (obase * S_max + s) * 128;
      rows.out_ml[i] = part_ml + obase * S_max + s;
      // index checks of the row's q heads and partials; a failing row is left out
      if (rows.n[i] > 0 &&
          (!INV_SPAN_IN_BOUNDS(status, obase * 128, (obase + G) * 128 - 1, (int64_t)T * Hq * 128) ||
           !INV_SPAN_IN_BOUNDS(status, (obase * S_max + s) * 128, ((obase + G - 1) * S_max + s) * 128 + 127,
                               (int64_t)T * Hq * S_max * 128) ||
           !INV_SPAN_IN_BOUNDS(status, obase * S_max + s, (obase + G - 1) * S_max + s, (int64_t)T * Hq * S_max)))
        rows.n[i] = 0;
    }
    // the q fragments of the rows use the start of the group's exchange buffer,
    // which is written only after the last V read
    split_rows<PF_R, true, false, false, false>(gtid, group_sync, rows, G, kbase, vbase, sm.ks, sm.vs, sm.rs[grp],
                                  sm.xo[grp][0], reinterpret_cast<uint32_t*>(sm.xo[grp][0]),
                                  sigma, (int64_t)S_max * 128, (int64_t)S_max, ok, status, LampArgs{}, []() {},
                                  [](bool okv) { return okv; }, [](bool okk) { return okk; },
                                  [](bool okv) { return okv; });
  }
  if (tid == 0) inv::mbar_wait(&sm.bar_kv, 0, wait_ns, nullptr, status);
}

// One warp per (row, head): fold splits s = 0, 1, ... in order.  Launched as a
// programmatic dependent of the split kernel: it waits for that grid's
// completion before its first load.
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                                    const int32_t* __restrict__ len, int B, int Hq, int S_max, int len_limit,
                                    float* __restrict__ out, __half* __restrict__ out_hi, __half* __restrict__ out_lo,
                                    int* status) {
  inv::grid_wait_prerequisites();
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)B * Hq) return;
  // index checks: the warp reads its S_max partials and writes one 128-wide row
  if (!INV_SPAN_IN_BOUNDS(status, wid * S_max, wid * S_max + S_max - 1, (int64_t)B * Hq * S_max) ||
      !INV_SPAN_IN_BOUNDS(status, wid * S_max * 128, (wid * S_max + S_max) * 128 - 1, (int64_t)B * Hq * S_max * 128) ||
      !INV_SPAN_IN_BOUNDS(status, wid * 128, wid * 128 + 127, (int64_t)B * Hq * 128))
    return;
  const int b = (int)(wid / Hq);
  const float2* ml = part_ml + wid * S_max;
  const float4* po = reinterpret_cast<const float4*>(part_o + wid * S_max * 128) + lane;
  // One memory round trip for len[b], the (m, l) of the first 32 splits (lane
  // j holds split j) and this lane's o of the first PF splits; entries past
  // the row's own split count are loaded (inside the partials buffer) but
  // never used.
  constexpr int PF = 8;
  const float2 ml0 = lane < S_max ? ml[lane] : make_float2(-INFINITY, 0.0f);
  float4 o[PF];
#pragma unroll
  for (int j = 0; j < PF; ++j) o[j] = j < S_max ? po[j * 32] : make_float4(0.f, 0.f, 0.f, 0.f);
  const int L = len[b];
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  if (L >= 1 && L <= len_limit) {
    const int S = (L + SPLIT - 1) / SPLIT;
    float M = lane < S ? ml0.x : -INFINITY;  // exact max: order does not matter
    for (int c = 32; c < S; c += 32) M = fmaxf(M, lane + c < S ? ml[lane + c].x : -INFINITY);
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, k));
    float l = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float fc = 0.0f, lc = 0.0f;  // this lane's split of the current 32: exp(m - M) and l
    // splits folded in ascending order; split s's factor and l come from lane s % 32
    for (int s0 = 0; s0 < S; s0 += PF) {
      if ((s0 & 31) == 0) {
        const float2 mlc = s0 == 0 ? ml0 : (lane + s0 < S ? ml[lane + s0] : make_float2(-INFINITY, 0.0f));
        fc = lane + s0 < S ? expf(__fsub_rn(mlc.x, M)) : 0.0f;
        lc = mlc.y;
      }
      if (s0 > 0) {  // PF loads in flight
#pragma unroll
        for (int j = 0; j < PF; ++j) o[j] = s0 + j < S ? po[(s0 + j) * 32] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < PF; ++j) {
        if (s0 + j >= S) break;
        const float f = __shfl_sync(0xffffffffu, fc, (s0 + j) & 31);
        const float lj = __shfl_sync(0xffffffffu, lc, (s0 + j) & 31);
        l = __fadd_rn(l, __fmul_rn(lj, f));
        acc.x = __fadd_rn(acc.x, __fmul_rn(o[j].x, f));
        acc.y = __fadd_rn(acc.y, __fmul_rn(o[j].y, f));
        acc.z = __fadd_rn(acc.z, __fmul_rn(o[j].z, f));
        acc.w = __fadd_rn(acc.w, __fmul_rn(o[j].w, f));
      }
    }
    res = make_float4(__fdiv_rn(acc.x, l), __fdiv_rn(acc.y, l), __fdiv_rn(acc.z, l), __fdiv_rn(acc.w, l));
  }
  reinterpret_cast<float4*>(out + wid * 128)[lane] = res;
  if (out_hi) {
    __half h[4], lo[4];
    inv::split_hi_lo(res.x, h[0], lo[0]);
    inv::split_hi_lo(res.y, h[1], lo[1]);
    inv::split_hi_lo(res.z, h[2], lo[2]);
    inv::split_hi_lo(res.w, h[3], lo[3]);
    if (inv::f16_overflow(res.x) | inv::f16_overflow(res.y) | inv::f16_overflow(res.z) | inv::f16_overflow(res.w))
      record_status(status, INV_ERR_RANGE);
    uint2 hv, lv;
    hv.x = pack_half2(h[0], h[1]);
    hv.y = pack_half2(h[2], h[3]);
    lv.x = pack_half2(lo[0], lo[1]);
    lv.y = pack_half2(lo[2], lo[3]);
    reinterpret_cast<uint2*>(out_hi + wid * 128)[lane] = hv;
    reinterpret_cast<uint2*>(out_lo + wid * 128)[lane] = lv;
  }
}

bool g_prefill_attr[64] = {};

}  // namespace

namespace inv {

static int splits_for(int max_len_bound) { return (max_len_bound + SPLIT - 1) / SPLIT; }

// [part_o: B Hq S 128 fp32][part_ml: B Hq S float2]
size_t attn_workspace_bytes(int B, int Hq, int max_len_bound) {
  const size_t S = (size_t)splits_for(max_len_bound);
  return (size_t)B * Hq * S * (128 * sizeof(float) + sizeof(float2));
}

// The decode split kernel (plain or LAMP), then the ordered combine.
// The ordered combine, one warp per (row, head), launched as a programmatic
// dependent of the split kernel just enqueued on the stream (its launch
// overlaps that grid's last wave; it waits for the grid before reading).
static int launch_combine(const float* part_o, const float2* part_ml, const int32_t* len, int rows, int Hq, int S_max,
                          int len_limit, float* out, uint16_t* out_hi, uint16_t* out_lo, cudaStream_t s) {
  const int64_t warps = (int64_t)rows * Hq;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((warps * 32 + 255) / 256));
  lc.blockDim = dim3(256);
  lc.dynamicSmemBytes = 0;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&lc, attn_combine_kernel, part_o, part_ml, len, rows, Hq, S_max, len_limit,
                                           out, reinterpret_cast<__half*>(out_hi), reinterpret_cast<__half*>(out_lo),
                                           status_ptr());
  if (e != cudaSuccess) return INV_ERR_CUDA;
  INV_CHECK_LAUNCH();
  return INV_OK;
}

template <bool kLamp>
static int launch_decode(const float* q, int B, int Hq, const inv_kv_cache& c, const int32_t* slot,
                         const int32_t* len, int max_len_bound, float sigma, float* out, uint16_t* out_hi,
                         uint16_t* out_lo, void* ws, cudaStream_t s, int trace_base, float tau, uint8_t* sel,
                         int64_t sel_ld) {
  static bool attr_set[64] = {};
  if (B == 0) return INV_OK;
  const int S_max = splits_for(max_len_bound);
  float* part_o = static_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(part_o + (size_t)B * Hq * S_max * 128);
  const uint64_t rows = (uint64_t)c.n_slots * c.n_kv_heads * c.max_len;
  CUtensorMap tk, tv;  // boxes of 32 keys x 64 d (each warp stages its keys in two halves)
  int rc = make_tensor_map_2d(&tk, c.k, CU_TENSOR_MAP_DATA_TYPE_UINT16, 128, rows, 256, 64, HALF_KEYS,
                              CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  rc = make_tensor_map_2d(&tv, c.v, CU_TENSOR_MAP_DATA_TYPE_UINT16, 128, rows, 256, 64, HALF_KEYS,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_split_kernel<kLamp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDecodeSmem) != cudaSuccess ||
        cudaFuncSetAttribute(attn_split_kernel<kLamp>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return INV_ERR_CUDA;
    attr_set[dev] = true;
  }
  trace_record(2 * trace_base, s);
  dim3 grid(S_max, c.n_kv_heads, B);
  attn_split_kernel<kLamp><<<grid, THREADS, kDecodeSmem, s>>>(
      tk, tv, q, c.k_scale, c.v_scale, slot, len, Hq, c.n_kv_heads, c.n_slots, c.max_len, max_len_bound, S_max, sigma,
      part_o, part_ml, status_ptr(), wait_limit_ns(), tau, sel, sel_ld);
  INV_CHECK_LAUNCH();
  trace_record(2 * trace_base + 1, s);
  trace_record(2 * trace_base + 2, s);
  rc = launch_combine(part_o, part_ml, len, B, Hq, S_max, max_len_bound, out, out_hi, out_lo, s);
  if (rc != INV_OK) return rc;
  trace_record(2 * trace_base + 3, s);
  return INV_OK;
}

int launch_attention(const float* q, int B, int Hq, const inv_kv_cache& c, const int32_t* slot, const int32_t* len,
                     int max_len_bound, float sigma, float* out, uint16_t* out_hi, uint16_t* out_lo, void* ws,
                     cudaStream_t s, int trace_base) {
  return launch_decode<false>(q, B, Hq, c, slot, len, max_len_bound, sigma, out, out_hi, out_lo, ws, s, trace_base,
                              0.0f, nullptr, 0);
}

int launch_attention_prefill(const float* q, int T, int Hq, const inv_kv_cache& c, int slot, int pos0,
                             const int32_t* len, int max_len_bound, float sigma, float* out, uint16_t* out_hi,
                             uint16_t* out_lo, void* ws, cudaStream_t s, int trace_base) {
  if (T == 0) return INV_OK;
  const int S_max = splits_for(max_len_bound);
  float* part_o = static_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(part_o + (size_t)T * Hq * S_max * 128);
  const uint64_t rows = (uint64_t)c.n_slots * c.n_kv_heads * c.max_len;
  CUtensorMap tk, tv;
  int rc = make_tensor_map_2d(&tk, c.k, CU_TENSOR_MAP_DATA_TYPE_UINT16, 128, rows, 256, 64, 64,
                              CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  rc = make_tensor_map_2d(&tv, c.v, CU_TENSOR_MAP_DATA_TYPE_UINT16, 128, rows, 256, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != INV_OK) return rc;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !g_prefill_attr[dev]) {
    if (cudaFuncSetAttribute(attn_prefill_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPrefillSmem) != cudaSuccess)
      return INV_ERR_CUDA;
    g_prefill_attr[dev] = true;
  }
  dim3 grid(splits_for(pos0 + T), c.n_kv_heads, (T + ROWS_PER_CTA - 1) / ROWS_PER_CTA);
  trace_record(2 * trace_base, s);
  attn_prefill_split_kernel<<<grid, PF_THREADS, kPrefillSmem, s>>>(tk, tv, q, c.k_scale, c.v_scale, slot, pos0, T, Hq,
                                                                c.n_kv_heads, c.max_len, S_max, sigma, part_o,
                                                                part_ml, status_ptr(), wait_limit_ns(), c.n_slots);
  INV_CHECK_LAUNCH();
  trace_record(2 * trace_base + 1, s);
  trace_record(2 * trace_base + 2, s);
  const int rcc = launch_combine(part_o, part_ml, len, T, Hq, S_max, max_len_bound, out, out_hi, out_lo, s);
  if (rcc != INV_OK) return rcc;
  trace_record(2 * trace_base + 3, s);
  return INV_OK;
}

}  // namespace inv

namespace {

// Host validation shared by the decode attention entry points; on success *mlb
// is the resolved length bound.
int validate_decode(const float* q, int B, int n_heads, const inv_kv_cache* cache, const int32_t* slot,
                    const int32_t* len, int max_len_bound, int split, float* out, uint16_t* out_hi, uint16_t* out_lo,
                    int* mlb) {
  if (!cache || B < 0 || n_heads <= 0) return INV_ERR_INVALID_ARG;
  if (split != INV_KV_SPLIT) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->head_dim != INV_HEAD_DIM || cache->n_kv_heads <= 0 || n_heads % cache->n_kv_heads != 0)
    return INV_ERR_UNSUPPORTED_SHAPE;
  const int G = n_heads / cache->n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->max_len <= 0 || cache->max_len % 64 != 0 || cache->n_slots <= 0) return INV_ERR_INVALID_ARG;
  if ((uint64_t)cache->n_slots * cache->n_kv_heads * cache->max_len >= (1ull << 31)) return INV_ERR_UNSUPPORTED_SHAPE;
  if (B > 65535) return INV_ERR_UNSUPPORTED_SHAPE;
  if (B > 0 && (!q || !slot || !len || !out || !cache->k || !cache->v || !cache->k_scale || !cache->v_scale))
    return INV_ERR_INVALID_ARG;
  if ((out_hi == nullptr) != (out_lo == nullptr)) return INV_ERR_INVALID_ARG;
  if (B > 0 && (!inv::aligned16(q) || !inv::aligned16(cache->k) || !inv::aligned16(cache->v) || !inv::aligned16(out)))
    return INV_ERR_INVALID_ARG;
  if (out_hi && ((reinterpret_cast<uintptr_t>(out_hi) | reinterpret_cast<uintptr_t>(out_lo)) & 7u))
    return INV_ERR_INVALID_ARG;
  *mlb = max_len_bound > 0 ? (max_len_bound < cache->max_len ? max_len_bound : cache->max_len) : cache->max_len;
  return INV_OK;
}

}  // namespace

extern "C" {

int attn_decode_lamp(const float* q, int B, int n_heads, const inv_kv_cache* cache, const int32_t* slot,
                     const int32_t* len, int max_len_bound, int split, float softmax_scale, float tau, float* out,
                     uint16_t* out_hi, uint16_t* out_lo, uint8_t* recompute, int64_t recompute_ld, void* workspace,
                     size_t ws_bytes, inv_stream stream) {
  int mlb = 0;
  const int rc = validate_decode(q, B, n_heads, cache, slot, len, max_len_bound, split, out, out_hi, out_lo, &mlb);
  if (rc != INV_OK) return rc;
  if (tau != tau) return INV_ERR_INVALID_ARG;  // NaN
  if (B == 0) return INV_OK;
  if (recompute != nullptr && recompute_ld < mlb) return INV_ERR_INVALID_ARG;
  if (!workspace || !inv::aligned16(workspace)) return INV_ERR_INVALID_ARG;
  if (ws_bytes < inv::attn_workspace_bytes(B, n_heads, mlb)) return INV_ERR_WORKSPACE;
  return inv::launch_decode<true>(q, B, n_heads, *cache, slot, len, mlb, softmax_scale, out, out_hi, out_lo, workspace,
                                  static_cast<cudaStream_t>(stream), -1, tau, recompute, recompute_ld);
}

size_t attn_decode_workspace_size(int B, int n_heads, int max_len_bound) {
  if (B <= 0 || n_heads <= 0 || max_len_bound <= 0) return 0;
  return inv::attn_workspace_bytes(B, n_heads, max_len_bound);
}

int attn_decode_fixedsplit(const float* q, int B, int n_heads, const inv_kv_cache* cache, const int32_t* slot,
                           const int32_t* len, int max_len_bound, int split, float softmax_scale, float* out,
                           uint16_t* out_hi, uint16_t* out_lo, void* workspace, size_t ws_bytes, inv_stream stream) {
  if (!cache || B < 0 || n_heads <= 0) return INV_ERR_INVALID_ARG;
  if (split != INV_KV_SPLIT) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->head_dim != INV_HEAD_DIM || cache->n_kv_heads <= 0 || n_heads % cache->n_kv_heads != 0)
    return INV_ERR_UNSUPPORTED_SHAPE;
  const int G = n_heads / cache->n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->max_len <= 0 || cache->max_len % 64 != 0 || cache->n_slots <= 0) return INV_ERR_INVALID_ARG;
  if ((uint64_t)cache->n_slots * cache->n_kv_heads * cache->max_len >= (1ull << 31)) return INV_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return INV_OK;
  if (B > 65535) return INV_ERR_UNSUPPORTED_SHAPE;
  if (!q || !slot || !len || !out || !cache->k || !cache->v || !cache->k_scale || !cache->v_scale || !workspace)
    return INV_ERR_INVALID_ARG;
  if ((out_hi == nullptr) != (out_lo == nullptr)) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(q) || !inv::aligned16(cache->k) || !inv::aligned16(cache->v) || !inv::aligned16(out) ||
      !inv::aligned16(workspace))
    return INV_ERR_INVALID_ARG;
  if (out_hi && ((reinterpret_cast<uintptr_t>(out_hi) | reinterpret_cast<uintptr_t>(out_lo)) & 7u))
    return INV_ERR_INVALID_ARG;
  const int mlb = max_len_bound > 0 ? (max_len_bound < cache->max_len ? max_len_bound : cache->max_len) : cache->max_len;
  if (ws_bytes < inv::attn_workspace_bytes(B, n_heads, mlb)) return INV_ERR_WORKSPACE;
  return inv::launch_attention(q, B, n_heads, *cache, slot, len, mlb, softmax_scale, out, out_hi, out_lo, workspace,
                               static_cast<cudaStream_t>(stream), -1);
}

}  // extern "C"
