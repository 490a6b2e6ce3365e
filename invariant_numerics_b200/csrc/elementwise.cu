// Bandwidth-bound kernels of the decode step: the binary16 hi/lo split, the
// offline weight packing, batch-invariant RMSNorm, the INT16 KV quantiser, and
// the per-row glue of the stack (rotary tables, embedding gather, greedy
// argmax).  The rotary embedding itself and the quantisation of a layer's new
// keys and values run in the QKV GEMM's epilogue (comp_gemm.cu).  All use 128-bit coalesced accesses where
// the layout allows and fixed, shape-independent reduction orders.
#include "common.cuh"
#include "internal.h"

namespace {

using inv::record_status;
using inv::split_hi_lo;

// ------------------------------------------------------------- heal_split ----

// One thread per 4 consecutive columns of a row.
__global__ void heal_split_kernel(const float* __restrict__ x, int64_t rows, int64_t cols, int64_t ld_x,
                                  __half* __restrict__ hi, __half* __restrict__ lo, int64_t ld_out,
                                  int* status) {
  const int64_t c4 = (cols + 3) / 4;
  const int64_t total = rows * c4;
  [[maybe_unused]] const int64_t n_x = (rows - 1) * ld_x + cols, n_out = (rows - 1) * ld_out + cols;  // extents
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / c4;
    const int64_t c = (i - r * c4) * 4;
    for (int j = 0; j < 4 && c + j < cols; ++j) {
      const int64_t ix = r * ld_x + c + j, io = r * ld_out + c + j;
      if (!INV_IN_BOUNDS(status, ix, n_x) || !INV_IN_BOUNDS(status, io, n_out)) continue;
      const float v = x[ix];
      __half h, l;
      split_hi_lo(v, h, l);
      bad |= inv::f16_overflow(v);
      hi[io] = h;
      lo[io] = l;
    }
  }
  if (bad) record_status(status, INV_ERR_RANGE);
}

// Vector path: cols % 4 == 0 and 16-byte aligned rows.
__global__ void heal_split_vec_kernel(const float4* __restrict__ x, int64_t rows, int64_t c4, int64_t ld4,
                                      uint2* __restrict__ hi, uint2* __restrict__ lo, int64_t ldo4, int* status) {
  const int64_t total = rows * c4;
  [[maybe_unused]] const int64_t n_x = (rows - 1) * ld4 + c4, n_out = (rows - 1) * ldo4 + c4;  // in float4s
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / c4;
    const int64_t c = i - r * c4;
    if (!INV_IN_BOUNDS(status, r * ld4 + c, n_x) || !INV_IN_BOUNDS(status, r * ldo4 + c, n_out)) continue;
    const float4 v = x[r * ld4 + c];
    __half h[4], l[4];
    split_hi_lo(v.x, h[0], l[0]);
    split_hi_lo(v.y, h[1], l[1]);
    split_hi_lo(v.z, h[2], l[2]);
    split_hi_lo(v.w, h[3], l[3]);
    bad |= inv::f16_overflow(v.x) | inv::f16_overflow(v.y) | inv::f16_overflow(v.z) | inv::f16_overflow(v.w);
    uint2 ho, lo2;
    ho.x = (uint32_t)__half_as_ushort(h[0]) | ((uint32_t)__half_as_ushort(h[1]) << 16);
    ho.y = (uint32_t)__half_as_ushort(h[2]) | ((uint32_t)__half_as_ushort(h[3]) << 16);
    lo2.x = (uint32_t)__half_as_ushort(l[0]) | ((uint32_t)__half_as_ushort(l[1]) << 16);
    lo2.y = (uint32_t)__half_as_ushort(l[2]) | ((uint32_t)__half_as_ushort(l[3]) << 16);
    hi[r * ldo4 + c] = ho;
    lo[r * ldo4 + c] = lo2;
  }
  if (bad) record_status(status, INV_ERR_RANGE);
}

// ------------------------------------------------------- heal_pack_weight ----

// Column exponent: max_k |W[k][n]| 2^e in [2^14, 2^15); one thread per column,
// consecutive threads read consecutive columns of a row (coalesced).
__global__ void col_exp_kernel(const float* __restrict__ W, int K, int N, int8_t* __restrict__ e_out, int* status) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  if (!INV_SPAN_IN_BOUNDS(status, n, (int64_t)(K - 1) * N + n, (int64_t)K * N) || !INV_IN_BOUNDS(status, n, N)) return;
  float m = 0.0f;
  for (int k = 0; k < K; ++k) m = fmaxf(m, fabsf(W[(int64_t)k * N + n]));
  int e = 0;
  if (m > 0.0f) {
    int E;
    frexpf(m, &E);  // m = f 2^E, f in [0.5, 1)
    e = 15 - E;
    e = e < -120 ? -120 : (e > 120 ? 120 : e);
  }
  e_out[n] = (int8_t)e;
}

// Packed image [N/128][2][128][K]; a block transposes a 64(k) x 64(n) tile.
__global__ void pack_kernel(const float* __restrict__ W, int K, int N, const int8_t* __restrict__ e,
                            __half* __restrict__ P, int* status) {
  constexpr int PW = INV_GEMM_BN;    // panel width
  __shared__ float tile[64][65];
  const int n0 = blockIdx.x * 64;    // 64 columns, inside one panel
  const int k0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;  // 256 threads: 64 x 4
  [[maybe_unused]] const int64_t n_w = (int64_t)K * N, n_p = 2 * (int64_t)K * N;
  for (int kk = ty; kk < 64; kk += 4) {
    const int64_t iw = (int64_t)(k0 + kk) * N + n0 + tx;
    tile[kk][tx] = INV_IN_BOUNDS(status, iw, n_w) ? W[iw] : 0.0f;
  }
  __syncthreads();
  for (int r = ty; r < 64; r += 4) {
    const int n = n0 + r;
    const int j = n / PW, rr = n % PW;
    if (!INV_IN_BOUNDS(status, n, N)) continue;
    const float s = inv::pow2f(e[n]);
    const float v = __fmul_rn(tile[tx][r], s);  // exact power-of-two scaling
    __half h, l;
    split_hi_lo(v, h, l);
    const int64_t ih = (((int64_t)j * 2 + 0) * PW + rr) * K + k0 + tx, il = ih + (int64_t)PW * K;
    if (INV_IN_BOUNDS(status, ih, n_p)) P[ih] = h;
    if (INV_IN_BOUNDS(status, il, n_p)) P[il] = l;
  }
}

// -------------------------------------------------------------- rmsnorm_bi ----

constexpr int kNormThreads = 256;

// One CTA per row, one fixed reduction order: thread t takes float4 chunks
// t, t+256, ... in order (fma x.x, x.y, x.z, x.w), then an xor-shuffle tree
// (16, 8, 4, 2, 1) inside each warp, then warps 0..7 summed in order.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ gamma,
                                                                int hidden, float eps, float* __restrict__ y,
                                                                __half* __restrict__ yh, __half* __restrict__ yl,
                                                                int* status) {
  __shared__ float warp_sum[kNormThreads / 32];
  __shared__ float r_sh;
  const int64_t row = blockIdx.x;
  // x and the outputs are [rows = gridDim.x][hidden]; the row is accessed whole
  if (!INV_SPAN_IN_BOUNDS(status, row * hidden, row * hidden + hidden - 1, (int64_t)gridDim.x * hidden)) return;
  const float4* xr = reinterpret_cast<const float4*>(x + row * hidden);
  const int n4 = hidden / 4;
  float s = 0.0f;
  for (int i = threadIdx.x; i < n4; i += kNormThreads) {
    const float4 v = xr[i];
    s = __fmaf_rn(v.x, v.x, s);
    s = __fmaf_rn(v.y, v.y, s);
    s = __fmaf_rn(v.z, v.z, s);
    s = __fmaf_rn(v.w, v.w, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = warp_sum[0];
    for (int w = 1; w < kNormThreads / 32; ++w) t = __fadd_rn(t, warp_sum[w]);
    const float mean = __fdiv_rn(t, (float)hidden);
    r_sh = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
  }
  __syncthreads();
  const float r = r_sh;
  const float4* g4 = reinterpret_cast<const float4*>(gamma);
  bool bad = false;
  for (int i = threadIdx.x; i < n4; i += kNormThreads) {
    const float4 v = xr[i];
    const float4 g = g4[i];
    float4 o;
    o.x = __fmul_rn(__fmul_rn(v.x, r), g.x);
    o.y = __fmul_rn(__fmul_rn(v.y, r), g.y);
    o.z = __fmul_rn(__fmul_rn(v.z, r), g.z);
    o.w = __fmul_rn(__fmul_rn(v.w, r), g.w);
    if (y) reinterpret_cast<float4*>(y + row * hidden)[i] = o;
    if (yh) {
      __half h[4], l[4];
      split_hi_lo(o.x, h[0], l[0]);
      split_hi_lo(o.y, h[1], l[1]);
      split_hi_lo(o.z, h[2], l[2]);
      split_hi_lo(o.w, h[3], l[3]);
      bad |= inv::f16_overflow(o.x) | inv::f16_overflow(o.y) | inv::f16_overflow(o.z) | inv::f16_overflow(o.w);
      uint2 hv, lv;
      hv.x = (uint32_t)__half_as_ushort(h[0]) | ((uint32_t)__half_as_ushort(h[1]) << 16);
      hv.y = (uint32_t)__half_as_ushort(h[2]) | ((uint32_t)__half_as_ushort(h[3]) << 16);
      lv.x = (uint32_t)__half_as_ushort(l[0]) | ((uint32_t)__half_as_ushort(l[1]) << 16);
      lv.y = (uint32_t)__half_as_ushort(l[2]) | ((uint32_t)__half_as_ushort(l[3]) << 16);
      reinterpret_cast<uint2*>(yh + row * hidden)[i] = hv;
      reinterpret_cast<uint2*>(yl + row * hidden)[i] = lv;
    }
  }
  if (bad) record_status(status, INV_ERR_RANGE);
}

// Single-pass form for hidden <= 256 * 4 * VPT: each thread keeps its VPT
// float4 chunks (the same chunks t, t+256, ... in the same order as above) in
// registers, so x is read once.  Same reduction order, same result bits.
template <int VPT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_reg_kernel(const float* __restrict__ x,
                                                                    const float* __restrict__ gamma, int hidden,
                                                                    float eps, float* __restrict__ y,
                                                                    __half* __restrict__ yh, __half* __restrict__ yl,
                                                                    int* status) {
  __shared__ float warp_sum[kNormThreads / 32];
  __shared__ float r_sh;
  const int64_t row = blockIdx.x;
  // x and the outputs are [rows = gridDim.x][hidden]; the row is accessed whole
  if (!INV_SPAN_IN_BOUNDS(status, row * hidden, row * hidden + hidden - 1, (int64_t)gridDim.x * hidden)) return;
  const float4* xr = reinterpret_cast<const float4*>(x + row * hidden);
  const int n4 = hidden / 4;
  const float4* g4 = reinterpret_cast<const float4*>(gamma);
  float4 v[VPT], gv[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int i = threadIdx.x + j * kNormThreads;
    v[j] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    gv[j] = i < n4 ? g4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    if (threadIdx.x + j * kNormThreads < n4) {
      s = __fmaf_rn(v[j].x, v[j].x, s);
      s = __fmaf_rn(v[j].y, v[j].y, s);
      s = __fmaf_rn(v[j].z, v[j].z, s);
      s = __fmaf_rn(v[j].w, v[j].w, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = warp_sum[0];
    for (int w = 1; w < kNormThreads / 32; ++w) t = __fadd_rn(t, warp_sum[w]);
    const float mean = __fdiv_rn(t, (float)hidden);
    r_sh = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
  }
  __syncthreads();
  const float r = r_sh;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int i = threadIdx.x + j * kNormThreads;
    if (i >= n4) continue;
    const float4 g = gv[j];
    float4 o;
    o.x = __fmul_rn(__fmul_rn(v[j].x, r), g.x);
    o.y = __fmul_rn(__fmul_rn(v[j].y, r), g.y);
    o.z = __fmul_rn(__fmul_rn(v[j].z, r), g.z);
    o.w = __fmul_rn(__fmul_rn(v[j].w, r), g.w);
    if (y) reinterpret_cast<float4*>(y + row * hidden)[i] = o;
    if (yh) {
      __half h[4], l[4];
      split_hi_lo(o.x, h[0], l[0]);
      split_hi_lo(o.y, h[1], l[1]);
      split_hi_lo(o.z, h[2], l[2]);
      split_hi_lo(o.w, h[3], l[3]);
      bad |= inv::f16_overflow(o.x) | inv::f16_overflow(o.y) | inv::f16_overflow(o.z) | inv::f16_overflow(o.w);
      uint2 hv, lv;
      hv.x = (uint32_t)__half_as_ushort(h[0]) | ((uint32_t)__half_as_ushort(h[1]) << 16);
      hv.y = (uint32_t)__half_as_ushort(h[2]) | ((uint32_t)__half_as_ushort(h[3]) << 16);
      lv.x = (uint32_t)__half_as_ushort(l[0]) | ((uint32_t)__half_as_ushort(l[1]) << 16);
      lv.y = (uint32_t)__half_as_ushort(l[2]) | ((uint32_t)__half_as_ushort(l[3]) << 16);
      reinterpret_cast<uint2*>(yh + row * hidden)[i] = hv;
      reinterpret_cast<uint2*>(yl + row * hidden)[i] = lv;
    }
  }
  if (bad) record_status(status, INV_ERR_RANGE);
}

// ------------------------------------------------------------- quantiser ----

// Quantise one (token, kv head) row of 128 values held as one float4 per lane.
__device__ __forceinline__ void quant_store_row(float4 v, int16_t* __restrict__ codes, float* __restrict__ scale,
                                                int lane) {
  float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));  // exact
  const float s = __fdiv_rn(m, 32767.0f);
  int q[4] = {0, 0, 0, 0};
  if (s != 0.0f) {
    const float in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int t = __float2int_rn(__fdiv_rn(in[j], s));  // IEEE division, round half to even
      q[j] = t > 32767 ? 32767 : (t < -32767 ? -32767 : t);
    }
  }
  uint2 packed;
  packed.x = (uint32_t)(uint16_t)q[0] | ((uint32_t)(uint16_t)q[1] << 16);
  packed.y = (uint32_t)(uint16_t)q[2] | ((uint32_t)(uint16_t)q[3] << 16);
  reinterpret_cast<uint2*>(codes)[lane] = packed;
  if (lane == 0) *scale = s;
}

// One warp per (token, kv head).
__global__ void kv_quant_kernel(const float* __restrict__ x, int T, int64_t ld_x, const int32_t* __restrict__ slot,
                                const int32_t* __restrict__ pos, inv_kv_cache c, int which, int* status) {
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int H = c.n_kv_heads;
  if (warp >= (int64_t)T * H) return;
  const int t = (int)(warp / H), h = (int)(warp - (int64_t)t * H);
  const int sl = slot[t], p = pos[t];
  if (sl < 0 || sl >= c.n_slots || p < 0 || p >= c.max_len) {
    if (lane == 0) record_status(status, INV_ERR_INVALID_ARG);
    return;
  }
  const int64_t ix = (int64_t)t * ld_x + (int64_t)h * 128;
  const int64_t rowi = ((int64_t)sl * H + h) * c.max_len + p;
  [[maybe_unused]] const int64_t n_rows = (int64_t)c.n_slots * H * c.max_len;  // cache rows
  if (!INV_SPAN_IN_BOUNDS(status, ix, ix + 127, (int64_t)(T - 1) * ld_x + (int64_t)H * 128) ||
      !INV_IN_BOUNDS(status, rowi, n_rows))
    return;
  const float4 v = reinterpret_cast<const float4*>(x + ix)[lane];
  int16_t* codes = (which == 0 ? c.k : c.v) + rowi * 128;
  float* scale = (which == 0 ? c.k_scale : c.v_scale) + rowi;
  quant_store_row(v, codes, scale, lane);
}

__global__ void embed_kernel(const float* __restrict__ table, int vocab, int hidden, const int32_t* __restrict__ ids,
                             int B, float* __restrict__ x, int* status) {
  const int b = blockIdx.x;
  const int id = ids[b];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) record_status(status, INV_ERR_INVALID_ARG);
  for (int i = threadIdx.x; i < hidden; i += blockDim.x) {
    const int64_t ix = (int64_t)b * hidden + i, it = (int64_t)id * hidden + i;
    if (!INV_IN_BOUNDS(status, ix, (int64_t)B * hidden) || (ok && !INV_IN_BOUNDS(status, it, (int64_t)vocab * hidden)))
      continue;
    x[ix] = ok ? table[it] : 0.0f;
  }
}

// Greedy argmax per row: lowest index among the maxima (NaN ignored).
__global__ void argmax_kernel(const float* __restrict__ logits, int n, int64_t ld, int32_t* __restrict__ ids,
                              int* status) {
  __shared__ float bv[32];
  __shared__ int bi[32];
  const int64_t b = blockIdx.x;  // logits [B = gridDim.x] rows of ld, the last one n long
  float best = -INFINITY;
  int besti = 0x7fffffff;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    if (!INV_IN_BOUNDS(status, b * ld + j, ((int64_t)gridDim.x - 1) * ld + n)) continue;
    const float v = logits[b * ld + j];
    if (v > best || (v == best && j < besti)) { best = v; besti = j; }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
    if (ov > best || (ov == best && oi < besti)) { best = ov; besti = oi; }
  }
  if ((threadIdx.x & 31) == 0) { bv[threadIdx.x >> 5] = best; bi[threadIdx.x >> 5] = besti; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (bv[w] > best || (bv[w] == best && bi[w] < besti)) { best = bv[w]; besti = bi[w]; }
    if (INV_IN_BOUNDS(status, b, gridDim.x)) ids[b] = besti == 0x7fffffff ? 0 : besti;
  }
}

// cos/sin(p * base^(-2i/128)) in double precision, rounded once to fp32.
__global__ void rope_table_kernel(int max_pos, double base, float* __restrict__ cs, float* __restrict__ sn,
                                  int* status) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (idx >= (int64_t)max_pos * 64 || !INV_IN_BOUNDS(status, idx, (int64_t)max_pos * 64)) return;
  const int p = (int)(idx / 64), i = (int)(idx % 64);
  const double theta = pow(base, -2.0 * i / 128.0);
  double sv, cv;
  sincos((double)p * theta, &sv, &cv);
  cs[idx] = (float)cv;
  sn[idx] = (float)sv;
}

int grid_for(int64_t work, int threads) {
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)inv::sm_count() * 16;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

}  // namespace

// ---------------------------------------------------------- internal API ----

namespace inv {

int launch_rmsnorm(const float* x, const float* gamma, int64_t rows, int hidden, float eps, float* y,
                   uint16_t* yh, uint16_t* yl, cudaStream_t s) {
  if (rows == 0) return INV_OK;
  __half* h = reinterpret_cast<__half*>(yh);
  __half* l = reinterpret_cast<__half*>(yl);
  const int n4 = hidden / 4;
  if (n4 <= kNormThreads)
    rmsnorm_reg_kernel<1><<<(unsigned)rows, kNormThreads, 0, s>>>(x, gamma, hidden, eps, y, h, l, status_ptr());
  else if (n4 <= 2 * kNormThreads)
    rmsnorm_reg_kernel<2><<<(unsigned)rows, kNormThreads, 0, s>>>(x, gamma, hidden, eps, y, h, l, status_ptr());
  else if (n4 <= 4 * kNormThreads)
    rmsnorm_reg_kernel<4><<<(unsigned)rows, kNormThreads, 0, s>>>(x, gamma, hidden, eps, y, h, l, status_ptr());
  else if (n4 <= 8 * kNormThreads)
    rmsnorm_reg_kernel<8><<<(unsigned)rows, kNormThreads, 0, s>>>(x, gamma, hidden, eps, y, h, l, status_ptr());
  else
    rmsnorm_kernel<<<(unsigned)rows, kNormThreads, 0, s>>>(x, gamma, hidden, eps, y, h, l, status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

}  // namespace inv

// ------------------------------------------------------------ public C ABI ----

extern "C" {

int heal_split(const float* x, int64_t rows, int64_t cols, int64_t ld_x, uint16_t* hi, uint16_t* lo,
               int64_t ld_out, inv_stream stream) {
  if (rows < 0 || cols < 0 || ld_x < cols || ld_out < cols) return INV_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return INV_OK;
  if (!x || !hi || !lo) return INV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int threads = 256;
  const bool vec = (cols % 4 == 0) && (ld_x % 4 == 0) && (ld_out % 4 == 0) && inv::aligned16(x) &&
                   ((reinterpret_cast<uintptr_t>(hi) & 7u) == 0) && ((reinterpret_cast<uintptr_t>(lo) & 7u) == 0);
  if (vec) {
    heal_split_vec_kernel<<<grid_for(rows * (cols / 4), threads), threads, 0, s>>>(
        reinterpret_cast<const float4*>(x), rows, cols / 4, ld_x / 4, reinterpret_cast<uint2*>(hi),
        reinterpret_cast<uint2*>(lo), ld_out / 4, inv::status_ptr());
  } else {
    heal_split_kernel<<<grid_for(rows * ((cols + 3) / 4), threads), threads, 0, s>>>(
        x, rows, cols, ld_x, reinterpret_cast<__half*>(hi), reinterpret_cast<__half*>(lo), ld_out,
        inv::status_ptr());
  }
  INV_CHECK_LAUNCH();
  return INV_OK;
}

size_t heal_packed_weight_bytes(int K, int N) {
  if (K <= 0 || N <= 0) return 0;
  return (size_t)K * (size_t)N * 2u * sizeof(uint16_t);
}

int heal_pack_weight(const float* W, int K, int N, uint16_t* packed, size_t packed_bytes, int8_t* col_exp,
                     inv_stream stream) {
  if (!W || !packed || !col_exp || K <= 0 || N <= 0) return INV_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % INV_GEMM_BN != 0) return INV_ERR_UNSUPPORTED_SHAPE;
  if (packed_bytes < heal_packed_weight_bytes(K, N)) return INV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  col_exp_kernel<<<(N + 255) / 256, 256, 0, s>>>(W, K, N, col_exp, inv::status_ptr());
  INV_CHECK_LAUNCH();
  pack_kernel<<<dim3(N / 64, K / 64), 256, 0, s>>>(W, K, N, col_exp, reinterpret_cast<__half*>(packed),
                                                   inv::status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

int rmsnorm_bi(const float* x, const float* gamma, int64_t rows, int hidden, float eps, float* y, uint16_t* y_hi,
               uint16_t* y_lo, inv_stream stream) {
  if (rows < 0 || hidden <= 0) return INV_ERR_INVALID_ARG;
  if (hidden % 4 != 0) return INV_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return INV_OK;
  if (!x || !gamma || (!y && !y_hi) || ((y_hi == nullptr) != (y_lo == nullptr))) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(x) || !inv::aligned16(gamma) || (y && !inv::aligned16(y)) ||
      (y_hi && ((reinterpret_cast<uintptr_t>(y_hi) | reinterpret_cast<uintptr_t>(y_lo)) & 7u)))
    return INV_ERR_INVALID_ARG;
  if (rows > 0x7fffffff) return INV_ERR_UNSUPPORTED_SHAPE;
  return inv::launch_rmsnorm(x, gamma, rows, hidden, eps, y, y_hi, y_lo, static_cast<cudaStream_t>(stream));
}

int kv_quant_int16(const float* x, int T, int64_t ld_x, const int32_t* slot, const int32_t* pos,
                   const inv_kv_cache* cache, int which, inv_stream stream) {
  if (!cache || T < 0 || (which != 0 && which != 1)) return INV_ERR_INVALID_ARG;
  if (cache->head_dim != INV_HEAD_DIM) return INV_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return INV_OK;
  if (!x || !slot || !pos || !cache->k || !cache->v || !cache->k_scale || !cache->v_scale) return INV_ERR_INVALID_ARG;
  if (cache->n_kv_heads <= 0 || cache->n_slots <= 0 || cache->max_len <= 0) return INV_ERR_INVALID_ARG;
  if (ld_x < (int64_t)cache->n_kv_heads * 128 || ld_x % 4 != 0 || !inv::aligned16(x)) return INV_ERR_INVALID_ARG;
  const int64_t warps = (int64_t)T * cache->n_kv_heads;
  const int threads = 256;
  kv_quant_kernel<<<(unsigned)((warps * 32 + threads - 1) / threads), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      x, T, ld_x, slot, pos, *cache, which, inv::status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

int rope_tables(int max_pos, double base, float* cos_out, float* sin_out, inv_stream stream) {
  if (max_pos <= 0 || !(base > 0.0) || !cos_out || !sin_out) return INV_ERR_INVALID_ARG;
  const int64_t n = (int64_t)max_pos * 64;
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      max_pos, base, cos_out, sin_out, inv::status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

int embed_gather(const float* table, int vocab, int hidden, const int32_t* ids, int B, float* x, inv_stream stream) {
  if (vocab <= 0 || hidden <= 0 || B < 0) return INV_ERR_INVALID_ARG;
  if (B == 0) return INV_OK;
  if (!table || !ids || !x) return INV_ERR_INVALID_ARG;
  embed_kernel<<<B, 256, 0, static_cast<cudaStream_t>(stream)>>>(table, vocab, hidden, ids, B, x, inv::status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

int argmax_rows(const float* logits, int B, int n, int64_t ld, int32_t* ids, inv_stream stream) {
  if (B < 0 || n <= 0 || ld < n) return INV_ERR_INVALID_ARG;
  if (B == 0) return INV_OK;
  if (!logits || !ids) return INV_ERR_INVALID_ARG;
  argmax_kernel<<<B, 1024, 0, static_cast<cudaStream_t>(stream)>>>(logits, n, ld, ids, inv::status_ptr());
  INV_CHECK_LAUNCH();
  return INV_OK;
}

}  // extern "C"
