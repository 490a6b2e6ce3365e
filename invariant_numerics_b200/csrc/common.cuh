// Device and host helpers shared by the libinvnum kernels (sm_100a only).
//
// PTX wrappers for mbarriers, TMA (cp.async.bulk / cp.async.bulk.tensor, each
// CTA loading only into its own shared memory), tcgen05 tensor-memory MMAs,
// and the bounded waits
// every kernel uses: a wait that exceeds the configured number of nanoseconds
// of GPU global time records INV_ERR_TIMEOUT in the status word and lets the
// kernel release what it holds and return.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "invnum.h"

namespace inv {

// ---------------------------------------------------------------- host side --

// Device status word of the current device (cudaGetSymbolAddress, cached).
int* status_ptr();
// Wait bound in ns for kernels launched now.
long long wait_limit_ns();
// decode_layer kernel tracing (see inv_trace_events).
void set_trace(void** events, int n);
void trace_record(int slot, cudaStream_t s);
// Number of SMs of the current device (cached).
int sm_count();
// cuTensorMapEncodeTiled through the runtime's driver entry point.
int make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                       uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                       uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

#define INV_CHECK_LAUNCH()                              \
  do {                                                  \
    if (cudaGetLastError() != cudaSuccess) return INV_ERR_CUDA; \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// -------------------------------------------------------------- device side --

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);  // first error wins
}

// Index checks of the INV_DEBUG_BOUNDS build: INV_IN_BOUNDS(status, i, n) is
// true when 0 <= i < n, else it records INV_ERR_BOUNDS and is false;
// INV_SPAN_IN_BOUNDS(status, first, last, n) checks a block accessed as a
// whole by its first and last index.  The normal build compiles both to true
// without evaluating the arguments.
#ifdef INV_DEBUG_BOUNDS
#define INV_IN_BOUNDS(status, i, n) ::inv::in_bounds((status), (int64_t)(i), (int64_t)(n))
#define INV_SPAN_IN_BOUNDS(status, first, last, n) \
  ::inv::span_in_bounds((status), (int64_t)(first), (int64_t)(last), (int64_t)(n))
#else
#define INV_IN_BOUNDS(status, i, n) true
#define INV_SPAN_IN_BOUNDS(status, first, last, n) true
#endif
__device__ __forceinline__ bool in_bounds(int* status, int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  record_status(status, INV_ERR_BOUNDS);
  return false;
}
__device__ __forceinline__ bool span_in_bounds(int* status, int64_t first, int64_t last, int64_t n) {
  if (first >= 0 && first <= last && last < n) return true;
  record_status(status, INV_ERR_BOUNDS);
  return false;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity.  Returns false when the wait gave
// up: either `limit_ns` of global time passed (INV_ERR_TIMEOUT is recorded and
// *abort is set) or another thread already set *abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit_ns,
                                          volatile int* abort, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort != nullptr && *abort) return false;
    if ((i & 63u) == 0 && (long long)(global_ns() - t0) > limit_ns) {
      record_status(status, INV_ERR_TIMEOUT);
      if (abort != nullptr) *abort = 1;
      return false;
    }
  }
}

// --------------------------------------------- producer/consumer grids ----
// A kernel launched as a programmatic dependent of the running one may start
// once every CTA of the running grid has executed grid_launch_dependents (or
// exited); grid_wait_prerequisites blocks until the prerequisite grid has
// completed and its memory is visible (immediately without one).
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Release add at GPU scope: the calling thread's earlier writes (and those
// ordered before it, e.g. by __syncwarp) are visible to a thread that observes
// the new value and then executes fence_acquire_gpu.
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// Orders this thread's generic-proxy view of global memory before its later
// async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 2-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c_inner, int c_outer) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c_inner), "r"(c_outer)
      : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing
// on `bar`; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ------------------------------------------------------------ tcgen05 / TMEM --

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (binary16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every previously issued tcgen05.mma of this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (the layout a SWIZZLE_128B TMA box
// of 64 binary16 x R rows produces).  Bits: [0,14) start>>4, [16,30) leading
// byte offset>>4 (unused for swizzled K-major), [32,46) stride byte
// offset>>4, [46,48) descriptor version 1, [61,64) swizzle mode 2 = 128B.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A/B binary16, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B: f16
         | (0u << 15) | (0u << 16)                   // K-major A and B
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------------------ binary16 split --

// hi = rn16(x); lo = rn16((x - hi) * 2^11).  x - hi is exact in fp32 whenever
// hi is finite; the product by 2^11 is an exact scaling.
__device__ __forceinline__ void split_hi_lo(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  const float r = __fsub_rn(x, __half2float(hi));
  lo = __float2half_rn(__fmul_rn(r, 2048.0f));
}

__device__ __forceinline__ bool f16_overflow(float x) { return fabsf(x) >= 65520.0f; }

__device__ __forceinline__ float pow2f(int e) {  // exact 2^e for -126 <= e <= 127
  return __int_as_float((127 + e) << 23);
}

}  // namespace inv
