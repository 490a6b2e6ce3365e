// Host runtime of libinvnum: the per-device status word, the wait bound,
// tensor-map encoding and the bounded-wait self-test.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace {

__device__ int g_inv_status;  // first device-side error since the last read

constexpr int kMaxDevices = 64;
int* g_status_addr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;
std::atomic<long long> g_wait_ns{2000000000LL};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

}  // namespace

namespace inv {

int* status_ptr() {
  const int d = current_device();
  if (d < 0) return nullptr;
  if (g_status_addr[d] == nullptr) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_status_addr[d] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_inv_status) != cudaSuccess) return nullptr;
      g_status_addr[d] = static_cast<int*>(p);
    }
  }
  return g_status_addr[d];
}

long long wait_limit_ns() { return g_wait_ns.load(); }

namespace {
void** g_trace = nullptr;
int g_trace_n = 0;
}  // namespace

void set_trace(void** events, int n) {
  g_trace = events;
  g_trace_n = n;
}

void trace_record(int slot, cudaStream_t s) {
  if (g_trace != nullptr && slot >= 0 && slot < g_trace_n && g_trace[slot] != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(g_trace[slot]), s);
}

int sm_count() {
  const int d = current_device();
  if (d < 0) return 148;
  if (g_sm_count[d] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[d] = n;
  }
  return g_sm_count[d];
}

int make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                       uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                       CUtensorMapSwizzle swizzle) {
  if (g_encode == nullptr) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return INV_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? INV_OK : INV_ERR_CUDA;
}

}  // namespace inv

namespace {

// One CTA waits on a barrier that nothing arrives at; the bounded wait must
// give up after `limit_ns` and record INV_ERR_TIMEOUT.
__global__ void selftest_wait_kernel(int* status, long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    inv::mbar_init(&bar, 1);
    abort_flag = 0;
    inv::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) inv::mbar_wait(&bar, 0, limit_ns, &abort_flag, status);
  __syncthreads();
}

// Stores i to buf[i] for i < n_written under the index check with extent
// n_declared (launched only by the checking build).
__global__ void selftest_bounds_kernel(float* buf, int n_declared, int n_written, int* status) {
#ifdef INV_DEBUG_BOUNDS
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_written; i += gridDim.x * blockDim.x)
    if (INV_IN_BOUNDS(status, i, n_declared)) buf[i] = (float)i;
#endif
}

}  // namespace

extern "C" {

const char* inv_status_string(int status) {
  switch (status) {
    case INV_OK: return "INV_OK";
    case INV_ERR_INVALID_ARG: return "INV_ERR_INVALID_ARG";
    case INV_ERR_UNSUPPORTED_SHAPE: return "INV_ERR_UNSUPPORTED_SHAPE";
    case INV_ERR_WORKSPACE: return "INV_ERR_WORKSPACE";
    case INV_ERR_CUDA: return "INV_ERR_CUDA";
    case INV_ERR_RANGE: return "INV_ERR_RANGE";
    case INV_ERR_TIMEOUT: return "INV_ERR_TIMEOUT";
    case INV_ERR_BOUNDS: return "INV_ERR_BOUNDS";
    default: return "INV_ERR_UNKNOWN";
  }
}

int inv_version(void) { return 1; }

int inv_get_device_status(int* status_out, inv_stream stream) {
  if (status_out == nullptr) return INV_ERR_INVALID_ARG;
  int* p = inv::status_ptr();
  if (p == nullptr) return INV_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return INV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return INV_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return INV_ERR_CUDA;
  *status_out = v;
  return INV_OK;
}

int inv_trace_events(void** events, int n_events) {
  if (events == nullptr || n_events <= 0) {
    inv::set_trace(nullptr, 0);
    return INV_OK;
  }
  if (n_events < 2 * INV_DECODE_LAYER_KERNELS) return INV_ERR_INVALID_ARG;
  inv::set_trace(events, n_events);
  return INV_OK;
}

int inv_set_wait_limit_ns(long long ns) {
  g_wait_ns.store(ns > 0 ? ns : 2000000000LL);
  return INV_OK;
}

int inv_selftest_wait_timeout(long long wait_ns, inv_stream stream) {
  if (wait_ns <= 0) return INV_ERR_INVALID_ARG;
  int* st = inv::status_ptr();
  if (st == nullptr) return INV_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(st, wait_ns);
  INV_CHECK_LAUNCH();
  return INV_OK;
}

int inv_debug_bounds_enabled(void) {
#ifdef INV_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

int inv_selftest_bounds(float* buf, int n_declared, int n_written, inv_stream stream) {
  if (buf == nullptr || n_declared < 0 || n_written < n_declared) return INV_ERR_INVALID_ARG;
  if (!inv_debug_bounds_enabled()) return INV_ERR_UNSUPPORTED_SHAPE;
  if (n_written == 0) return INV_OK;
  int* st = inv::status_ptr();
  if (st == nullptr) return INV_ERR_CUDA;
  selftest_bounds_kernel<<<(n_written + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(buf, n_declared,
                                                                                                 n_written, st);
  INV_CHECK_LAUNCH();
  return INV_OK;
}

}  // extern "C"
