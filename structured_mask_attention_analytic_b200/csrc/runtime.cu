// Per-device state of the library: the device error word kernels report
// into, and the SM count used to size persistent grids.
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"

namespace sma {

namespace {
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int* g_error_ptr[kMaxDevices] = {nullptr};
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mutex;
}  // namespace

int* device_error_word(cudaError_t* status) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    if (status) *status = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_error_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) {
      if (status) *status = e;
      return nullptr;
    }
    g_error_ptr[dev] = static_cast<int*>(p);
  }
  if (status) *status = cudaSuccess;
  return g_error_ptr[dev];
}

namespace {
// Waits on an mbarrier that nothing arrives on, with the same bounded wait the
// pipelines use, and reports what happened.  out[0] = 1 if the wait gave up,
// out[1] = nanoseconds spent.
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns, int* err, int64_t* out) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_timer_ns();
    const bool ok = mbar_wait_for(smem_u32(&bar), 0, &abort_flag, err, timeout_ns);
    out[0] = ok ? 0 : 1;
    out[1] = static_cast<int64_t>(global_timer_ns() - t0);
  }
}
}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, int* err, int64_t* out,
                                         cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(timeout_ns, err, out);
  return cudaGetLastError();
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

}  // namespace sma
