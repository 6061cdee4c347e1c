// Per-context state of the library: the device error word kernels report
// into, and the SM count used to size persistent grids.
#include <cudaTypedefs.h>

#include <mutex>

#include "device_common.cuh"
#include "kernels.h"

namespace sma {

namespace {
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mutex;
ContextAddressCache g_error_cache;

PFN_cuCtxGetCurrent_v4000 g_ctx_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_get_id = nullptr;
std::once_flag g_ctx_fns_once;

void load_ctx_fns() {
  cudaDriverEntryPointQueryResult q;
  void* f = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  f = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
}
}  // namespace

unsigned long long current_context_id() {
  std::call_once(g_ctx_fns_once, load_ctx_fns);
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return 0;
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (g_ctx_get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

void* ContextAddressCache::find(unsigned long long ctx_id) {
  if (ctx_id == 0) return nullptr;
  std::lock_guard<std::mutex> lock(mutex);
  for (int i = 0; i < count; ++i)
    if (ids[i] == ctx_id) return ptrs[i];
  return nullptr;
}

void ContextAddressCache::insert(unsigned long long ctx_id, void* ptr) {
  if (ctx_id == 0) return;
  std::lock_guard<std::mutex> lock(mutex);
  for (int i = 0; i < count; ++i)
    if (ids[i] == ctx_id) {
      ptrs[i] = ptr;
      return;
    }
  const int slot = count < kSlots ? count++ : static_cast<int>(next_evict++ % kSlots);
  ids[slot] = ctx_id;
  ptrs[slot] = ptr;
}

int* device_error_word(cudaError_t* status) {
  void* p = g_error_cache.find(current_context_id());
  if (p == nullptr) {
    const cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess || p == nullptr) {
      if (status) *status = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    // the lookup makes the device's primary context current if none was
    g_error_cache.insert(current_context_id(), p);
  }
  if (status) *status = cudaSuccess;
  return static_cast<int*>(p);
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
