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
