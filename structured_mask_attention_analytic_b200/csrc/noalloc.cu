// dfa_attn_fwd_noalloc: the DFlash attention forward for callers that cannot
// hand the library a device workspace.
//
// Some callers have no way to allocate device memory for us: a plain C host
// program that links libsma without any CUDA memory manager of its own, or a
// runtime whose device memory is entirely pre-reserved by another allocator
// (a framework's caching pool or a fixed arena), where an extra cudaMalloc
// would fail or fragment that pool.  This entry point keeps the one piece of
// scratch the forward needs -- the block map of full/partial key tiles -- in
// a fixed array compiled into the library, so the caller passes only inputs
// and outputs.
//
// Limits and behaviour:
// * The array is kNoAllocScratchBytes (4 MiB) of device memory that every GPU
//   which loads the library holds until the process exits.  Problems whose
//   block map needs more (batch * ceil(q_len/128) * (ceil(k_len/128) + 1) *
//   8 bytes, plus alignment) are rejected with SMA_ERR_WORKSPACE; use
//   dfa_attn_fwd with a caller workspace for those.  Short-query problems
//   split each unit's key tiles over several SMs only when the partial
//   results fit in the array beside the block map.
// * Every call shares the array and overwrites it.  Calls that can run at the
//   same time on the GPU (e.g. on two streams without ordering between them)
//   race on it; order them on one stream.  Nothing in the array needs to start
//   at zero: each call rewrites every entry it later reads.
// * The first call in a CUDA context looks the array's device address up
//   (with that context current) and caches it for that context; make that
//   first call before any stream capture begins.  A new context (after
//   cudaDeviceReset, or a caller's own non-primary context) gets its own
//   lookup on its first call, since the address belongs to the context the
//   library's module is loaded in.
// * No cudaMalloc, cudaFree or other allocating routine is called.
#include <cuda_runtime.h>

#include <cstdio>

#include "kernels.h"
#include "sma.h"

namespace sma {
size_t dfa_fwd_map_bytes(const dfa_mask_desc* desc);
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

// In host code this name is only a stand-in for the symbol, not a device
// address; the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_dfa_scratch[kNoAllocScratchBytes];

sma::ContextAddressCache g_scratch_cache;

}  // namespace

extern "C" sma_status dfa_attn_fwd_noalloc(const dfa_mask_desc* desc, const int32_t* anchors,
                                           int32_t dtype, int32_t heads, int32_t kv_heads,
                                           int32_t head_dim, float scale, const void* q,
                                           const int64_t q_strides[3], const void* k,
                                           const int64_t k_strides[3], const void* v,
                                           const int64_t v_strides[3], void* out,
                                           const int64_t o_strides[3], float* lse, void* stream) {
  size_t full = 0;  // validates the arguments
  sma_status s = dfa_attn_fwd_workspace_size(desc, heads, kv_heads, head_dim, &full);
  if (s != SMA_OK) return s;
  // the block map must fit; the key-range split's partials are used only if
  // they fit as well
  const size_t need = sma::dfa_fwd_map_bytes(desc);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "dfa_attn_fwd_noalloc: this problem's block map needs %zu bytes, above the %zu-byte "
             "scratch array the entry point holds; call dfa_attn_fwd with a workspace instead",
             need, kNoAllocScratchBytes);
    return sma::set_last_error(SMA_ERR_WORKSPACE, msg);
  }
  void* ptr = g_scratch_cache.find(sma::current_context_id());
  if (ptr == nullptr) {
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_dfa_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "dfa_attn_fwd_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      return sma::set_last_error(SMA_ERR_CUDA, msg);
    }
    // the lookup makes the device's primary context current if none was
    g_scratch_cache.insert(sma::current_context_id(), ptr);
  }
  return dfa_attn_fwd(desc, anchors, dtype, heads, kv_heads, head_dim, scale, q, q_strides, k,
                      k_strides, v, v_strides, out, o_strides, lse, nullptr, ptr,
                      kNoAllocScratchBytes, stream);
}
