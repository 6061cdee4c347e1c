// TMA tensor-map encoding through the driver entry point (no libcuda link).
#include <cudaTypedefs.h>

#include <cstdio>

#include "sma.h"
#include "tma_map.h"

namespace sma {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

}  // namespace

// 4D map over [B][len][heads][d] (d contiguous), box = 64 x box_heads x
// (128 / box_heads) x 1, 128-byte swizzle, zero fill outside the tensor.
bool encode_map(CUtensorMap* map, const void* ptr, int dtype, int d, int heads, int len, int batch,
                int64_t s_head, int64_t s_row, int64_t s_batch, char* msg, size_t msg_len,
                int box_heads) {
  auto enc = get_encode_fn();
  if (enc == nullptr) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled is unavailable");
    return false;
  }
  const int esz = 2;
  // A size-1 dim's stride is never used; give it a legal value.
  if (heads == 1) s_head = d;
  if (len == 1) s_row = s_head * heads;
  if (batch == 1) s_batch = s_row * len;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(len), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s_head * esz),
                           static_cast<cuuint64_t>(s_row * esz),
                           static_cast<cuuint64_t>(s_batch * esz)};
  if (box_heads < 1 || box_heads > heads || SMA_TILE % box_heads != 0) {
    snprintf(msg, msg_len, "invalid heads per TMA box (%d)", box_heads);
    return false;
  }
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_heads),
                       static_cast<cuuint32_t>(SMA_TILE / box_heads), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dtype == SMA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return false;
  }
  return true;
}

bool encode_map_f32(CUtensorMap* map, const void* ptr, int d, int heads, int len, int batch,
                    int box_d, int box_rows, char* msg, size_t msg_len) {
  auto enc = get_encode_fn();
  if (enc == nullptr) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled is unavailable");
    return false;
  }
  const uint64_t s_head = static_cast<uint64_t>(d) * 4;
  const uint64_t s_row = s_head * heads;
  const uint64_t s_batch = s_row * len;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(len), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {s_head, s_row, s_batch};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_d), 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled (float32 accumulator) failed (%d)",
             static_cast<int>(r));
    return false;
  }
  return true;
}

}  // namespace sma
