// Packed <-> padded copies of variable-length batches (the pad / unpad pair
// flash-sparse-attention PR #197 wires next to the varlen entry point,
// Changes list): sequence b holds rows [cu[b], cu[b+1]) of a packed
// [total, heads, d] tensor and rows [0, cu[b+1] - cu[b]) of a padded
// [batch, max_len, heads, d] one.  One thread per 16-byte chunk of a row.
#include "device_common.cuh"
#include "kernels.h"

namespace sma {
namespace {

// pad: padded row (b, t) <- packed row cu[b] + t, or zeros past the length.
__global__ void varlen_pad_kernel(const uint8_t* __restrict__ packed, uint8_t* __restrict__ padded,
                                  const int32_t* __restrict__ cu, int max_len, int heads, int cpr,
                                  int esz, int64_t p_row, int64_t p_head, int64_t d_sb,
                                  int64_t d_sr, int64_t d_sh) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  const int64_t per_row = static_cast<int64_t>(heads) * cpr;
  if (t >= static_cast<int64_t>(max_len) * per_row) return;
  const int row = static_cast<int>(t / per_row);
  const int rem = static_cast<int>(t - static_cast<int64_t>(row) * per_row);
  const int h = rem / cpr, ch = rem - h * cpr;
  const int len = cu[b + 1] - cu[b];
  uint4 v = make_uint4(0, 0, 0, 0);
  if (row < len)
    v = *reinterpret_cast<const uint4*>(packed + ((cu[b] + static_cast<int64_t>(row)) * p_row + h * p_head) * esz + ch * 16);
  *reinterpret_cast<uint4*>(padded + (b * d_sb + static_cast<int64_t>(row) * d_sr + h * d_sh) * esz + ch * 16) = v;
}

// unpad: packed row cu[b] + t <- padded row (b, t), for t below the length.
__global__ void varlen_unpad_kernel(const uint8_t* __restrict__ padded, uint8_t* __restrict__ packed,
                                    const int32_t* __restrict__ cu, int max_len, int heads, int cpr,
                                    int esz, int64_t p_row, int64_t p_head, int64_t s_sb,
                                    int64_t s_sr, int64_t s_sh) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  const int64_t per_row = static_cast<int64_t>(heads) * cpr;
  if (t >= static_cast<int64_t>(max_len) * per_row) return;
  const int row = static_cast<int>(t / per_row);
  const int rem = static_cast<int>(t - static_cast<int64_t>(row) * per_row);
  const int h = rem / cpr, ch = rem - h * cpr;
  const int len = cu[b + 1] - cu[b];
  if (row >= len) return;
  const uint4 v = *reinterpret_cast<const uint4*>(padded + (b * s_sb + static_cast<int64_t>(row) * s_sr + h * s_sh) * esz + ch * 16);
  *reinterpret_cast<uint4*>(packed + ((cu[b] + static_cast<int64_t>(row)) * p_row + h * p_head) * esz + ch * 16) = v;
}

}  // namespace

cudaError_t launch_varlen_pad(const void* packed, void* padded, const int32_t* cu, int batch,
                              int max_len, int heads, int d, int esz, int64_t p_row, int64_t p_head,
                              int64_t d_sb, int64_t d_sr, int64_t d_sh, cudaStream_t stream) {
  const int cpr = d * esz / 16;
  const int64_t n = static_cast<int64_t>(max_len) * heads * cpr;
  if (n == 0 || batch == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((n + 255) / 256), batch);
  varlen_pad_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(packed),
                                              static_cast<uint8_t*>(padded), cu, max_len, heads, cpr,
                                              esz, p_row, p_head, d_sb, d_sr, d_sh);
  return cudaGetLastError();
}

cudaError_t launch_varlen_unpad(const void* padded, void* packed, const int32_t* cu, int batch,
                                int max_len, int heads, int d, int esz, int64_t p_row,
                                int64_t p_head, int64_t s_sb, int64_t s_sr, int64_t s_sh,
                                cudaStream_t stream) {
  const int cpr = d * esz / 16;
  const int64_t n = static_cast<int64_t>(max_len) * heads * cpr;
  if (n == 0 || batch == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((n + 255) / 256), batch);
  varlen_unpad_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(padded),
                                                static_cast<uint8_t*>(packed), cu, max_len, heads,
                                                cpr, esz, p_row, p_head, s_sb, s_sr, s_sh);
  return cudaGetLastError();
}

}  // namespace sma
