// Index-gather preparation for attention under a query-broadcast keep mask,
// such as the dynamic top-k mask of flash-sparse-attention PR #197 (one
// selection per (batch, KV head) row, shared by every query; Usage and
// Implementation notes).
//
// Walking all 128-key tiles of the original key range would leave every tile
// PARTIAL with only the selected fraction of its keys alive.  Instead the
// selected keys of each gather row are listed in ascending order, their K/V
// rows (and bias columns) are copied into dense compacted operands, and the
// attention kernels run over those.  The softmax over the kept set does not
// depend on the order of the keys, so the result is the masked attention's.
// Causal masking on the original indices becomes a per-row limit on the
// compacted index (gather_row_limit).
//
//   select_keys_kernel   one CTA per gather row: ascending kept indices
//   gather_kv_kernel     one thread per 16-byte chunk of a compacted K/V row
//   gather_bias_kernel   one thread per compacted bias column
//   gather_lists_kernel  FULL / PARTIAL tile lists over the compacted keys
#include "device_common.cuh"
#include "gather.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kSelThreads = 256;

// Stream compaction of one mask row: each thread takes 4 columns per step, a
// block-wide exclusive scan of the kept counts gives the output positions.
__global__ void __launch_bounds__(kSelThreads)
select_keys_kernel(const uint8_t* __restrict__ mask, int64_t m_sb, int64_t m_sh, int m_kd, int LH,
                   int Lk, int cap, int32_t* __restrict__ idx, int32_t* __restrict__ count, int* err) {
  const int grow = blockIdx.x;
  const int lb = grow / LH, lh = grow - lb * LH;
  const uint8_t* row = mask + lb * m_sb + lh * m_sh;
  int32_t* out = idx + static_cast<int64_t>(grow) * cap;
  __shared__ uint32_t s_warp[kSelThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t base = 0;
  const int kpad = (Lk + kTile - 1) / kTile * kTile;
  for (int c0 = 0; c0 < kpad; c0 += kSelThreads * 4) {
    const int c = c0 + threadIdx.x * 4;
    uint32_t bits = 0;
    if (c + 4 <= m_kd) {  // c is a multiple of 4
      const uint32_t wv = *reinterpret_cast<const uint32_t*>(row + c);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (((wv >> (8 * e)) & 0xffu) != 0u && c + e < Lk) bits |= 1u << e;
    } else if (c < kpad) {  // a row of Lk columns ends here, or one column stands for every key
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c + e < Lk && row[aux_col(c + e, m_kd)] != 0) bits |= 1u << e;
    }
    const uint32_t n = __popc(bits);
    uint32_t incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    uint32_t wb = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
      const uint32_t sw = s_warp[w];
      wb += w < warp ? sw : 0u;
      tot += sw;
    }
    __syncthreads();  // s_warp is rewritten by the next step
    uint32_t pos = base + wb + incl - n;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((bits >> e) & 1u) {
        if (pos < static_cast<uint32_t>(cap)) out[pos] = c + e;
        ++pos;
      }
    }
    base += tot;
  }
  if (threadIdx.x == 0) {
    if (base > static_cast<uint32_t>(cap)) {
      report_error(err, SMA_ERR_DEVICE_INPUT);  // more kept keys than the stated maximum
      base = static_cast<uint32_t>(cap);
    }
    count[grow] = static_cast<int32_t>(base);
  }
}

// Compacted row j of (b, kv head): original row idx[j] for j < count, zeros
// up to the end of the last tile in use (V must be finite there: P is 0 on
// those columns but 0 * NaN would poison O), untouched beyond.
__global__ void gather_kv_kernel(const AttnProblem p, const uint8_t* __restrict__ k, int64_t k_sb,
                                 int64_t k_sr, int64_t k_sh, const uint8_t* __restrict__ v,
                                 int64_t v_sb, int64_t v_sr, int64_t v_sh, int esz, int cpr) {
  const int hk = blockIdx.y, b = blockIdx.z;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int j = static_cast<int>(t / cpr);
  const int ch = static_cast<int>(t - static_cast<int64_t>(j) * cpr);
  if (j >= p.gather.cap) return;
  const int64_t grow = gather_row(p, b, hk);
  const int cnt = p.gather.count[grow];
  if (j >= (cnt + kTile - 1) / kTile * kTile) return;
  uint8_t* kd = reinterpret_cast<uint8_t*>(const_cast<void*>(p.k)) +
                (b * p.k_sb + static_cast<int64_t>(j) * p.k_sr + hk * p.k_sh) * esz + ch * 16;
  uint8_t* vd = reinterpret_cast<uint8_t*>(const_cast<void*>(p.v)) +
                (b * p.v_sb + static_cast<int64_t>(j) * p.v_sr + hk * p.v_sh) * esz + ch * 16;
  uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
  if (j < cnt) {
    const int64_t key = p.gather.idx[grow * p.gather.cap + j];
    kv = *reinterpret_cast<const uint4*>(k + (b * k_sb + key * k_sr + hk * k_sh) * esz + ch * 16);
    vv = *reinterpret_cast<const uint4*>(v + (b * v_sb + key * v_sr + hk * v_sh) * esz + ch * 16);
  }
  *reinterpret_cast<uint4*>(kd) = kv;
  *reinterpret_cast<uint4*>(vd) = vv;
}

// Compacted bias row (b, head row hc, query row qc): column j < count takes
// the original column idx[j]; the rest are 0 (masked by the row limit).
template <typename T>
__global__ void gather_bias_kernel(const AttnProblem p, const T* __restrict__ src, int64_t s_sb,
                                   int64_t s_sh, int64_t s_sq, int s_kd, int rows_h, int rows_q,
                                   int heads_are_query) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int hq = blockIdx.y, b = blockIdx.z;
  if (j >= p.gather.cap) return;
  const int hc = hq / rows_q, qc = hq - hc * rows_q;
  const int hk = heads_are_query ? hc / p.group : hc;
  const int64_t grow = gather_row(p, b, hk);
  const int cnt = p.gather.count[grow];
  T val = T(0.f);
  if (j < cnt) {
    const int64_t key = p.gather.idx[grow * p.gather.cap + j];
    val = src[b * s_sb + hc * s_sh + qc * s_sq + aux_col(static_cast<int>(key), s_kd)];
  }
  T* dst = reinterpret_cast<T*>(const_cast<void*>(p.bias.ptr));
  dst[b * p.bias.sb + hc * p.bias.sh + qc * p.bias.sq + j] = val;
}

constexpr int kGlThreads = 128;

// Per (gather row, query tile): compacted tiles wholly below the smallest
// row limit of the tile are FULL, those below the largest are PARTIAL.
__global__ void __launch_bounds__(kGlThreads) gather_lists_kernel(const AttnProblem p) {
  const int qt = blockIdx.x, lh = blockIdx.y, lb = blockIdx.z;
  const int64_t grow = static_cast<int64_t>(lb) * p.lists.LH + lh;
  const int q0 = qt * kTile, q1 = min(q0 + kTile, p.Lq) - 1;
  const int lo = gather_row_limit(p, grow, q0);
  const int hi = gather_row_limit(p, grow, q1);
  const int n_full = lo / kTile;
  const int n_part = (hi + kTile - 1) / kTile - n_full;
  const int64_t row = grow * p.QT + qt;
  int32_t* fi = const_cast<int32_t*>(p.lists.full_idx) + row * p.KT;
  int32_t* pi = const_cast<int32_t*>(p.lists.part_idx) + row * p.KT;
  for (int t = threadIdx.x; t < p.KT; t += kGlThreads) {
    fi[t] = t < n_full ? t : -1;
    pi[t] = t < n_part ? n_full + t : -1;
  }
  if (threadIdx.x == 0) {
    const_cast<int32_t*>(p.lists.num_full)[row] = n_full;
    const_cast<int32_t*>(p.lists.num_part)[row] = n_part;
  }
}

}  // namespace

cudaError_t launch_select_keys(const uint8_t* mask, int64_t m_sb, int64_t m_sh, int m_kd, int LB,
                               int LH, int Lk, int cap, int32_t* idx, int32_t* count, int* err,
                               cudaStream_t stream) {
  select_keys_kernel<<<LB * LH, kSelThreads, 0, stream>>>(mask, m_sb, m_sh, m_kd, LH, Lk, cap, idx,
                                                          count, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_kv(const AttnProblem& p, const void* k, const int64_t k_strides[3],
                             const void* v, const int64_t v_strides[3], cudaStream_t stream) {
  const int esz = p.dtype == SMA_FP32 ? 4 : 2;
  const int cpr = p.d * esz / 16;  // 16-byte chunks per row
  const int block = 256;
  const dim3 grid(static_cast<unsigned>(ceil_div(static_cast<int64_t>(p.gather.cap) * cpr, block)),
                  p.KVH, p.B);
  gather_kv_kernel<<<grid, block, 0, stream>>>(
      p, static_cast<const uint8_t*>(k), k_strides[0], k_strides[1], k_strides[2],
      static_cast<const uint8_t*>(v), v_strides[0], v_strides[1], v_strides[2], esz, cpr);
  return cudaGetLastError();
}

cudaError_t launch_gather_bias(const AttnProblem& p, const AuxView& bias, int rows_h, int rows_q,
                               cudaStream_t stream) {
  const int block = 256;
  const dim3 grid(static_cast<unsigned>(ceil_div(p.gather.cap, block)), rows_h * rows_q, p.B);
  const int hq = bias.head_per_query;
  if (bias.dtype == SMA_FP32)
    gather_bias_kernel<float><<<grid, block, 0, stream>>>(
        p, static_cast<const float*>(bias.ptr), bias.sb, bias.sh, bias.sq, bias.kd, rows_h, rows_q,
        hq);
  else  // bf16 / fp16 move as raw 16-bit words
    gather_bias_kernel<uint16_t><<<grid, block, 0, stream>>>(
        p, static_cast<const uint16_t*>(bias.ptr), bias.sb, bias.sh, bias.sq, bias.kd, rows_h, rows_q,
        hq);
  return cudaGetLastError();
}

cudaError_t launch_gather_lists(const AttnProblem& p, cudaStream_t stream) {
  const dim3 grid(p.QT, p.lists.LH, p.lists.LB);
  gather_lists_kernel<<<grid, kGlThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sma
