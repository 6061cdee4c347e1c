// Dynamic top-k keep mask (flash-sparse-attention PR #197, "Centralize
// dynamic mask creation for FDMA": Design and Implementation Notes).
//
// Per row of the bias, positions the pre-mask rejects take the bias dtype's
// minimum finite value, the window_size largest values are selected, and the
// result is written as a boolean row.  The page's selection is unsorted and
// leaves ties open; here equal values are taken in ascending key order and
// -0.0 equals +0.0, which makes the mask unique.
//
// Method (no sort): values map to order-preserving unsigned keys; a radix
// select on 8-bit digits (2 passes for 16-bit dtypes, 4 for fp32) finds the
// threshold key T and how many entries equal to T are still needed; a final
// pass keeps every key > T plus the first `need` keys == T in index order,
// found with a block-wide prefix count.  One CTA per row; the row is re-read
// from L2 on each pass.
#include "device_common.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kPerThread = 8;

template <int DT>
struct KeyTraits;
template <>
struct KeyTraits<SMA_BF16> {
  using U = uint32_t;
  static constexpr int kBits = 16;
  static constexpr uint32_t kSentinel = 0xFF7Fu;  // -(2 - 2^-7) * 2^127
};
template <>
struct KeyTraits<SMA_FP16> {
  using U = uint32_t;
  static constexpr int kBits = 16;
  static constexpr uint32_t kSentinel = 0xFBFFu;  // -65504
};
template <>
struct KeyTraits<SMA_FP32> {
  using U = uint32_t;
  static constexpr int kBits = 32;
  static constexpr uint32_t kSentinel = 0xFF7FFFFFu;  // -(2 - 2^-23) * 2^127
};

// Order-preserving map of IEEE bits (sign-magnitude) to unsigned keys, with
// -0 folded onto +0.
template <int BITS>
__device__ __forceinline__ uint32_t order_key(uint32_t u) {
  constexpr uint32_t sign = 1u << (BITS - 1);
  constexpr uint32_t all = BITS == 32 ? 0xffffffffu : ((1u << BITS) - 1u);
  if (u == sign) u = 0u;
  return (u & sign) ? (~u & all) : (u | sign);
}

template <int DT>
__device__ __forceinline__ void load_bits8(const uint8_t* row, int c, uint32_t (&u)[kPerThread]) {
  if (DT == SMA_FP32) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + c * 4);
    const uint4 b = *reinterpret_cast<const uint4*>(row + c * 4 + 16);
    u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w; u[4] = b.x; u[5] = b.y; u[6] = b.z; u[7] = b.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(row + c * 2);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      u[2 * e] = w[e] & 0xffffu;
      u[2 * e + 1] = w[e] >> 16;
    }
  }
}

struct RowCtx {
  const uint8_t* brow;  // bias row
  const uint8_t* prow;  // pre-mask row or null
  int pk;               // pre-mask length
  int Lk, Kpad;
};

template <int DT>
__device__ __forceinline__ void row_keys(const RowCtx& rc, int c, uint32_t (&key)[kPerThread],
                                         bool (&valid)[kPerThread], bool (&pm)[kPerThread]) {
  using T = KeyTraits<DT>;
  uint32_t u[kPerThread];
  if (c < rc.Kpad) {
    load_bits8<DT>(rc.brow, c, u);
  } else {
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) u[e] = 0;
  }
#pragma unroll
  for (int e = 0; e < kPerThread; ++e) {
    const int k = c + e;
    valid[e] = k < rc.Lk;
    pm[e] = rc.prow == nullptr ? true : (k < rc.pk && rc.prow[k] != 0);
    key[e] = order_key<T::kBits>(pm[e] ? u[e] : T::kSentinel);
  }
}

// NT threads per row: 1024 when there are few rows (latency), 256 otherwise.
template <int DT, int NT>
__global__ void __launch_bounds__(NT)
topk_mask_kernel(const TopkProblem p) {
  using T = KeyTraits<DT>;
  constexpr int kTkThreads = NT;
  constexpr int kTkWarps = NT / 32;
  constexpr int kRowStep = NT * kPerThread;
  __shared__ uint32_t hist[kTkWarps][256];
  __shared__ uint32_t total[256];
  __shared__ uint32_t s_digit, s_remaining, s_scan[kTkWarps];

  const int64_t row = blockIdx.x;
  const int64_t i2 = row % p.b_sizes[2];
  const int64_t i1 = (row / p.b_sizes[2]) % p.b_sizes[1];
  const int64_t i0 = row / (p.b_sizes[2] * p.b_sizes[1]);
  const int esz = DT == SMA_FP32 ? 4 : 2;
  RowCtx rc;
  rc.brow = reinterpret_cast<const uint8_t*>(p.bias) +
            (i0 * p.b_strides[0] + i1 * p.b_strides[1] + i2 * p.b_strides[2]) * esz;
  rc.prow = p.pre == nullptr
                ? nullptr
                : p.pre + (p.p_sizes[0] > 1 ? i0 : 0) * p.p_strides[0] +
                      (p.p_sizes[1] > 1 ? i1 : 0) * p.p_strides[1] +
                      (p.p_sizes[2] > 1 ? i2 : 0) * p.p_strides[2];
  rc.pk = p.pre == nullptr ? 0 : static_cast<int>(p.p_sizes[3]);
  rc.Lk = p.Lk;
  rc.Kpad = p.Kpad;
  uint8_t* orow = p.out + row * p.Kpad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const bool take_all = p.window >= p.Lk;
  uint32_t prefix = 0, prefix_mask = 0, remaining = static_cast<uint32_t>(p.window);
  if (!take_all) {
    for (int shift = T::kBits - 8; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < kTkWarps * 256; i += kTkThreads) (&hist[0][0])[i] = 0;
      __syncthreads();
      for (int c0 = 0; c0 < p.Lk; c0 += kRowStep) {
        const int c = c0 + threadIdx.x * kPerThread;
        uint32_t key[kPerThread];
        bool valid[kPerThread], pm[kPerThread];
        row_keys<DT>(rc, c, key, valid, pm);
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          const bool cand = valid[e] && (key[e] & prefix_mask) == prefix;
          const uint32_t digit = (key[e] >> shift) & 0xffu;
          const uint32_t act = __ballot_sync(0xffffffffu, cand);
          if (cand) {
            const uint32_t peers = __match_any_sync(act, digit);
            if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp][digit], __popc(peers));
          }
        }
      }
      __syncthreads();
      // total[d] and the digit where the running count from the top reaches `remaining`.
      if (threadIdx.x < 256) {
        const int d = threadIdx.x;
        uint32_t cnt = 0;
#pragma unroll
        for (int w = 0; w < kTkWarps; ++w) cnt += hist[w][d];
        total[d] = cnt;
      }
      __syncthreads();
      {
        // suffix sums over digits: above[d] = sum of total[d'] for d' > d
        // (threads 0..255 take digits 255..0, so a prefix scan gives suffixes)
        const int d = 255 - threadIdx.x;
        const uint32_t v = threadIdx.x < 256 ? total[d] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (lane == 31 && warp < 8) s_scan[warp] = incl;
        __syncthreads();
        if (threadIdx.x < 256) {
          uint32_t wbase = 0;
          for (int w = 0; w < warp; ++w) wbase += s_scan[w];
          const uint32_t above = wbase + incl - v;
          if (above < remaining && remaining <= above + v) {
            s_digit = static_cast<uint32_t>(d);
            s_remaining = remaining - above;
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      prefix_mask |= 0xffu << shift;
      remaining = s_remaining;
      __syncthreads();
    }
  }
  // Output pass: key > T, or key == T among the first `remaining` in index order.
  const uint32_t thr = prefix;
  uint32_t eq_before = 0;  // running count of key == T in earlier steps
  for (int c0 = 0; c0 < p.Kpad; c0 += kRowStep) {
    const int c = c0 + threadIdx.x * kPerThread;
    uint32_t key[kPerThread];
    bool valid[kPerThread], pm[kPerThread];
    row_keys<DT>(rc, c, key, valid, pm);
    uint32_t my_eq = 0;
    if (!take_all) {
#pragma unroll
      for (int e = 0; e < kPerThread; ++e) my_eq += (valid[e] && key[e] == thr) ? 1u : 0u;
    }
    uint32_t incl = my_eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) s_scan[warp] = incl;
    __syncthreads();
    uint32_t wbase = 0, step_total = 0;
    for (int w = 0; w < kTkWarps; ++w) {
      if (w < warp) wbase += s_scan[w];
      step_total += s_scan[w];
    }
    uint32_t rank = eq_before + wbase + incl - my_eq;
    uint8_t out[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      bool keep = false;
      if (valid[e]) {
        if (take_all) {
          keep = true;
        } else if (key[e] > thr) {
          keep = true;
        } else if (key[e] == thr) {
          keep = rank < remaining;
          ++rank;
        }
      }
      out[e] = (keep && pm[e]) ? 1 : 0;
    }
    if (c < p.Kpad) {
      uint2 v;
      v.x = out[0] | (out[1] << 8) | (out[2] << 16) | (static_cast<uint32_t>(out[3]) << 24);
      v.y = out[4] | (out[5] << 8) | (out[6] << 16) | (static_cast<uint32_t>(out[7]) << 24);
      *reinterpret_cast<uint2*>(orow + c) = v;
    }
    eq_before += step_total;
  }
}

template <int NT>
void launch_nt(const TopkProblem& p, unsigned grid, cudaStream_t stream) {
  if (p.bias_dtype == SMA_BF16) topk_mask_kernel<SMA_BF16, NT><<<grid, NT, 0, stream>>>(p);
  else if (p.bias_dtype == SMA_FP16) topk_mask_kernel<SMA_FP16, NT><<<grid, NT, 0, stream>>>(p);
  else topk_mask_kernel<SMA_FP32, NT><<<grid, NT, 0, stream>>>(p);
}

}  // namespace

cudaError_t launch_topk(const TopkProblem& p, cudaStream_t stream) {
  const int64_t rows = p.b_sizes[0] * p.b_sizes[1] * p.b_sizes[2];
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(rows);
  // Few rows: one wide CTA per row finishes each row sooner.
  if (rows < 2 * num_sms()) launch_nt<1024>(p, grid, stream);
  else launch_nt<256>(p, grid, stream);
  return cudaGetLastError();
}

}  // namespace sma
