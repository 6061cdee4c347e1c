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
// from L2 on each pass.  Rows of 16-bit values up to 16384 columns take
// topk16_kernel below instead (same result, values held in registers).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>

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
  int Lk, Kcols;
};

template <int DT>
__device__ __forceinline__ void row_keys(const RowCtx& rc, int c, uint32_t (&key)[kPerThread],
                                         bool (&valid)[kPerThread], bool (&pm)[kPerThread]) {
  using T = KeyTraits<DT>;
  uint32_t u[kPerThread];
  if (c + kPerThread <= rc.Kcols) {
    load_bits8<DT>(rc.brow, c, u);
  } else {  // the row's last columns (rows of Lk columns need not end on a chunk)
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int k = c + e;
      if (k >= rc.Kcols) u[e] = 0;
      else if (DT == SMA_FP32) u[e] = reinterpret_cast<const uint32_t*>(rc.brow)[k];
      else u[e] = reinterpret_cast<const uint16_t*>(rc.brow)[k];
    }
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
  rc.Kcols = p.Kcols;
  uint8_t* orow = p.out + row * p.Kcols;
  const bool out8 = (reinterpret_cast<uintptr_t>(orow) & 7u) == 0;
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
  for (int c0 = 0; c0 < p.Kcols; c0 += kRowStep) {
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
    if (c + kPerThread <= p.Kcols && out8) {
      uint2 v;
      v.x = out[0] | (out[1] << 8) | (out[2] << 16) | (static_cast<uint32_t>(out[3]) << 24);
      v.y = out[4] | (out[5] << 8) | (out[6] << 16) | (static_cast<uint32_t>(out[7]) << 24);
      *reinterpret_cast<uint2*>(orow + c) = v;
    } else {  // unaligned rows (Lk columns) and the row's last columns
#pragma unroll
      for (int e = 0; e < kPerThread; ++e)
        if (c + e < p.Kcols) orow[c + e] = out[e];
    }
    eq_before += step_total;
  }
}


// ---------------------------------------------------------------------------
// topk16_kernel: 16-bit values, rows of at most 16384 columns.
//
// Each thread owns SPAN consecutive columns, kept in registers as packed
// pairs of the raw 16-bit values: pre-masked positions hold the sentinel
// (the dtype's lowest finite value), columns at or past Lk hold NaN.
// Comparisons are packed half-precision compares (one instruction per pair),
// which order the values as numbers: -0 equals +0 (the tie rule above), and
// NaN compares false, so padding columns never count.  Thresholds live in
// the order-preserving 16-bit key space of the non-NaN values; a key is
// turned back into a value for the compares.
//
//  1. Samples spread over the row are binned by the top 11 bits of their key
//     (2048 bins of 32 keys); the bins holding the sample ranks of the
//     window's quantile -/+ 3 standard deviations of the sampling error give
//     a key bracket [k_lo, k_hi] of whole bins.
//  2. One packed block scan counts values above k_hi and at or above k_lo;
//     each thread records which of its columns fall inside the bracket.
//  3. If the bracket holds the window's threshold and spans at most 512
//     keys, the in-bracket values are binned by their full key and one
//     block scan from the top gives the threshold T and the number `need` of
//     values equal to T that complete the window.  Otherwise the block
//     bisects the key space over every value (16 steps).
//  4. A block scan of per-thread counts of values equal to T ranks ties in
//     column order: a value is kept if > T, or equal to T with rank < need.
// The result is the radix select's, bit for bit.
constexpr int kCoarseShift = 5;                 // sample bins of 32 keys
constexpr int kCoarseBins = 65536 >> kCoarseShift;
constexpr int kFineBins = 512;                  // widest bracket binned by full key

template <int DT>
struct Half16;
template <>
struct Half16<SMA_BF16> {
  static constexpr uint32_t kSentinel = 0xFF7Fu, kNaN = 0x7FC0u, kNegInf = 0xFF80u,
                            kPosInf = 0x7F80u;
  static __device__ __forceinline__ __nv_bfloat162 v(uint32_t u) {
    __nv_bfloat162 r;
    memcpy(&r, &u, 4);
    return r;
  }
  static __device__ __forceinline__ uint32_t ge(uint32_t a, uint32_t b) { return __hge2_mask(v(a), v(b)); }
  static __device__ __forceinline__ uint32_t gt(uint32_t a, uint32_t b) { return __hgt2_mask(v(a), v(b)); }
  static __device__ __forceinline__ uint32_t eq(uint32_t a, uint32_t b) { return __heq2_mask(v(a), v(b)); }
};
template <>
struct Half16<SMA_FP16> {
  static constexpr uint32_t kSentinel = 0xFBFFu, kNaN = 0x7E00u, kNegInf = 0xFC00u,
                            kPosInf = 0x7C00u;
  static __device__ __forceinline__ __half2 v(uint32_t u) {
    __half2 r;
    memcpy(&r, &u, 4);
    return r;
  }
  static __device__ __forceinline__ uint32_t ge(uint32_t a, uint32_t b) { return __hge2_mask(v(a), v(b)); }
  static __device__ __forceinline__ uint32_t gt(uint32_t a, uint32_t b) { return __hgt2_mask(v(a), v(b)); }
  static __device__ __forceinline__ uint32_t eq(uint32_t a, uint32_t b) { return __heq2_mask(v(a), v(b)); }
};

__device__ __forceinline__ uint32_t key16(uint32_t b) { return (b & 0x8000u) ? (~b & 0xffffu) : (b | 0x8000u); }
__device__ __forceinline__ uint32_t bits16(uint32_t k) { return (k & 0x8000u) ? (k & 0x7fffu) : (~k & 0xffffu); }
__device__ __forceinline__ uint32_t pair16(uint32_t b) { return b | (b << 16); }

// 16 pre-mask bytes of columns [c, c+16) (0 at and past pk), as four words.
__device__ __forceinline__ uint4 load_pre16(const uint8_t* prow, int pk, int c) {
  if (c + 16 <= pk && (reinterpret_cast<uintptr_t>(prow + c) & 15u) == 0)
    return *reinterpret_cast<const uint4*>(prow + c);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 16; ++e)
    if (c + e < pk && prow[c + e] != 0) w[e >> 2] |= 1u << (8 * (e & 3));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Lane masks (0xffff per kept column) of the two pairs in 4 pre-mask bytes.
__device__ __forceinline__ void pre_lanes(uint32_t p4, uint32_t& m0, uint32_t& m1) {
  const uint32_t nz = ((((p4 & 0x7f7f7f7fu) + 0x7f7f7f7fu) | p4) & 0x80808080u) >> 7;  // 0/1 per byte
  m0 = __byte_perm(nz, 0u, 0x1100) * 0xffu;
  m1 = __byte_perm(nz, 0u, 0x3322) * 0xffu;
}

// Block-wide exclusive scan (one barrier); consecutive calls alternate `buf`.
// After the barrier every warp scans the NT / 32 warp totals itself (lane w
// holds warp w's), so each thread spends one shared load and a few shuffles
// on them instead of reading all of them.
template <int NT>
__device__ __forceinline__ uint32_t scan_excl(uint32_t v, uint32_t* buf, uint32_t* total) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 32, "one warp scans the warp totals");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  const uint32_t wv = lane < NW ? buf[lane] : 0u;
  uint32_t wincl = wv;
#pragma unroll
  for (int o = 1; o < NW; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, wincl, o);
    if (lane >= o) wincl += t;
  }
  const uint32_t base = __shfl_sync(0xffffffffu, wincl - wv, warp);
  *total = __shfl_sync(0xffffffffu, wincl, NW - 1);
  return base + incl - v;
}

// Largest key in [lo, hi] whose value has count(x >= value) >= target, where
// `count_ge` counts over the block (uniform result); also count(x > result).
// Invariants: count(>= lo) >= target, count(>= hi + 1) == above < target.
template <class CountGe>
__device__ __forceinline__ uint32_t bisect_keys(uint32_t lo, uint32_t hi, uint32_t target,
                                                uint32_t* above, CountGe count_ge) {
  uint32_t ab = 0;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    const uint32_t c = count_ge(pair16(bits16(mid)));
    if (c >= target) {
      lo = mid;
    } else {
      hi = mid - 1;
      ab = c;
    }
  }
  *above = ab;
  return lo;
}

template <int DT, int NT>
__global__ void __launch_bounds__(NT, NT == 512 ? 3 : 1)
topk16_kernel(const TopkProblem p) {
  using H = Half16<DT>;
  constexpr int SPAN = 16384 / NT;  // columns per thread
  constexpr int WORDS = SPAN / 2;
  constexpr int SPT = NT >= 512 ? 1 : 512 / NT;  // samples per thread
  constexpr int NS = NT * SPT;
  constexpr int NW = NT / 32;
  static_assert(NT >= kFineBins && SPAN % 16 == 0 && SPAN <= 32 && WORDS % SPT == 0, "layout");
  __shared__ uint32_t s_h1[kCoarseBins];
  __shared__ uint32_t s_h2[kFineBins];
  __shared__ uint32_t s_red[2][NW];
  __shared__ uint32_t s_bc[4];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // Row coordinates in 32-bit arithmetic (the grid has fewer than 2^31 rows).
  const uint32_t row = blockIdx.x;
  const uint32_t n2 = static_cast<uint32_t>(p.b_sizes[2]), n1 = static_cast<uint32_t>(p.b_sizes[1]);
  const uint32_t r12 = row / n2;
  const int64_t i2 = row - r12 * n2;
  const int64_t i1 = r12 % n1;
  const int64_t i0 = r12 / n1;
  const uint8_t* brow = reinterpret_cast<const uint8_t*>(p.bias) +
                        (i0 * p.b_strides[0] + i1 * p.b_strides[1] + i2 * p.b_strides[2]) * 2;
  const uint8_t* prow = p.pre == nullptr
                            ? nullptr
                            : p.pre + (p.p_sizes[0] > 1 ? i0 : 0) * p.p_strides[0] +
                                  (p.p_sizes[1] > 1 ? i1 : 0) * p.p_strides[1] +
                                  (p.p_sizes[2] > 1 ? i2 : 0) * p.p_strides[2];
  const int pk = p.pre == nullptr ? 0 : static_cast<int>(p.p_sizes[3]);
  const int Lk = p.Lk;
  const int c0 = SPAN * threadIdx.x;
  const bool mine = c0 < p.Kcols;  // Kcols is a multiple of 128 here, so spans never straddle it

  // ---- values
  uint32_t x[WORDS];
  if (mine) {
#pragma unroll
    for (int i = 0; i < SPAN / 8; ++i) {
      const uint4 a = *reinterpret_cast<const uint4*>(brow + (c0 + 8 * i) * 2);
      x[4 * i] = a.x; x[4 * i + 1] = a.y; x[4 * i + 2] = a.z; x[4 * i + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < WORDS; ++j) x[j] = pair16(H::kNaN);
  }
  if (prow != nullptr && mine) {
    constexpr uint32_t S2 = H::kSentinel | (H::kSentinel << 16);
#pragma unroll
    for (int i = 0; i < SPAN / 16; ++i) {
      const uint4 pm = load_pre16(prow, pk, c0 + 16 * i);
      const uint32_t pw[4] = {pm.x, pm.y, pm.z, pm.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t m0, m1;
        pre_lanes(pw[q], m0, m1);
        uint32_t& a = x[8 * i + 2 * q];
        uint32_t& b = x[8 * i + 2 * q + 1];
        a = (a & m0) | (S2 & ~m0);
        b = (b & m1) | (S2 & ~m1);
      }
    }
  }
  if (mine && c0 + SPAN > Lk) {  // columns past Lk never count
#pragma unroll
    for (int j = 0; j < WORDS; ++j) {
      const int c = c0 + 2 * j;
      if (c >= Lk) x[j] = pair16(H::kNaN);
      else if (c + 1 >= Lk) x[j] = (x[j] & 0xffffu) | (H::kNaN << 16);
    }
  }

  const uint32_t w = static_cast<uint32_t>(p.window);
  const bool take_all = p.window >= Lk;
  const uint32_t kmin = key16(H::kNegInf), kmax = key16(H::kPosInf);
  uint32_t T = kmin, need = 0;
  uint32_t cand = 0;  // columns that can equal the threshold (bit c - c0)
  int red = 0;        // which s_red buffer the next block reduction uses
  if (!take_all) {
    // ---- 1. bracket from samples
    for (int i = threadIdx.x; i < kCoarseBins; i += NT) s_h1[i] = 0u;
    for (int i = threadIdx.x; i < kFineBins; i += NT) s_h2[i] = 0u;
    if (threadIdx.x == 0) {
      s_bc[0] = kmax >> kCoarseShift;
      s_bc[1] = kmin >> kCoarseShift;
    }
    constexpr int kStep = SPAN / SPT;  // columns between samples
    const int ns_valid = min(NS, (Lk + kStep - 1) / kStep);
    const float q = static_cast<float>(w) / static_cast<float>(Lk);
    const float r = q * static_cast<float>(ns_valid);
    const int delta = static_cast<int>(ceilf(3.f * sqrtf(r * (1.f - q)))) + 2;
    const int r_hi = static_cast<int>(floorf(r)) - delta;   // sample rank from the top
    const int r_lo = static_cast<int>(ceilf(r)) + delta;
    __syncthreads();
#pragma unroll
    for (int s2 = 0; s2 < SPT; ++s2) {
      if (c0 + s2 * kStep < Lk) {
        uint32_t b = x[s2 * (WORDS / SPT)] & 0xffffu;
        b = b == 0x8000u ? 0u : b;  // -0 bins with +0
        atomicAdd(&s_h1[key16(b) >> kCoarseShift], 1u);
      }
    }
    __syncthreads();
    {
      // thread t holds the BPT bins just below the top BPT * t, highest first
      constexpr int BPT = kCoarseBins / NT;
      uint32_t v[BPT], sum = 0;
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        v[i] = s_h1[kCoarseBins - 1 - (BPT * threadIdx.x + i)];
        sum += v[i];
      }
      uint32_t tot1;
      uint32_t before = scan_excl<NT>(sum, s_red[red], &tot1);
      red ^= 1;
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        const uint32_t bin = kCoarseBins - 1 - (BPT * threadIdx.x + i);
        if (r_hi >= 1 && before < static_cast<uint32_t>(r_hi) && static_cast<uint32_t>(r_hi) <= before + v[i])
          s_bc[0] = bin;
        if (r_lo <= ns_valid && before < static_cast<uint32_t>(r_lo) &&
            static_cast<uint32_t>(r_lo) <= before + v[i])
          s_bc[1] = bin;
        before += v[i];
      }
    }
    __syncthreads();
    const uint32_t k_hi = min(kmax, (s_bc[0] << kCoarseShift) | ((1u << kCoarseShift) - 1u));
    const uint32_t k_lo = max(kmin, s_bc[1] << kCoarseShift);
    const uint32_t thi2 = pair16(bits16(k_hi)), tlo2 = pair16(bits16(k_lo));

    // ---- 2. counts above the bracket and in it; cand: 1 bit per column in it
    uint32_t n_gt = 0, n_ge = 0;
#pragma unroll
    for (int j = 0; j < WORDS; ++j) {
      const uint32_t ge = H::ge(x[j], tlo2), gt = H::gt(x[j], thi2);
      n_ge += __popc(ge);
      n_gt += __popc(gt);
      const uint32_t cm = ge & ~gt;  // 0xffff per lane in the bracket
      cand |= (((cm >> 15) & 1u) | ((cm >> 30) & 2u)) << (2 * j);
    }
    uint32_t tot;
    scan_excl<NT>(((n_gt >> 4) << 16) | (n_ge >> 4), s_red[red], &tot);
    red ^= 1;
    const uint32_t c_gt = tot >> 16, c_ge = tot & 0xffffu;
    const uint32_t nbins = k_hi - k_lo + 1;
    if (c_gt < w && w <= c_ge && nbins <= static_cast<uint32_t>(kFineBins)) {
      // ---- 3a. bin the in-bracket values by key; scan from the top
      // +-0 are one value: their key is the bracket's zero key.
      const uint32_t zero_key = k_hi >= 0x8000u ? 0x8000u : 0x7fffu;
#pragma unroll
      for (int j = 0; j < WORDS; ++j) {
        const uint32_t cb = (cand >> (2 * j)) & 3u;
        if (cb != 0u) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if ((cb >> e) & 1u) {
              const uint32_t b = (x[j] >> (16 * e)) & 0xffffu;
              const uint32_t k = (b & 0x7fffu) == 0u ? zero_key : key16(b);
              const uint32_t bin = k - k_lo;
              if (bin < static_cast<uint32_t>(kFineBins)) atomicAdd(&s_h2[bin], 1u);
            }
          }
        }
      }
      __syncthreads();
      const uint32_t want = w - c_gt;
      const int t = threadIdx.x;  // thread t holds key k_hi - t
      const uint32_t v = t < static_cast<int>(nbins) ? s_h2[nbins - 1 - t] : 0u;
      uint32_t tot2;
      const uint32_t before = scan_excl<NT>(v, s_red[red], &tot2);
      red ^= 1;
      if (v != 0u && before < want && want <= before + v) {
        s_bc[2] = k_hi - static_cast<uint32_t>(t);
        s_bc[3] = want - before;
      }
      __syncthreads();
      T = s_bc[2];
      need = s_bc[3];
    } else {
      // ---- 3b. the bracket missed (or spans too many keys): bisect over every value
      uint32_t above;
      T = bisect_keys(kmin, kmax, w, &above, [&](uint32_t t2) {
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < WORDS; ++j) c += __popc(H::ge(x[j], t2));
        c = __reduce_add_sync(0xffffffffu, c) >> 4;
        if (lane == 0) s_red[red][warp] = c;
        __syncthreads();
        const uint32_t all = __reduce_add_sync(0xffffffffu, lane < NW ? s_red[red][lane] : 0u);
        red ^= 1;
        return all;
      });
      need = w - above;
      cand = SPAN == 32 ? 0xffffffffu : ((1u << SPAN) - 1u);
    }
  }

  // ---- 4. output in column order
  const uint32_t t2 = take_all ? pair16(H::kNegInf) : pair16(bits16(T));
  uint32_t rank = 0;
  if (!take_all) {
    uint32_t n_eq = 0;  // values equal to T lie among the candidates
#pragma unroll
    for (int j = 0; j < WORDS; ++j)
      if ((cand >> (2 * j)) & 3u) n_eq += __popc(H::eq(x[j], t2));
    uint32_t tot;
    rank = scan_excl<NT>(n_eq >> 4, s_red[red], &tot);
  }
  // Pre-masked columns hold the sentinel: they can pass only when T is at or
  // below it, and are then cleared with the pre-mask.
  const bool and_pre = prow != nullptr && (take_all || T <= key16(H::kSentinel));
  if (!mine) return;
  uint8_t* orow = p.out + static_cast<int64_t>(row) * p.Kcols + c0;
#pragma unroll
  for (int i = 0; i < SPAN / 16; ++i) {
    uint32_t pmw[8];
    if (and_pre) {
      const uint4 pm = load_pre16(prow, pk, c0 + 16 * i);
      const uint32_t pw[4] = {pm.x, pm.y, pm.z, pm.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) pre_lanes(pw[q], pmw[2 * q], pmw[2 * q + 1]);
    }
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      uint32_t ob[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = 8 * i + 2 * h + e;
        uint32_t gm;
        if (take_all) {
          gm = H::ge(x[j], t2);
        } else {
          gm = H::gt(x[j], t2);
          const uint32_t em = ((cand >> (2 * j)) & 3u) ? H::eq(x[j], t2) : 0u;
          if (em != 0u) {
            if (em & 0xffffu) {
              if (rank < need) gm |= 0xffffu;
              ++rank;
            }
            if (em >> 16) {
              if (rank < need) gm |= 0xffff0000u;
              ++rank;
            }
          }
        }
        if (and_pre) gm &= pmw[2 * h + e];
        ob[e] = (gm & 1u) | ((gm >> 8) & 0x100u);  // two bytes, 0/1
      }
      o[h] = ob[0] | (ob[1] << 16);
    }
    *reinterpret_cast<uint4*>(orow + 16 * i) = make_uint4(o[0], o[1], o[2], o[3]);
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
  const bool few = rows < 2 * num_sms();
  // The register-resident kernel stores 16 bytes at a time.
  const bool out16 = (reinterpret_cast<uintptr_t>(p.out) & 15u) == 0;
  // It also takes whole 128-column rows (the padded key dim) only.
  if (p.bias_dtype != SMA_FP32 && p.Kcols <= 16384 && p.Kcols % kTile == 0 && out16) {
    if (p.bias_dtype == SMA_BF16) {
      if (few) topk16_kernel<SMA_BF16, 1024><<<grid, 1024, 0, stream>>>(p);
      else topk16_kernel<SMA_BF16, 512><<<grid, 512, 0, stream>>>(p);
    } else {
      if (few) topk16_kernel<SMA_FP16, 1024><<<grid, 1024, 0, stream>>>(p);
      else topk16_kernel<SMA_FP16, 512><<<grid, 512, 0, stream>>>(p);
    }
    return cudaGetLastError();
  }
  if (few) launch_nt<1024>(p, grid, stream);
  else launch_nt<256>(p, grid, stream);
  return cudaGetLastError();
}

}  // namespace sma
