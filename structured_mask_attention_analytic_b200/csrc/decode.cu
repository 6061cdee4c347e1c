// Single-query attention (q_len == 1) with the grouped-head swap.
//
// flash-sparse-attention PR #190, "Swapped path (seqlen_q==1 and H>H_k)":
// the query heads of one KV head are reshaped to act as rows of a single
// problem, while mask/bias keep their original batch/head meaning and the lse
// write-back follows the original [B, H] order.  Here the swap is a change of
// loop order: a CTA owns (batch, KV head, key chunk) and evaluates all G query
// heads of that KV head against every key it loads, so K and V are read from
// HBM once per KV head instead of once per query head.
//
// The work is HBM-bound (each K/V element feeds G fused multiply-adds), so
// keys are split into chunks across CTAs (split-KV) to fill every SM; a second
// kernel merges the per-chunk (max, sum, unnormalised O) triples.
//
// Lane layout: each warp takes two keys per step, 16 lanes per key, each lane
// owning 8 consecutive head_dim elements (one 16-byte load for bf16/fp16).
#include "device_common.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&f)[8]) {
  if (DT == SMA_FP32) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 c = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + idx);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (DT == SMA_BF16) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      } else {
        const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
      }
    }
  }
}

// grid: (splits, KVH * row_groups, B); rows [rg*G, rg*G+G) of the group.
template <int D, int G, int DT>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const DecodeProblem p) {
  constexpr int LPK = D / 8;           // lanes per key (8 elements each)
  constexpr int KPW = 32 / LPK;        // keys per warp step
  const int split = blockIdx.x;
  const int row_groups = (p.group + G - 1) / G;
  const int hk = blockIdx.y / row_groups;
  const int rg = blockIdx.y - hk * row_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = lane / LPK, dl = lane - slot * LPK;
  const int e0 = dl * 8;
  const int k_begin = split * p.chunk;
  const int k_end = min(p.Lk, k_begin + p.chunk);

  float qf[G][8];
  bool rvalid[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const int gr = rg * G + r;
    rvalid[r] = gr < p.group;
    const int h = hk * p.group + (rvalid[r] ? gr : 0);
    load8<DT>(p.q, b * p.q_sb + h * p.q_sh + e0, qf[r]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[r][e] *= p.scale_log2;
  }
  float m[G], l[G], o[G][8];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[r][e] = 0.f;
  }

  const int esz = p.has_bias && p.bias.dtype == SMA_FP32 ? 4 : 2;
  for (int kb = k_begin + warp * KPW; kb < k_end; kb += kDecWarps * KPW) {
    const int k = kb + slot;
    const bool kvalid = k < k_end;
    float kf[8], vf[8];
    if (kvalid) {
      load8<DT>(p.k, b * p.k_sb + static_cast<int64_t>(k) * p.k_sr + hk * p.k_sh + e0, kf);
      load8<DT>(p.v, b * p.v_sb + static_cast<int64_t>(k) * p.v_sr + hk * p.v_sh + e0, vf);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) { kf[e] = 0.f; vf[e] = 0.f; }
    }
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(qf[r][e], kf[e], s);
#pragma unroll
      for (int off = 1; off < LPK; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const int h = hk * p.group + rg * G + r;
      bool keep = kvalid && rvalid[r];
      if (keep && p.has_mask) {
        const int hm = p.mask.head_per_query ? h : hk;
        keep = reinterpret_cast<const uint8_t*>(p.mask.ptr)[b * p.mask.sb + hm * p.mask.sh + k] != 0;
      }
      if (keep && p.has_bias) {
        const int hb = p.bias.head_per_query ? h : hk;
        const int64_t bi = b * p.bias.sb + hb * p.bias.sh + k;
        s = fmaf(load_any_as_float(p.bias.ptr, p.bias.dtype, bi), kLog2e, s);
      }
      s = keep ? s : -INFINITY;
      float mx = s;
#pragma unroll
      for (int off = LPK; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[r], mx);
      if (m_new != -INFINITY) {
        const float alpha = m[r] == -INFINITY ? 0.f : fast_exp2(m[r] - m_new);
        const float pk = fast_exp2(s - m_new);
        float ps = pk;
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l[r] = l[r] * alpha + ps;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[r][e] = fmaf(pk, vf[e], o[r][e] * alpha);
        m[r] = m_new;
      }
    }
  }
  (void)esz;

  // Sum the key slots of the warp, then merge warps through shared memory.
#pragma unroll
  for (int r = 0; r < G; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int off = LPK; off < 32; off <<= 1)
        o[r][e] += __shfl_xor_sync(0xffffffffu, o[r][e], off);

  __shared__ float s_o[kDecWarps][G][D];
  __shared__ float s_m[kDecWarps][G], s_l[kDecWarps][G];
  if (slot == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_o[warp][r][e0 + e] = o[r][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < G; ++r) { s_m[warp][r] = m[r]; s_l[warp][r] = l[r]; }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int r = i / D, e = i - r * D;
    const int gr = rg * G + r;
    if (gr >= p.group) continue;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w][r]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float sc = s_m[w][r] == -INFINITY ? 0.f : fast_exp2(s_m[w][r] - M);
        acc += sc * s_o[w][r][e];
        lsum += sc * s_l[w][r];
      }
    }
    const int h = hk * p.group + gr;
    const int64_t pi = (static_cast<int64_t>(b) * p.H + h) * p.splits + split;
    p.part_o[pi * D + e] = acc;
    if (e == 0) {
      p.part_ml[pi * 2] = M;
      p.part_ml[pi * 2 + 1] = lsum;
    }
  }
}

template <int D, int DT>
__global__ void decode_combine_kernel(const DecodeProblem p) {
  const int bh = blockIdx.x;  // b * H + h
  const int b = bh / p.H, h = bh - b * p.H;
  const int e = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[(static_cast<int64_t>(bh) * p.splits + s) * 2]);
  float acc = 0.f, l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const int64_t pi = static_cast<int64_t>(bh) * p.splits + s;
      const float ms = p.part_ml[pi * 2];
      const float sc = ms == -INFINITY ? 0.f : exp2f(ms - M);
      acc += sc * p.part_o[pi * D + e];
      l += sc * p.part_ml[pi * 2 + 1];
    }
  }
  const float out = l > 0.f ? acc / l : 0.f;
  const int64_t oi = b * p.o_sb + h * p.o_sh + e;
  if (DT == SMA_FP32) reinterpret_cast<float*>(p.o)[oi] = out;
  else if (DT == SMA_BF16) reinterpret_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(out);
  else reinterpret_cast<__half*>(p.o)[oi] = __float2half_rn(out);
  if (e == 0 && p.lse != nullptr) p.lse[bh] = l > 0.f ? (M + log2f(l)) * kLn2 : -INFINITY;
}

template <int D, int G, int DT>
cudaError_t launch3(const DecodeProblem& p, cudaStream_t stream) {
  const int row_groups = (p.group + G - 1) / G;
  dim3 grid(p.splits, p.KVH * row_groups, p.B);
  decode_split_kernel<D, G, DT><<<grid, kDecThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D, DT><<<p.B * p.H, D, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int DT>
cudaError_t launch2(const DecodeProblem& p, cudaStream_t stream) {
  if (p.group <= 1) return launch3<D, 1, DT>(p, stream);
  if (p.group <= 2) return launch3<D, 2, DT>(p, stream);
  if (p.group <= 4) return launch3<D, 4, DT>(p, stream);
  return launch3<D, 8, DT>(p, stream);
}

template <int D>
cudaError_t launch1(const DecodeProblem& p, cudaStream_t stream) {
  if (p.dtype == SMA_BF16) return launch2<D, SMA_BF16>(p, stream);
  if (p.dtype == SMA_FP16) return launch2<D, SMA_FP16>(p, stream);
  return launch2<D, SMA_FP32>(p, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t stream) {
  if (p.B == 0 || p.H == 0) return cudaSuccess;
  return p.d == 128 ? launch1<128>(p, stream) : launch1<64>(p, stream);
}

}  // namespace sma
