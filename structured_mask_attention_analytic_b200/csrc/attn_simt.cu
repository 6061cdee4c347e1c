// fp32 attention forward with plain FFMA arithmetic (no TF32), for fp32
// inputs.  Walks the same key-tile lists and applies the same two mask
// families as the tensor-core kernel; exists because TF32 products cannot
// reach a 1e-4 absolute agreement with a float64 reference.
//
// One CTA per (batch, query head, 128-row query tile); two threads per row,
// each owning the even or odd half of head_dim; keys in chunks of 32 staged
// through shared memory.  Packed sequences (varlen): batch entry b is
// sequence b, its rows offset by the cumulative arrays.
#include "device_common.cuh"
#include "gather.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kChunkKeys = 32;

template <int D, int POLICY>
__global__ void __launch_bounds__(kSimtThreads)
attn_simt_kernel(const AttnProblem p) {
  constexpr int E = D / 2;  // elements per thread
  __shared__ float sk[kChunkKeys][D];
  __shared__ float sv[kChunkKeys][D];
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const int r = threadIdx.x >> 1, hf = threadIdx.x & 1;
  const int q = qt * kTile + r;
  const SeqRows sr = seq_rows<POLICY>(p, b);  // packed sequences: this sequence's rows
  const bool row_valid = q < sr.lq;

  const int lb = p.lists.LB > 1 ? b : 0;
  int lh = 0;
  if (p.lists.head_mode == 1) lh = hk;
  else if (p.lists.head_mode == 2) lh = hk * p.npairs + (h - hk * p.group) / 2;
  const int64_t row = (static_cast<int64_t>(lb) * p.lists.LH + lh) * p.QT + qt;
  const int nf = p.lists.num_full[row], np = p.lists.num_part[row];

  const float* Q = reinterpret_cast<const float*>(p.q);
  const float* K = reinterpret_cast<const float*>(p.k);
  const float* V = reinterpret_cast<const float*>(p.v);
  float qr[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qr[e] = row_valid ? Q[b * p.q_sb + static_cast<int64_t>(sr.q_off + q) * p.q_sr + h * p.q_sh +
                          2 * e + hf] *
                            p.scale_log2
                      : 0.f;
    o[e] = 0.f;
  }

  int clo = 0, chi = 0, dlo = 0, dhi = 0;
  const uint8_t* mrow = nullptr;
  const void* brow = nullptr;
  int causal_lim = 0x7fffffff;
  if (POLICY == kPolicyDflash) {
    if (row_valid) {
      const int j = q / p.bs, i = q - j * p.bs;
      int a = p.anchors[static_cast<int64_t>(b) * p.N + j];
      a = a < 0 ? 0 : (a > p.Lc ? p.Lc : a);
      chi = a;
      clo = p.window > 0 ? max(0, a + i - p.window + 1) : 0;
      if (clo > chi) clo = chi;
      const int base = p.Lc + j * p.bs;
      dlo = base + (p.window > 0 ? max(0, i - p.window + 1) : 0);
      dhi = base + (p.causal_in_block ? i + 1 : p.bs);
    }
  } else {
    const int qq = row_valid ? q : 0;
    if (p.has_mask) {
      const int hm = p.mask.head_per_query ? h : hk;
      mrow = reinterpret_cast<const uint8_t*>(p.mask.ptr) + b * p.mask.sb + hm * p.mask.sh +
             static_cast<int64_t>(qq) * p.mask.sq;
    }
    if (p.has_bias) {
      const int hb = p.bias.head_per_query ? h : hk;
      const int esz = p.bias.dtype == SMA_FP32 ? 4 : 2;
      brow = reinterpret_cast<const uint8_t*>(p.bias.ptr) +
             (b * p.bias.sb + hb * p.bias.sh + static_cast<int64_t>(qq) * p.bias.sq) * esz;
    }
    if (p.gather.idx != nullptr)  // compacted keys: the row's limit on the compacted index
      causal_lim = row_valid ? gather_row_limit(p, static_cast<int64_t>(lb) * p.lists.LH + lh, q) - 1 : -1;
    else if (p.causal)
      causal_lim = q + sr.lk - sr.lq;
  }

  float m = -INFINITY, l = 0.f;
  for (int t = 0; t < nf + np; ++t) {
    const bool partial = t >= nf;
    const int kt = partial ? p.lists.part_idx[row * p.KT + (t - nf)]
                           : p.lists.full_idx[row * p.KT + t];
    for (int c0 = kt * kTile; c0 < kt * kTile + kTile; c0 += kChunkKeys) {
      __syncthreads();
      for (int i = threadIdx.x; i < kChunkKeys * D; i += kSimtThreads) {
        const int kk = i / D, e = i - kk * D;
        const int k = c0 + kk;
        float kv = 0.f, vv = 0.f;
        if (k < sr.lk) {
          kv = K[b * p.k_sb + static_cast<int64_t>(sr.k_off + k) * p.k_sr + hk * p.k_sh + e];
          vv = V[b * p.v_sb + static_cast<int64_t>(sr.k_off + k) * p.v_sr + hk * p.v_sh + e];
        }
        sk[kk][e] = kv;
        sv[kk][e] = vv;
      }
      __syncthreads();
      float s[kChunkKeys];
      float mx = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kChunkKeys; ++kk) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc = fmaf(qr[e], sk[kk][2 * e + hf], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        const int k = c0 + kk;
        if (POLICY != kPolicyDflash && p.has_bias && k < sr.lk)
          acc = fmaf(load_any_as_float(brow, p.bias.dtype, aux_col(k, p.bias.kd)), kLog2e, acc);
        bool keep = row_valid;
        if (partial) {
          if (POLICY == kPolicyDflash) {
            keep = keep && ((k >= clo && k < chi) || (k >= dlo && k < dhi));
          } else {
            keep = keep && k < sr.lk && k <= causal_lim && (!p.has_mask || mrow[aux_col(k, p.mask.kd)] != 0);
          }
        }
        s[kk] = keep ? acc : -INFINITY;
        mx = fmaxf(mx, s[kk]);
      }
      const float m_new = fmaxf(m, mx);
      if (m_new != -INFINITY) {
        const float alpha = m == -INFINITY ? 0.f : exp2f(m - m_new);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] *= alpha;
#pragma unroll
        for (int kk = 0; kk < kChunkKeys; ++kk) {
          const float pk = exp2f(s[kk] - m_new);
          l += pk;
#pragma unroll
          for (int e = 0; e < E; ++e) o[e] = fmaf(pk, sv[kk][2 * e + hf], o[e]);
        }
        m = m_new;
      }
    }
  }
  if (row_valid) {
    float* O = reinterpret_cast<float*>(p.o);
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
      O[b * p.o_sb + static_cast<int64_t>(sr.q_off + q) * p.o_sr + h * p.o_sh + 2 * e + hf] = o[e] * inv;
    if (hf == 0 && p.lse != nullptr)
      p.lse[row_index<POLICY>(p, b, h, sr, q)] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attn_simt(const AttnProblem& p, cudaStream_t stream) {
  dim3 grid(p.QT, p.H, p.B);
  if (p.QT == 0) return cudaSuccess;
  if (p.d == 128) {
    if (p.policy == kPolicyDflash)
      attn_simt_kernel<128, kPolicyDflash><<<grid, kSimtThreads, 0, stream>>>(p);
    else if (p.policy == kPolicyVarlen)
      attn_simt_kernel<128, kPolicyVarlen><<<grid, kSimtThreads, 0, stream>>>(p);
    else
      attn_simt_kernel<128, kPolicyExplicit><<<grid, kSimtThreads, 0, stream>>>(p);
  } else {
    if (p.policy == kPolicyDflash)
      attn_simt_kernel<64, kPolicyDflash><<<grid, kSimtThreads, 0, stream>>>(p);
    else if (p.policy == kPolicyVarlen)
      attn_simt_kernel<64, kPolicyVarlen><<<grid, kSimtThreads, 0, stream>>>(p);
    else
      attn_simt_kernel<64, kPolicyExplicit><<<grid, kSimtThreads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sma
