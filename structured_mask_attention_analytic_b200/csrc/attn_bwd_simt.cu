// fp32 attention backward with plain FFMA arithmetic (no TF32), for fp32
// inputs: the gradients of the fp32 forward (attn_simt.cu) under the same
// mask families.  Same formulas as the tensor-core backward (attn_bwd.cu):
//   P = exp(scale q.k + bias - lse),  dP = dO.v,  dS = P (dP - D),
//   dQ = scale sum_k dS K,  dK = scale sum_q dS Q,  dV = sum_q P dO,
// with D = rowsum(dO * O) from the preparation kernel and the forward's lse.
//
// attn_bwd_simt_dq_kernel: one CTA per (batch, query head, 128-row query
// tile), two threads per row (even / odd half of head_dim), keys in chunks
// of 32 staged through shared memory, over the row tile's key-tile list;
// writes sum_k dS K (unscaled) to the fp32 dQ accumulator and, when asked,
// dbias.
// attn_bwd_simt_dkv_kernel: one CTA per (batch, KV head, 128-key tile), two
// threads per key row, over the query heads of the group and the query tiles
// of the transposed list, queries in chunks of 32 staged through shared
// memory (Q, dO, lse, D); writes dK and dV.
// The keep rule and bias of each (query, key) pair are evaluated exactly as
// in the forward; on FULL pairs only the key-length bound applies.  Packed
// sequences (varlen): batch entry b is sequence b, its query and key rows
// offset by the cumulative arrays, its per-row data at [H, total_q].
#include "device_common.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kBsThreads = 256;
constexpr int kBsChunk = 32;

// Mask parameters of one query row (the forward's per-row state).
struct RowKeep {
  int clo, chi, dlo, dhi;  // DFlash keep intervals
  const uint8_t* mrow;     // explicit mask row (null: none)
  const void* brow;        // bias row (null: none)
  int causal_lim;          // explicit: keys above are dropped
  bool valid;
};

template <int POLICY>
__device__ __forceinline__ RowKeep row_keep(const AttnProblem& p, int b, int h, int hk, int q,
                                            const SeqRows& sr) {
  RowKeep r{};
  r.valid = q < sr.lq;
  r.causal_lim = 0x7fffffff;
  if (!r.valid) return r;
  if (POLICY == kPolicyDflash) {
    const int j = q / p.bs, i = q - j * p.bs;
    int a = p.anchors[static_cast<int64_t>(b) * p.N + j];
    a = a < 0 ? 0 : (a > p.Lc ? p.Lc : a);
    r.chi = a;
    r.clo = p.window > 0 ? max(0, a + i - p.window + 1) : 0;
    if (r.clo > r.chi) r.clo = r.chi;
    const int base = p.Lc + j * p.bs;
    r.dlo = base + (p.window > 0 ? max(0, i - p.window + 1) : 0);
    r.dhi = base + (p.causal_in_block ? i + 1 : p.bs);
  } else {
    if (p.has_mask) {
      const int hm = p.mask.head_per_query ? h : hk;
      r.mrow = reinterpret_cast<const uint8_t*>(p.mask.ptr) + b * p.mask.sb + hm * p.mask.sh +
               static_cast<int64_t>(q) * p.mask.sq;
    }
    if (p.has_bias) {
      const int hb = p.bias.head_per_query ? h : hk;
      const int esz = p.bias.dtype == SMA_FP32 ? 4 : 2;
      r.brow = reinterpret_cast<const uint8_t*>(p.bias.ptr) +
               (b * p.bias.sb + hb * p.bias.sh + static_cast<int64_t>(q) * p.bias.sq) * esz;
    }
    if (p.causal) r.causal_lim = q + sr.lk - sr.lq;
  }
  return r;
}

// Is key k kept for the row (PARTIAL tiles evaluate the whole rule)?
template <int POLICY>
__device__ __forceinline__ bool keeps(const AttnProblem& p, const RowKeep& r, int k, bool partial,
                                     const SeqRows& sr) {
  if (!r.valid || k >= sr.lk) return false;
  if (!partial) return true;
  if (POLICY == kPolicyDflash) return (k >= r.clo && k < r.chi) || (k >= r.dlo && k < r.dhi);
  return k <= r.causal_lim && (r.mrow == nullptr || r.mrow[aux_col(k, p.mask.kd)] != 0);
}

// dS of one (query row, key): log2-domain score s2 (scale * log2 e folded
// into q), the row's lse in log2 units, dP and D.
__device__ __forceinline__ float ds_of(float s2, float lse2, float dp, float dd, bool keep) {
  const float pr = keep ? exp2f(s2 - lse2) : 0.f;
  return pr * (dp - dd);
}

template <int D, int POLICY>
__global__ void __launch_bounds__(kBsThreads) attn_bwd_simt_dq_kernel(const BwdProblem bp) {
  constexpr int E = D / 2;
  const AttnProblem& p = bp.f;
  __shared__ float sk[kBsChunk][D];
  __shared__ float sv[kBsChunk][D];
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const int r = threadIdx.x >> 1, hf = threadIdx.x & 1;
  const int q = qt * kTile + r;
  const SeqRows sr = seq_rows<POLICY>(p, b);  // packed sequences: this sequence's rows
  const RowKeep rk = row_keep<POLICY>(p, b, h, hk, q, sr);

  const int lb = p.lists.LB > 1 ? b : 0;
  int lh = 0;
  if (p.lists.head_mode == 1) lh = hk;
  else if (p.lists.head_mode == 2) lh = hk * p.npairs + (h - hk * p.group) / 2;
  const int64_t row = (static_cast<int64_t>(lb) * p.lists.LH + lh) * p.QT + qt;
  const int nf = p.lists.num_full[row], np = p.lists.num_part[row];

  const float* Q = reinterpret_cast<const float*>(p.q);
  const float* K = reinterpret_cast<const float*>(p.k);
  const float* V = reinterpret_cast<const float*>(p.v);
  const float* G = reinterpret_cast<const float*>(bp.dout);
  float qr[E], gr[E], acc[E];
  float lse2 = -INFINITY, dd = 0.f;
  if (rk.valid) {
    const float l = p.lse[row_index<POLICY>(p, b, h, sr, q)];
    lse2 = l * kLog2e;
    dd = bp.dvec[row_index<POLICY>(p, b, h, sr, q)];
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t qi = b * p.q_sb + static_cast<int64_t>(sr.q_off + q) * p.q_sr + h * p.q_sh + 2 * e + hf;
    const int64_t gi =
        b * bp.do_sb + static_cast<int64_t>(sr.q_off + q) * bp.do_sr + h * bp.do_sh + 2 * e + hf;
    qr[e] = rk.valid ? Q[qi] * p.scale_log2 : 0.f;
    gr[e] = rk.valid ? G[gi] : 0.f;
    acc[e] = 0.f;
  }
  float* dbrow = nullptr;
  if (POLICY != kPolicyDflash && bp.db_mode != kDbiasNone && rk.valid)
    dbrow = bp.dbias + b * bp.db_sb + (bp.db_head_per_query ? h : hk) * bp.db_sh +
            static_cast<int64_t>(q) * bp.db_sq;

  for (int t = 0; t < nf + np; ++t) {
    const bool partial = t >= nf;
    const int kt = partial ? p.lists.part_idx[row * p.KT + (t - nf)] : p.lists.full_idx[row * p.KT + t];
    for (int c0 = kt * kTile; c0 < kt * kTile + kTile; c0 += kBsChunk) {
      __syncthreads();
      for (int i = threadIdx.x; i < kBsChunk * D; i += kBsThreads) {
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
      for (int kk = 0; kk < kBsChunk; ++kk) {
        float s2 = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s2 = fmaf(qr[e], sk[kk][2 * e + hf], s2);
          dp = fmaf(gr[e], sv[kk][2 * e + hf], dp);
        }
        s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
        dp += __shfl_xor_sync(0xffffffffu, dp, 1);
        const int k = c0 + kk;
        if (POLICY != kPolicyDflash && rk.brow != nullptr && k < sr.lk)
          s2 = fmaf(load_any_as_float(rk.brow, p.bias.dtype, aux_col(k, p.bias.kd)), kLog2e, s2);
        const bool keep = keeps<POLICY>(p, rk, k, partial, sr) && lse2 != -INFINITY;
        const float ds = ds_of(s2, lse2, dp, dd, keep);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(ds, sk[kk][2 * e + hf], acc[e]);
        if (dbrow != nullptr && hf == 0 && k < sr.lk && k < bp.db_kd) {
          if (bp.db_mode == kDbiasStore) dbrow[k] = ds;
          else if (ds != 0.f) atomicAdd(dbrow + k, ds);
        }
      }
    }
  }
  if (rk.valid) {
    // [B, Lq, H, d], or [total_q, H, d] for packed sequences
    const int64_t arow = POLICY == kPolicyVarlen ? static_cast<int64_t>(sr.q_off) + q
                                                 : static_cast<int64_t>(b) * p.Lq + q;
    float* A = bp.dq_acc + (arow * p.H + h) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) A[2 * e + hf] = acc[e];
  }
}

template <int D, int POLICY>
__global__ void __launch_bounds__(kBsThreads) attn_bwd_simt_dkv_kernel(const BwdProblem bp) {
  constexpr int E = D / 2;
  const AttnProblem& p = bp.f;
  __shared__ float sq[kBsChunk][D];   // Q rows
  __shared__ float sg[kBsChunk][D];   // dO rows
  __shared__ float sl[kBsChunk], sd[kBsChunk];
  const int kt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x >> 1, hf = threadIdx.x & 1;
  const int k = kt * kTile + r;
  const SeqRows sr = seq_rows<POLICY>(p, b);  // packed sequences: this sequence's rows
  const bool key_valid = k < sr.lk;
  const float* Q = reinterpret_cast<const float*>(p.q);
  const float* K = reinterpret_cast<const float*>(p.k);
  const float* V = reinterpret_cast<const float*>(p.v);
  const float* G = reinterpret_cast<const float*>(bp.dout);
  float kr[E], vr[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kr[e] = key_valid ? K[b * p.k_sb + static_cast<int64_t>(sr.k_off + k) * p.k_sr + hk * p.k_sh + 2 * e + hf]
                      : 0.f;
    vr[e] = key_valid ? V[b * p.v_sb + static_cast<int64_t>(sr.k_off + k) * p.v_sr + hk * p.v_sh + 2 * e + hf]
                      : 0.f;
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  for (int g = 0; g < p.group; ++g) {
    const int h = hk * p.group + g;
    const int lb = p.lists.LB > 1 ? b : 0;
    int lh = 0;
    if (p.lists.head_mode == 1) lh = hk;
    else if (p.lists.head_mode == 2) lh = hk * p.npairs + g / 2;
    const int64_t trow = (static_cast<int64_t>(lb) * p.lists.LH + lh) * p.KT + kt;
    const int nf = bp.t_num_full[trow], np = bp.t_num_part[trow];
    for (int t = 0; t < nf + np; ++t) {
      const bool partial = t >= nf;
      const int qt = partial ? bp.t_part[trow * p.QT + (t - nf)] : bp.t_full[trow * p.QT + t];
      for (int c0 = qt * kTile; c0 < qt * kTile + kTile; c0 += kBsChunk) {
        __syncthreads();
        for (int i = threadIdx.x; i < kBsChunk * D; i += kBsThreads) {
          const int qq = i / D, e = i - qq * D;
          const int q = c0 + qq;
          float qv = 0.f, gv = 0.f;
          if (q < sr.lq) {
            qv = Q[b * p.q_sb + static_cast<int64_t>(sr.q_off + q) * p.q_sr + h * p.q_sh + e];
            gv = G[b * bp.do_sb + static_cast<int64_t>(sr.q_off + q) * bp.do_sr + h * bp.do_sh + e];
          }
          sq[qq][e] = qv;
          sg[qq][e] = gv;
        }
        if (threadIdx.x < kBsChunk) {
          const int q = c0 + threadIdx.x;
          float l2 = -INFINITY, dd = 0.f;
          if (q < sr.lq) {
            l2 = p.lse[row_index<POLICY>(p, b, h, sr, q)] * kLog2e;
            dd = bp.dvec[row_index<POLICY>(p, b, h, sr, q)];
          }
          sl[threadIdx.x] = l2;
          sd[threadIdx.x] = dd;
        }
        __syncthreads();
        for (int qq = 0; qq < kBsChunk; ++qq) {
          const int q = c0 + qq;
          float s2 = 0.f, dp = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            s2 = fmaf(kr[e], sq[qq][2 * e + hf], s2);
            dp = fmaf(vr[e], sg[qq][2 * e + hf], dp);
          }
          s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
          dp += __shfl_xor_sync(0xffffffffu, dp, 1);
          s2 *= p.scale_log2;
          const RowKeep rk = row_keep<POLICY>(p, b, h, hk, q, sr);
          if (POLICY != kPolicyDflash && rk.brow != nullptr && key_valid)
            s2 = fmaf(load_any_as_float(rk.brow, p.bias.dtype, aux_col(k, p.bias.kd)), kLog2e, s2);
          const bool keep = key_valid && keeps<POLICY>(p, rk, k, partial, sr) && sl[qq] != -INFINITY;
          const float pr = keep ? exp2f(s2 - sl[qq]) : 0.f;
          const float ds = pr * (dp - sd[qq]);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            dk[e] = fmaf(ds, sq[qq][2 * e + hf], dk[e]);
            dv[e] = fmaf(pr, sg[qq][2 * e + hf], dv[e]);
          }
        }
      }
    }
  }
  if (key_valid) {
    float* DK = reinterpret_cast<float*>(bp.dk);
    float* DV = reinterpret_cast<float*>(bp.dv);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      DK[b * bp.dk_sb + static_cast<int64_t>(sr.k_off + k) * bp.dk_sr + hk * bp.dk_sh + 2 * e + hf] =
          dk[e] * bp.scale;
      DV[b * bp.dv_sb + static_cast<int64_t>(sr.k_off + k) * bp.dv_sr + hk * bp.dv_sh + 2 * e + hf] = dv[e];
    }
  }
}

template <int D, int POLICY>
cudaError_t launch_typed(const BwdProblem& p, cudaStream_t stream) {
  if (p.f.QT > 0) {
    attn_bwd_simt_dq_kernel<D, POLICY><<<dim3(p.f.QT, p.f.H, p.f.B), kBsThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.f.KT > 0)
    attn_bwd_simt_dkv_kernel<D, POLICY><<<dim3(p.f.KT, p.f.KVH, p.f.B), kBsThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_simt(const BwdProblem& p, cudaStream_t stream) {
  if (p.f.d == 128) {
    if (p.f.policy == kPolicyDflash) return launch_typed<128, kPolicyDflash>(p, stream);
    if (p.f.policy == kPolicyVarlen) return launch_typed<128, kPolicyVarlen>(p, stream);
    return launch_typed<128, kPolicyExplicit>(p, stream);
  }
  if (p.f.policy == kPolicyDflash) return launch_typed<64, kPolicyDflash>(p, stream);
  if (p.f.policy == kPolicyVarlen) return launch_typed<64, kPolicyVarlen>(p, stream);
  return launch_typed<64, kPolicyExplicit>(p, stream);
}

}  // namespace sma
