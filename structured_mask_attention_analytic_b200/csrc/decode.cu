// Single-query attention (q_len == 1) with the grouped-head swap.
//
// flash-sparse-attention PR #190, "Swapped path (seqlen_q==1 and H>H_k)":
// the query heads of one KV head are reshaped to act as rows of a single
// problem, while mask/bias keep their original batch/head meaning and the lse
// write-back follows the original [B, H] order.  Here the swap is a change of
// loop order: a CTA owns (batch, KV head, group of up to G query heads, key
// chunk) and evaluates all its query heads against every key it loads, so K
// and V are read from HBM once per KV head instead of once per query head.
//
// The work is HBM-bound (each K/V element feeds G fused multiply-adds).  A
// producer warp streams K/V tiles with TMA (no multicast) into a ring of
// shared-memory stages and stages the matching bias/mask values next to them;
// four consumer warps compute from shared memory.  Keys are split into chunks
// across CTAs (split-KV); a second kernel merges the per-chunk (max, sum,
// unnormalised O) triples.
//
// Consumer lane layout: a key row is read by d/8 lanes, 8 elements each; the
// G dot products of a key are summed over those lanes in transposed form, so
// that each lane ends with one head's score and keeps that head's softmax.
#include <cudaTypedefs.h>

#include <cstdio>

#include "device_common.cuh"
#include "kernels.h"

namespace sma {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kDecThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kRing = 3;
constexpr int kTileBytes = 16384;  // one K (or V) tile per stage

template <int D, int DT>
struct DecLayout {
  static constexpr int kEsz = DT == SMA_FP32 ? 4 : 2;
  static constexpr int kT = kTileBytes / (D * kEsz);  // keys per tile
};

template <int DT>
__device__ __forceinline__ void smem8(const uint8_t* p, float (&f)[8]) {
  if (DT == SMA_FP32) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 c = *reinterpret_cast<const float4*>(p + 16);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
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

template <int DT>
__device__ __forceinline__ void global8(const void* base, int64_t idx, float (&f)[8]) {
  smem8<DT>(reinterpret_cast<const uint8_t*>(base) + idx * (DT == SMA_FP32 ? 4 : 2), f);
}

// grid: (splits, KVH * row_groups, B); rows [rg*G, rg*G+G) of the group.
template <int D, int G, int DT>
__global__ void __launch_bounds__(kDecThreads, G <= 4 ? 2 : 1)
decode_split_kernel(const DecodeProblem p, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v) {
  using L = DecLayout<D, DT>;
  constexpr int T = L::kT;
  constexpr int LPK = D / 8;     // lanes per key row
  constexpr int KPW = 32 / LPK;  // keys per warp step
  constexpr int kStageBytes = 2 * kTileBytes;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;                                          // kRing x (K tile, V tile)
  float* s_bias = reinterpret_cast<float*>(smem + kRing * kStageBytes);       // [kRing][G][T]
  uint8_t* s_keep = reinterpret_cast<uint8_t*>(s_bias + kRing * G * T);       // [kRing][G][T]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_keep + kRing * G * T);      // full, empty
  int* abort_i = reinterpret_cast<int*>(bars + 2 * kRing);
  volatile int* abort_flag = abort_i;
  float* s_o = reinterpret_cast<float*>(abort_i + 4);                         // [warps][G][D]
  float* s_ml = s_o + kConsumerWarps * G * D;                                 // [warps][G][2]

  const int split = blockIdx.x;
  const int row_groups = (p.group + G - 1) / G;
  const int hk = blockIdx.y / row_groups;
  const int rg = blockIdx.y - hk * row_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // split s takes key tiles [s nt / splits, (s + 1) nt / splits): shares
  // differ by at most one tile, and every range starts on a tile boundary
  const int nt_all = (p.Lk + T - 1) / T;
  const int k_begin = static_cast<int>(static_cast<int64_t>(split) * nt_all / p.splits) * T;
  const int k_end = min(p.Lk, static_cast<int>(static_cast<int64_t>(split + 1) * nt_all / p.splits) * T);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + T - 1) / T : 0;
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + kRing + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(full(s), 1 + 32);  // TMA byte count + the producer warp's 32 lanes
      mbar_init(empty(s), kConsumerWarps);
    }
    *abort_i = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------- producer
    bool ok = true;
    int issued = 0;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int s = t % kRing;
      const uint32_t use = t / kRing;
      if (use > 0 && !mbar_wait_warp(empty(s), (use - 1) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      const int k0 = k_begin + t * T;
      if (elect_one()) {
        mbar_arrive_expect_tx(full(s), 2 * kTileBytes);
        tma_load_4d(smem_u32(ring + s * kStageBytes), &map_k, full(s), 0, hk, k0, b);
        tma_load_4d(smem_u32(ring + s * kStageBytes + kTileBytes), &map_v, full(s), 0, hk, k0, b);
      }
      // bias / keep values of this tile for the CTA's G query heads: each lane
      // takes 8 consecutive keys of one row with one vector load per operand
      // (keys are 8-aligned and rows 16-byte aligned; ranges start on a
      // tile boundary, a multiple of 32 keys).
      constexpr int kGroups = T / 8;
#pragma unroll
      for (int i0 = 0; i0 < G * kGroups; i0 += 32) {
        const int i = i0 + lane;
        if (i < G * kGroups) {
          const int r = i / kGroups, c = (i - r * kGroups) * 8;
          const int k = k0 + c;
          const int gr = rg * G + r;
          const bool rv = gr < p.group;
          const int h = hk * p.group + (rv ? gr : 0);
          uint2 mb = make_uint2(0x01010101u, 0x01010101u);
          if (p.has_mask) {
            const int hm = p.mask.head_per_query ? h : hk;
            const uint8_t* mrow =
                reinterpret_cast<const uint8_t*>(p.mask.ptr) + b * p.mask.sb + hm * p.mask.sh;
            if (k + 8 <= p.mask.kd) {
              mb = *reinterpret_cast<const uint2*>(mrow + k);
            } else {  // a row of Lk or 1 columns: column by column, inside the row
              uint32_t w2[2] = {0u, 0u};
#pragma unroll
              for (int e = 0; e < 8; ++e)
                w2[e >> 2] |= (mrow[aux_col(k + e, p.mask.kd)] != 0 ? 1u : 0u) << (8 * (e & 3));
              mb = make_uint2(w2[0], w2[1]);
            }
          }
          float bv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          if (p.has_bias) {
            const int hb = p.bias.head_per_query ? h : hk;
            const int64_t bi = b * p.bias.sb + hb * p.bias.sh;
            if (k + 8 <= p.bias.kd) {
              if (p.bias.dtype == SMA_FP32) {
                global8<SMA_FP32>(p.bias.ptr, bi + k, bv);
              } else if (p.bias.dtype == SMA_BF16) {
                global8<SMA_BF16>(p.bias.ptr, bi + k, bv);
              } else {
                global8<SMA_FP16>(p.bias.ptr, bi + k, bv);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e)
                bv[e] = load_any_as_float(p.bias.ptr, p.bias.dtype, bi + aux_col(k + e, p.bias.kd));
            }
          }
          const uint32_t mw[2] = {mb.x, mb.y};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const bool keep = rv && (k + e) < k_end && ((mw[e >> 2] >> (8 * (e & 3))) & 0xffu) != 0u;
            s_bias[(s * G + r) * T + c + e] = keep ? bv[e] * kLog2e : 0.f;
            s_keep[(s * G + r) * T + c + e] = keep ? 1 : 0;
          }
        }
      }
      mbar_arrive(full(s));
      ++issued;
    }
    if (!ok) {
      // Copies already issued must land before the CTA exits.
      int never = 0;
      for (int t = max(0, issued - kRing); t < issued; ++t)
        mbar_wait(full(t % kRing), (t / kRing) & 1, &never, p.err);
    }
  } else {
    // ---------------------------------------------------------- consumers
    const int slot = lane / LPK, dl = lane - slot * LPK;
    const int e0 = dl * 8;
    float qf[G][8];
#pragma unroll
    for (int r = 0; r < G; ++r) {
      const int gr = rg * G + r;
      const int h = hk * p.group + (gr < p.group ? gr : 0);
      global8<DT>(p.q, b * p.q_sb + h * p.q_sh + e0, qf[r]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[r][e] *= p.scale_log2;
    }
    // Each lane keeps the online softmax of one query head of the CTA: head
    // hsel, the top log2(G) bits of its lane index within the key slot.
    constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
    constexpr int LL = LPK == 8 ? 3 : 4;
    static_assert(LPK == (1 << LL) && G == (1 << LG) && LG <= LL, "lane layout");
    const int hsel = dl >> (LL - LG);
    const int hbase = slot * LPK;  // first lane of this key slot
    float m_own = -INFINITY, l_own = 0.f;
    float o[G][8];
#pragma unroll
    for (int r = 0; r < G; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[r][e] = 0.f;
    // Per tile: the own head's score of every key of this warp first, then one
    // max / sum / rescale, then the P.V pass -- no branch.
    constexpr int kSteps = T / (kConsumerWarps * KPW);
    constexpr int kSub = kSteps < 4 ? kSteps : 4;  // key-steps per online-softmax update
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int s = t % kRing;
      if (!mbar_wait_warp(full(s), (t / kRing) & 1, abort_flag, p.err)) { ok = false; break; }
      const uint8_t* kt = ring + s * kStageBytes;
      const uint8_t* vt = kt + kTileBytes;
#pragma unroll
      for (int st0 = 0; st0 < kSteps; st0 += kSub) {
        float sc[kSub];  // the own head's scores, then probabilities
#pragma unroll
        for (int st = 0; st < kSub; ++st) {
          const int c = ((st0 + st) * kConsumerWarps + warp) * KPW + slot;
          float kf[8];
          smem8<DT>(kt + (c * D + e0) * L::kEsz, kf);
          float d[G];
#pragma unroll
          for (int r = 0; r < G; ++r) {
            // two products per instruction (fp32 pairs), the halves added last
            float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 8; e += 2)
              d2 = fma2(make_float2(qf[r][e], qf[r][e + 1]), make_float2(kf[e], kf[e + 1]), d2);
            d[r] = d2.x + d2.y;
          }
          // Sum over the LPK lanes of the key, transposed: step i (lane
          // offset LPK >> (i + 1)) keeps the half of the remaining heads that
          // the lane's bit selects and adds the partner's partial sums of it
          // (log2 G exchanges in place of G butterflies); a butterfly over
          // the remaining offsets completes the one head left.
#pragma unroll
          for (int i = 0; i < LG; ++i) {
            const int off = LPK >> (i + 1);
            const bool up = (dl & off) != 0;
            const int n = G >> i;
#pragma unroll
            for (int j = 0; j < (G >> (i + 1)); ++j) {
              const float mine = up ? d[j + n / 2] : d[j];
              const float give = up ? d[j] : d[j + n / 2];
              d[j] = mine + __shfl_xor_sync(0xffffffffu, give, off);
            }
          }
          float v = d[0];
#pragma unroll
          for (int off = LPK >> (LG + 1); off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
          const bool keep = s_keep[(s * G + hsel) * T + c] != 0;
          sc[st] = keep ? v + s_bias[(s * G + hsel) * T + c] : -INFINITY;
        }
        // the own head over these keys of every slot of the warp
        float mx = sc[0];
#pragma unroll
        for (int st = 1; st < kSub; ++st) mx = fmaxf(mx, sc[st]);
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_own, mx);
        const bool dead = m_new == -INFINITY;
        const float alpha = dead ? 1.f : fast_exp2(m_own - m_new);  // exp2(-inf) = 0
        const float msub = dead ? 0.f : m_new;
        float ps = 0.f;
#pragma unroll
        for (int st = 0; st < kSub; ++st) {
          sc[st] = fast_exp2(sc[st] - msub);
          ps += sc[st];
        }
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l_own = l_own * alpha + ps;
        m_own = m_new;
        // every head's rescale factor, from a lane of this slot that owns it
#pragma unroll
        for (int r = 0; r < G; ++r) {
          const float a_r = __shfl_sync(0xffffffffu, alpha, hbase + (r << (LL - LG)));
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 oo = mul2(make_float2(o[r][e], o[r][e + 1]), make_float2(a_r, a_r));
            o[r][e] = oo.x;
            o[r][e + 1] = oo.y;
          }
        }
#pragma unroll
        for (int st = 0; st < kSub; ++st) {
          const int c = ((st0 + st) * kConsumerWarps + warp) * KPW + slot;
          float vf[8];
          smem8<DT>(vt + (c * D + e0) * L::kEsz, vf);
#pragma unroll
          for (int r = 0; r < G; ++r) {
            const float p_r = __shfl_sync(0xffffffffu, sc[st], hbase + (r << (LL - LG)));
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 oo = fma2(make_float2(p_r, p_r), make_float2(vf[e], vf[e + 1]),
                                     make_float2(o[r][e], o[r][e + 1]));
              o[r][e] = oo.x;
              o[r][e + 1] = oo.y;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
    // Sum the key slots of the warp, then merge warps through shared memory.
#pragma unroll
    for (int r = 0; r < G; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1)
          o[r][e] += __shfl_xor_sync(0xffffffffu, o[r][e], off);
    if (slot == 0) {
#pragma unroll
      for (int r = 0; r < G; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) s_o[(warp * G + r) * D + e0 + e] = o[r][e];
    }
    // (max, sum) of each head from the first lane of slot 0 that owns it
    if (slot == 0 && (dl & ((1 << (LL - LG)) - 1)) == 0) {
      s_ml[(warp * G + hsel) * 2] = m_own;
      s_ml[(warp * G + hsel) * 2 + 1] = l_own;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int r = i / D, e = i - r * D;
    const int gr = rg * G + r;
    if (gr >= p.group) continue;
    float M = -INFINITY;
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_ml[(w * G + r) * 2]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = s_ml[(w * G + r) * 2];
        const float sc = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
        acc += sc * s_o[(w * G + r) * D + e];
        lsum += sc * s_ml[(w * G + r) * 2 + 1];
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
  for (int s = 0; s < p.splits; ++s)
    M = fmaxf(M, p.part_ml[(static_cast<int64_t>(bh) * p.splits + s) * 2]);
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [B][Lk][KVH][d] map; box = d x 1 x keys x 1, no swizzle, zero fill.
bool kv_map(CUtensorMap* m, const void* ptr, int dtype, int d, int kvh, int lk, int batch,
            int64_t s_head, int64_t s_row, int64_t s_batch, int box_rows) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  const int esz = dtype == SMA_FP32 ? 4 : 2;
  if (kvh == 1) s_head = d;
  if (lk == 1) s_row = s_head * kvh;
  if (batch == 1) s_batch = s_row * lk;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(kvh),
                        static_cast<cuuint64_t>(lk), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s_head * esz), static_cast<cuuint64_t>(s_row * esz),
                           static_cast<cuuint64_t>(s_batch * esz)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(d), 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  const CUtensorMapDataType t = dtype == SMA_FP32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dtype == SMA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return enc(m, t, 4, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, int DT>
cudaError_t launch3(const DecodeProblem& p, cudaStream_t stream) {
  using L = DecLayout<D, DT>;
  constexpr int T = L::kT;
  CUtensorMap mk, mv;
  if (!kv_map(&mk, p.k, p.dtype, D, p.KVH, p.Lk, p.B, p.k_sh, p.k_sr, p.k_sb, T) ||
      !kv_map(&mv, p.v, p.dtype, D, p.KVH, p.Lk, p.B, p.v_sh, p.v_sr, p.v_sb, T))
    return cudaErrorInvalidValue;
  const size_t smem = kRing * 2 * kTileBytes + kRing * G * T * 5 + 2 * kRing * 8 + 16 +
                      (kConsumerWarps * G * D + kConsumerWarps * G * 2) * 4;
  auto kern = decode_split_kernel<D, G, DT>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int row_groups = (p.group + G - 1) / G;
  dim3 grid(p.splits, p.KVH * row_groups, p.B);
  kern<<<grid, kDecThreads, smem, stream>>>(p, mk, mv);
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
