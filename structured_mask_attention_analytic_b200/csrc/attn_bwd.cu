// Attention backward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Gradients of the forward in attn_tc.cu for an upstream gradient dO, under
// the same mask families (DFlash analytic intervals, explicit mask / bias /
// causal): flash-sparse-attention PR #190 (Changes, mha_bwd) names the
// outputs dQ, dK, dV; the formulas are the derivative of softmax attention:
//   P  = exp(scale * Q K^T + bias - lse)          (recomputed from the forward's lse)
//   dV = P^T dO              dP = dO V^T          D = rowsum(dO * O)
//   dS = P * (dP - D)        dQ = scale * dS K    dK = scale * dS^T Q
//
// One kernel serves head dims 64 and 128 (attn_bwd_t_kernel below).  One
// persistent CTA per SM walks units (batch, KV head, 128-key tile).  A unit
// loops over the (query head of the group, 128-row query tile) pairs that
// attend its key tile -- the transposed tile lists -- accumulating dK and dV
// in TMEM over the whole group; each pair's dQ tile is added into an fp32
// accumulator in global memory by bulk tensor reductions from shared memory.
// The products are formed transposed (key rows in TMEM lanes), so P^T can
// stay in TMEM as dV's A operand and dS^T, stored once in shared memory,
// serves both dK (read K-major) and dQ (read MN-major); the layout of TMEM
// and shared memory and the warp roles are given with the kernel.
//
// The bias gradient is dS itself for a full bias and dS summed over the
// broadcast query axis otherwise.  Such sums are added with atomics by
// default; in the deterministic mode each 64-query group's sum is stored to
// its own slot and a second kernel (dbias_reduce_kernel) adds the slots in a
// fixed order, so dbias is bit-identical from run to run.
// Every mbarrier wait is bounded; on expiry the CTA raises its abort flag,
// drains its own copies and products, frees TMEM and returns.
#include <cstdio>
#include <type_traits>

#include "device_common.cuh"
#include "kernels.h"
#include "tma_map.h"

namespace sma {
namespace {

constexpr uint32_t kBTmemCols = 512;

// Transposed-list row of the query heads g of a unit.
__device__ __forceinline__ int64_t bwd_row(const BwdProblem& p, int b, int hk, int g) {
  const int lb = p.f.lists.LB > 1 ? b : 0;
  int lh = 0;
  if (p.f.lists.head_mode == 1) lh = hk;
  else if (p.f.lists.head_mode == 2) lh = hk * p.f.npairs + g / 2;
  return static_cast<int64_t>(lb) * p.f.lists.LH + lh;
}

// A unit's rows: padded batches read batch b's rows [0, Lq) / [0, Lk) at
// batch coordinate b; packed batches (cu_q / cu_k set) read sequence b's rows
// [q_off, q_off + lq) / [k_off, k_off + lk) of the one packed batch.
struct BUnit {
  int b, hk, kt, n_pairs;
  int bt;                    // batch coordinate of the operands
  int q_off, k_off, lq, lk;  // the unit's first rows and lengths
};

__device__ __forceinline__ BUnit bwd_unit(const BwdProblem& p, int u) {
  BUnit w;
  const int per_kt = p.f.B * p.f.KVH;
  w.kt = u / per_kt;  // key tiles in ascending order: early (context) tiles carry the most pairs
  const int r = u - w.kt * per_kt;
  w.b = r / p.f.KVH;
  w.hk = r - w.b * p.f.KVH;
  bool empty = false;
  if (p.f.cu_q != nullptr) {
    w.bt = 0;
    w.q_off = p.f.cu_q[w.b];
    w.lq = p.f.cu_q[w.b + 1] - w.q_off;
    w.k_off = p.f.cu_k[w.b];
    w.lk = p.f.cu_k[w.b + 1] - w.k_off;
    // malformed offsets (reported by the list kernel): nothing of the sequence
    // is read or written
    if (w.lq < 0 || w.lq > p.f.Lq || w.q_off < 0 || w.q_off + w.lq > p.f.total_q || w.lk < 0 ||
        w.lk > p.f.Lk || w.k_off < 0 || w.k_off + w.lk > p.f.total_k) {
      w.q_off = w.k_off = w.lq = w.lk = 0;
      empty = true;
    }
  } else {
    w.bt = w.b;
    w.q_off = w.k_off = 0;
    w.lq = p.f.Lq;
    w.lk = p.f.Lk;
  }
  int n = 0;
  for (int g = 0; g < p.f.group; ++g) {
    const int64_t row = bwd_row(p, w.b, w.hk, g);
    n += p.t_num_full[row * p.f.KT + w.kt] + p.t_num_part[row * p.f.KT + w.kt];
  }
  w.n_pairs = empty ? 0 : n;
  return w;
}

// Index of (head h, query q of the unit) in the [B, H, rows] per-query arrays
// (lse, rowsum(dO * O)); packed batches: [H, total_q].
__device__ __forceinline__ int64_t qrow(const BwdProblem& p, const BUnit& w, int h, int q) {
  const int rows = p.f.cu_q != nullptr ? p.f.total_q : p.f.Lq;
  return (static_cast<int64_t>(w.bt) * p.f.H + h) * rows + w.q_off + q;
}

// Walks the pairs of a unit in the order every role uses: heads of the group
// outer, the key tile's query tiles (FULL first, then PARTIAL) inner.
struct PairWalk {
  int g, t, nf, np, G;
  int64_t row;
  __device__ __forceinline__ void begin(const BwdProblem& p, const BUnit& w) {
    G = p.f.group;
    g = 0;
    t = 0;
    load(p, w);
    settle(p, w);
  }
  __device__ __forceinline__ void load(const BwdProblem& p, const BUnit& w) {
    row = bwd_row(p, w.b, w.hk, g);
    nf = p.t_num_full[row * p.f.KT + w.kt];
    np = p.t_num_part[row * p.f.KT + w.kt];
  }
  __device__ __forceinline__ void settle(const BwdProblem& p, const BUnit& w) {
    while (t >= nf + np && g + 1 < G) {
      ++g;
      t = 0;
      load(p, w);
    }
  }
  __device__ __forceinline__ void next(const BwdProblem& p, const BUnit& w) {
    ++t;
    settle(p, w);
  }
  __device__ __forceinline__ int head(const BUnit& w) const { return w.hk * G + g; }
  __device__ __forceinline__ int qtile(const BwdProblem& p, const BUnit& w, bool* partial) const {
    const int64_t base = (row * p.f.KT + w.kt) * p.f.QT;
    if (t < nf) {
      *partial = false;
      return p.t_full[base + t];
    }
    *partial = true;
    return p.t_part[base + (t - nf)];
  }
};

__device__ __forceinline__ void bdrain_wait(uint32_t bar, uint32_t parity, int* err) {
  int never = 0;
  volatile int* nv = &never;
  mbar_wait(bar, parity, nv, err);
}

// 16-byte unit u (8 columns) of row r of a 128-byte-swizzled [128][128] tile.
__device__ __forceinline__ uint32_t sw128_unit(uint32_t base, int r, int u) {
  return base + static_cast<uint32_t>((u >> 3) * (kTile * 128) + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

template <int DT>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if (DT == SMA_BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// ---------------------------------------------------------------------------
// The transposed form (head dim 64 or 128).  The compute threads own key rows:
//   S^T  = K Q^T        A = K (K-major)        B = Q (K-major)        SS
//   dP^T = V dO^T       A = V (K-major)        B = dO (K-major)       SS
//   dV  += P^T dO       A = P^T from TMEM      B = dO (MN-major)      TS
//   dK  += dS^T Q       A = dS^T from TMEM     B = Q (MN-major)       TS
//   dQ   = dS K         A = dS (MN-major)      B = K (MN-major)       SS
// P^T goes to TMEM as packed 16-bit pairs over S^T's columns (pcol below),
// as the forward's P does, so dV reads its A operand from TMEM; dS^T is
// packed beside it (dscol) for dK.  dS^T is also written once to shared
// memory, where read MN-major it is dS itself (queries contiguous), so dQ
// comes out with query rows in TMEM.  Shared-memory bandwidth is what binds
// this kernel at head dim 128 (the products read 8 KB of operands per
// 128x128x16 step from it), so operands come from TMEM wherever the layout
// allows.  Two 128-column TMEM regions X alternate between pairs:
// pair i puts S^T / P^T and later dQ in region X_i, dP^T in Y_i.  At head
// dim 128 (dV and dK take the other 256 columns) Y_i is X_{i+1}: S^T(i+1)
// is issued as soon as the compute threads have read dP^T(i) into
// registers (early in forming dS^T(i)), and dP^T(i+1) once dQ(i) has been
// drained.  At head dim 64 dV and dK take 128
// columns and Y has the last 128 of its own: S^T(i+1) is issued once dQ(i-1)
// has left X_{i+1} (while pair i is still forming P^T and dS^T), and
// dP^T(i+1) once dS^T(i) is formed.
// The producer stages, per pair, -lse * log2(e) and rowsum(dO * O) of the
// 128 queries (and, for DFlash, each query's kept key intervals) in shared
// memory next to the Q stage.
// Bulk tensor reduction (add) of a swizzled shared-memory box into global
// memory, tracked by the issuing thread's bulk group.
__device__ __forceinline__ void bulk_reduce_add_4d(const CUtensorMap* map, uint32_t src, int c0,
                                                   int c1, int c2, int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
      ::"l"(map), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16 warps in four warpgroups: compute (0-3, 4-7; each key row's 128 queries
// split in two halves), dQ drain + epilogue (8-11), and producer / MMA /
// per-query data / idle (12-15).  setmaxnreg moves registers from the last
// group to the drain group; the shares add up to at most the launch
// allocation (512 x kTLaunchRegs), and the host refuses to launch if the
// compiled register count differs.
constexpr int kBwdTThreads = 512;
constexpr int kTDrainWarp0 = 8;
constexpr int kTLoadWarp = 12;
constexpr int kTMmaWarp = 13;
constexpr int kBAuxWarp = 14;
constexpr int kTLaunchRegs = 128;
constexpr int kTDrainRegs = 144;
constexpr int kTCtrlRegs = 112;
static_assert(256 * kTLaunchRegs + 128 * kTDrainRegs + 128 * kTCtrlRegs <= kBwdTThreads * kTLaunchRegs,
              "register split must fit the launch allocation");

template <int D_>
struct TLayout {
  static constexpr int D = D_;
  static constexpr int kChunks = D / 64;              // 128-byte-swizzled column chunks of a tile
  static constexpr uint32_t kChunk = kTile * 128;
  static constexpr uint32_t kTileD = kTile * D * 2;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTileD;
  static constexpr uint32_t kQ = kV + kTileD;        // 2 stages
  static constexpr uint32_t kDO = kQ + 2 * kTileD;   // 1 stage
  static constexpr uint32_t kDS = kDO + kTileD;      // dS^T [key][query], 128 x 128 at any D
  static constexpr uint32_t kAux = kDS + kTile * kTile * 2;  // 2 stages of kAuxBytes
  static constexpr uint32_t kAuxBytes = 6 * kTile * 4;  // nl, dd, clo, chi, dlo, dhi
  // dQ staging for the bulk reductions: per drain warp 32 rows x 32 floats
  static constexpr uint32_t kStage = (kAux + 2 * kAuxBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kStageWarp = 32 * 32 * 4;
  static constexpr uint32_t kBars = kStage + 4 * kStageWarp;
  enum : int {
    kKVFull = 0, kKVEmpty, kQFull, kQEmpty = kQFull + 2, kAuxFull = kQEmpty + 2,
    kOFull = kAuxFull + 2, kOEmpty, kSFull, kSFull1, kPDone, kDPFull, kDPRead, kDSDone, kDQFull, kDQFree, kDSFree,
    kAccDone, kAccFree, kDrain, kNumBars
  };
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  // TMEM: S^T / P^T / dQ regions X at columns 0 and 128 (alternating by
  // pair), dV and dK accumulators, and dP^T in Y.  At head dim 128 the four
  // 128-column regions fill TMEM and Y is the other X region; at head dim 64
  // dV and dK take 64 columns each and Y has a region of its own (columns
  // 384-511), so S^T of the next pair can go in while this pair is in flight.
  static constexpr bool kOwnY = D == 64;
  static constexpr uint32_t kColDV = 256, kColDK = D == 64 ? 320 : 384, kColY = 384;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// Packed P^T column of query column q: each 64-query half packs into the
// first half of its own S^T columns (queries 0-63 -> columns 0-31, queries
// 64-127 -> columns 64-95), so the two compute warps of a key row never
// write columns the other has yet to read.
__host__ __device__ constexpr uint32_t pcol(int q) {
  return static_cast<uint32_t>((q & ~63) + (q & 63) / 2);
}
// Packed dS^T column of query column q: the other half of the same 64
// columns (queries 0-63 -> columns 32-63, queries 64-127 -> 96-127), again
// written only by the thread that read them.
__host__ __device__ constexpr uint32_t dscol(int q) { return pcol(q) + 32u; }

template <int D, int POLICY, int DT>
__global__ void __launch_bounds__(kBwdTThreads, 1)
attn_bwd_t_kernel(const BwdProblem p, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_dq,
                  int n_units) {
  using L = TLayout<D>;
  // Head dim 128, DFlash: the dS pass releases Y as soon as it has read
  // dP^T, and the next pair's S^T is issued then.  The explicit-mask kernel
  // keeps the later hand-over: the extra registers it needs there spill and
  // cost more than the earlier start gains (packed-sequence backward 9.3 ->
  // 9.8 ms).
  constexpr bool kEarlyY = !L::kOwnY && POLICY == kPolicyDflash;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned by offsetting the shared array itself, so that pointers
  // derived from it keep the shared state space (shared loads, not generic)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  auto aux_f = [&](int stage, int which) -> float* {
    return reinterpret_cast<float*>(smem + L::kAux + stage * L::kAuxBytes + which * kTile * 4);
  };
  auto aux_i = [&](int stage, int which) -> int* {
    return reinterpret_cast<int*>(smem + L::kAux + stage * L::kAuxBytes + which * kTile * 4);
  };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // units are listed by key tile, which orders them by work except across
  // packed sequences of different lengths
  const bool snake = p.f.cu_q == nullptr;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kKVFull), 1);
    mbar_init(bar(L::kKVEmpty), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::kQFull + s), 1);
      mbar_init(bar(L::kQEmpty + s), 1);
      mbar_init(bar(L::kAuxFull + s), 32);
    }
    mbar_init(bar(L::kOFull), 1);
    mbar_init(bar(L::kOEmpty), 1);
    mbar_init(bar(L::kSFull), 1);
    mbar_init(bar(L::kSFull1), 1);
    mbar_init(bar(L::kPDone), 256);
    mbar_init(bar(L::kDPFull), 1);
    mbar_init(bar(L::kDPRead), 256);
    mbar_init(bar(L::kDSDone), 256);
    mbar_init(bar(L::kDQFull), 1);
    mbar_init(bar(L::kDQFree), 128);
    mbar_init(bar(L::kDSFree), 1);
    mbar_init(bar(L::kAccDone), 1);
    mbar_init(bar(L::kAccFree), 128);
    mbar_init(bar(L::kDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kBTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kTLoadWarp) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kTCtrlRegs));
   if (warp == kTLoadWarp) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_map(&map_q);
      tma_prefetch_map(&map_k);
      tma_prefetch_map(&map_v);
      tma_prefetch_map(&map_do);
    }
    __syncwarp();
    uint32_t kv_it = 0, q_it = 0, o_it = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0, snake); u < n_units && ok; u = snake_unit(++rnd, snake)) {
      const BUnit w = bwd_unit(p, u);
      if (w.n_pairs == 0) continue;
      if (kv_it > 0 && !mbar_wait_warp(bar(L::kKVEmpty), (kv_it - 1) & 1, abort_flag, p.f.err)) {
        ok = false;
        break;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(L::kKVFull), 2 * L::kTileD);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_4d(sbase + L::kK + c * L::kChunk, &map_k, bar(L::kKVFull), c * 64, w.hk,
                      w.k_off + w.kt * kTile, w.bt);
          tma_load_4d(sbase + L::kV + c * L::kChunk, &map_v, bar(L::kKVFull), c * 64, w.hk,
                      w.k_off + w.kt * kTile, w.bt);
        }
      }
      __syncwarp();
      ++kv_it;
      PairWalk pw;
      pw.begin(p, w);
      for (int i = 0; i < w.n_pairs && ok; ++i, pw.next(p, w)) {
        bool partial;
        const int qt = pw.qtile(p, w, &partial);
        const int h = pw.head(w);
        const int s = q_it & 1;
        const uint32_t use = q_it >> 1;
        if (use > 0 && !mbar_wait_warp(bar(L::kQEmpty + s), (use - 1) & 1, abort_flag, p.f.err)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::kQFull + s), L::kTileD);
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sbase + L::kQ + s * L::kTileD + c * L::kChunk, &map_q, bar(L::kQFull + s),
                        c * 64, h, w.q_off + qt * kTile, w.bt);
        }
        __syncwarp();
        ++q_it;
        if (o_it > 0 && !mbar_wait_warp(bar(L::kOEmpty), (o_it - 1) & 1, abort_flag, p.f.err)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::kOFull), L::kTileD);
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sbase + L::kDO + c * L::kChunk, &map_do, bar(L::kOFull), c * 64, h,
                        w.q_off + qt * kTile, w.bt);
        }
        __syncwarp();
        ++o_it;
      }
    }
    if (!ok) {
      if (kv_it > 0) bdrain_wait(bar(L::kKVFull), (kv_it - 1) & 1, p.f.err);
      for (uint32_t t = 0; t < 2; ++t) {
        if (q_it > t) {
          const uint32_t nn = q_it - 1 - t;
          bdrain_wait(bar(L::kQFull + (nn & 1)), (nn >> 1) & 1, p.f.err);
        }
      }
      if (o_it > 0) bdrain_wait(bar(L::kOFull), (o_it - 1) & 1, p.f.err);
    }
   } else if (warp == kBAuxWarp) {
    // ------------------------------------------------------------ per-query data
    // -lse * log2(e), rowsum(dO * O) and (DFlash) the kept key intervals of the
    // pair's 128 queries, 4 per lane; the global reads of the next pair are in
    // flight while the stage is still in use.
    uint32_t q_it = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0, snake); u < n_units && ok; u = snake_unit(++rnd, snake)) {
      const BUnit w = bwd_unit(p, u);
      if (w.n_pairs == 0) continue;
      PairWalk pw;
      pw.begin(p, w);
      for (int i = 0; i < w.n_pairs && ok; ++i, pw.next(p, w)) {
        bool partial;
        const int qt = pw.qtile(p, w, &partial);
        const int h = pw.head(w);
        float n_l[4], d_v[4];
        int clo[4], chi[4], dlo[4], dhi[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int q = qt * kTile + lane * 4 + j;
          n_l[j] = -INFINITY;
          d_v[j] = 0.f;
          clo[j] = chi[j] = dlo[j] = dhi[j] = 0;
          if (q < w.lq) {
            const int64_t row = qrow(p, w, h, q);
            const float l = p.f.lse[row];
            n_l[j] = l == -INFINITY ? -INFINITY : -l * kLog2e;
            d_v[j] = p.dvec[row];
            if (POLICY == kPolicyDflash) {
              const int jb = q / p.f.bs, ii = q - jb * p.f.bs;
              int a = p.f.anchors[static_cast<int64_t>(w.b) * p.f.N + jb];
              a = a < 0 ? 0 : (a > p.f.Lc ? p.f.Lc : a);
              chi[j] = a;
              clo[j] = p.f.window > 0 ? max(0, a + ii - p.f.window + 1) : 0;
              if (clo[j] > chi[j]) clo[j] = chi[j];
              const int base = p.f.Lc + jb * p.f.bs;
              dlo[j] = base + (p.f.window > 0 ? max(0, ii - p.f.window + 1) : 0);
              dhi[j] = base + (p.f.causal_in_block ? ii + 1 : p.f.bs);
            }
          }
        }
        const int s = q_it & 1;
        const uint32_t use = q_it >> 1;
        if (use > 0 && !mbar_wait_warp(bar(L::kQEmpty + s), (use - 1) & 1, abort_flag, p.f.err)) {
          ok = false;
          break;
        }
        float4* nl4 = reinterpret_cast<float4*>(aux_f(s, 0)) + lane;
        float4* dd4 = reinterpret_cast<float4*>(aux_f(s, 1)) + lane;
        int4* iv4 = reinterpret_cast<int4*>(aux_i(s, 2)) + lane;
        *nl4 = make_float4(n_l[0], n_l[1], n_l[2], n_l[3]);
        *dd4 = make_float4(d_v[0], d_v[1], d_v[2], d_v[3]);
        iv4[0] = make_int4(clo[0], clo[1], clo[2], clo[3]);
        iv4[kTile / 4] = make_int4(chi[0], chi[1], chi[2], chi[3]);
        iv4[2 * kTile / 4] = make_int4(dlo[0], dlo[1], dlo[2], dlo[3]);
        iv4[3 * kTile / 4] = make_int4(dhi[0], dhi[1], dhi[2], dhi[3]);
        mbar_arrive(bar(L::kAuxFull + s));
        ++q_it;
      }
    }
   } else if (warp == kTMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t fmt = DT == SMA_BF16 ? 1u : 0u;
    constexpr uint32_t idesc_ss = mma_idesc_f16(fmt, 128, 128, 0, 0);  // S^T, dP^T
    constexpr uint32_t idesc_ts = mma_idesc_f16(fmt, 128, D, 0, 1);    // dV, dK (A in TMEM)
    constexpr uint32_t idesc_dq = mma_idesc_f16(fmt, 128, D, 1, 1);    // dQ (A = dS from dS^T, MN-major)
    auto with_lo = [](uint64_t d, uint32_t add) -> uint64_t {
      return (d & 0xffffffff00000000ull) | static_cast<uint32_t>(static_cast<uint32_t>(d) + add);
    };
    // C[128 keys][128 queries] = A[keys][d] B[queries][d]^T, both K-major
    auto issue_t = [&](uint32_t col, uint32_t a_addr, uint32_t b_addr) {
      const uint64_t ad = smem_desc_sw128(a_addr, 16, 1024);
      const uint64_t bd = smem_desc_sw128(b_addr, 16, 1024);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = ((s >> 2) * L::kChunk + (s & 3) * 32) >> 4;
        tc_mma_ss(tmem + col, with_lo(ad, off), with_lo(bd, off), idesc_ss, s > 0 ? 1u : 0u);
      }
    };
    // S^T and dP^T with k-steps interleaved
    auto issue_st_dpt = [&](uint32_t xcol, uint32_t ycol, uint32_t q_addr) {
      const uint64_t kd = smem_desc_sw128(sbase + L::kK, 16, 1024);
      const uint64_t qd = smem_desc_sw128(q_addr, 16, 1024);
      const uint64_t vd = smem_desc_sw128(sbase + L::kV, 16, 1024);
      const uint64_t od = smem_desc_sw128(sbase + L::kDO, 16, 1024);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = ((s >> 2) * L::kChunk + (s & 3) * 32) >> 4;
        tc_mma_ss(tmem + xcol, with_lo(kd, off), with_lo(qd, off), idesc_ss, s > 0 ? 1u : 0u);
        tc_mma_ss(tmem + ycol, with_lo(vd, off), with_lo(od, off), idesc_ss, s > 0 ? 1u : 0u);
      }
    };
    // acc[keys][d] (+)= A^T[keys][queries] B[queries][d], A packed in TMEM
    // (queries 16 s .. 16 s + 15 at packed column pcol(16 s))
    auto issue_ts = [&](uint32_t dcol, uint32_t acol, uint32_t b_addr, bool acc) {
      const uint64_t bd = smem_desc_sw128(b_addr, L::kChunk, 1024);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s)
        tc_mma_ts(tmem + dcol, tmem + acol + pcol(16 * s), with_lo(bd, (s * 2048) >> 4), idesc_ts,
                  (acc || s > 0) ? 1u : 0u);
    };
    // dK += dS^T Q (A = dS^T packed in TMEM beside P^T, queries 16 s ..
    // 16 s + 15 at dscol(16 s)), then dQ = dS K (A = the dS^T tile in shared
    // memory read MN-major: dS with queries contiguous).  dQ's first step
    // overwrites all of X, so every dK step is issued before it: one
    // thread's MMAs run in order.
    auto issue_dk_dq = [&](uint32_t xcol, uint32_t q_addr, bool acc) {
      const uint64_t qd = smem_desc_sw128(q_addr, L::kChunk, 1024);
      const uint64_t kd = smem_desc_sw128(sbase + L::kK, L::kChunk, 1024);
      const uint64_t sd = smem_desc_sw128(sbase + L::kDS, L::kChunk, 1024);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s)
        tc_mma_ts(tmem + L::kColDK, tmem + xcol + dscol(16 * s), with_lo(qd, (s * 2048) >> 4), idesc_ts,
                  (acc || s > 0) ? 1u : 0u);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s) {
        const uint32_t off = (s * 2048) >> 4;
        tc_mma_ss(tmem + xcol, with_lo(sd, off), with_lo(kd, off), idesc_dq, s > 0 ? 1u : 0u);
      }
    };
    uint32_t kv_it = 0, q_it = 0, o_it = 0, pit = 0, uit = 0;
    bool ok = true;
    auto wait = [&](int b_, uint32_t parity) -> bool {
      if (!mbar_wait_warp(bar(b_), parity, abort_flag, p.f.err)) ok = false;
      return ok;
    };
    for (int rnd = 0, u = snake_unit(0, snake); u < n_units && ok; u = snake_unit(++rnd, snake)) {
      const BUnit w = bwd_unit(p, u);
      const int n = w.n_pairs;
      if (n == 0) continue;
      if (!wait(L::kKVFull, kv_it & 1)) break;
      ++kv_it;
      {  // S^T(0), dP^T(0)
        const uint32_t X = (pit & 1) ? 128u : 0u, Y = L::kOwnY ? L::kColY : 128u - X;
        if (!wait(L::kQFull + (q_it & 1), (q_it >> 1) & 1)) break;
        if (!wait(L::kOFull, o_it & 1)) break;
        // Head dim 128: Y held dQ of the last pair.  Own Y: X held dQ two
        // pairs back, waited for during the last pair.
        if (!L::kOwnY && pit > 0 && !wait(L::kDQFree, (pit - 1) & 1)) break;
        tc_fence_after();
        if (elect_one()) {
          issue_st_dpt(X, Y, sbase + L::kQ + (q_it & 1) * L::kTileD);
          tc_commit(bar(L::kSFull + (pit & 1)));
          tc_commit(bar(L::kDPFull));
        }
        __syncwarp();
      }
      for (int i = 0; i < n && ok; ++i) {
        const uint32_t X = (pit & 1) ? 128u : 0u, Y = L::kOwnY ? L::kColY : 128u - X;
        const int qs = q_it & 1;
        const uint32_t nq = q_it + 1;
        // dV += P^T dO
        if (!wait(L::kPDone, pit & 1)) break;
        if (i == 0 && uit > 0 && !wait(L::kAccFree, (uit - 1) & 1)) break;
        tc_fence_after();
        if (elect_one()) {
          issue_ts(L::kColDV, X, sbase + L::kDO, i > 0);
          tc_commit(bar(L::kOEmpty));
        }
        __syncwarp();
        ++o_it;
        if (kEarlyY) {
          // Head dim 128, DFlash: Y is free once the compute threads have
          // read dP^T(i), early in forming dS^T(i): S^T(i+1) goes there then.
          if (!wait(L::kDPRead, pit & 1)) break;
          if (i + 1 < n) {
            if (!wait(L::kQFull + (nq & 1), (nq >> 1) & 1)) break;
            tc_fence_after();
            if (elect_one()) {
              issue_t(Y, sbase + L::kK, sbase + L::kQ + (nq & 1) * L::kTileD);
              tc_commit(bar(L::kSFull + ((pit + 1) & 1)));
            }
            __syncwarp();
          }
        } else if (L::kOwnY) {
          // S^T(i+1) into the other X region as soon as dQ(i-1) has left it,
          // while this pair's dS^T is still being formed.  The wait is taken
          // after a unit's last pair too, so that a unit's first pair finds
          // its X region free.
          if (pit > 0 && !wait(L::kDQFree, (pit - 1) & 1)) break;
          if (i + 1 < n) {
            if (!wait(L::kQFull + (nq & 1), (nq >> 1) & 1)) break;
            tc_fence_after();
            if (elect_one()) {
              issue_t(128u - X, sbase + L::kK, sbase + L::kQ + (nq & 1) * L::kTileD);
              tc_commit(bar(L::kSFull + ((pit + 1) & 1)));
            }
            __syncwarp();
          }
        }
        // dS^T(i) is formed: dK += dS^T Q and dQ = dS K (into X, after dV
        // read P^T).  Head dim 128 with explicit masks: S^T(i+1) goes into Y
        // first, Y being free now (dP^T(i) consumed).
        if (!wait(L::kDSDone, pit & 1)) break;
        constexpr bool kLateY = !L::kOwnY && !kEarlyY;
        if (kLateY && i + 1 < n && !wait(L::kQFull + (nq & 1), (nq >> 1) & 1)) break;
        tc_fence_after();
        if (elect_one()) {
          if (kLateY && i + 1 < n) {
            issue_t(Y, sbase + L::kK, sbase + L::kQ + (nq & 1) * L::kTileD);
            tc_commit(bar(L::kSFull + ((pit + 1) & 1)));
          }
          issue_dk_dq(X, sbase + L::kQ + qs * L::kTileD, i > 0);
          tc_commit(bar(L::kDQFull));
          tc_commit(bar(L::kDSFree));
          tc_commit(bar(L::kQEmpty + qs));
        }
        __syncwarp();
        ++q_it;
        ++pit;
        if (i + 1 < n) {
          // dP^T(i+1): head dim 128 into X once dQ(i) is drained (pair i+1's
          // Y); own Y once dP^T(i) is consumed (dS^T(i) formed, above)
          if (!wait(L::kOFull, o_it & 1)) break;
          if (!L::kOwnY && !wait(L::kDQFree, (pit - 1) & 1)) break;
          tc_fence_after();
          if (elect_one()) {
            issue_t(L::kOwnY ? L::kColY : X, sbase + L::kV, sbase + L::kDO);
            tc_commit(bar(L::kDPFull));
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (elect_one()) {
        tc_commit(bar(L::kAccDone));
        tc_commit(bar(L::kKVEmpty));
      }
      __syncwarp();
      ++uit;
    }
    if (!ok) {
      if (elect_one()) tc_commit(bar(L::kDrain));
      __syncwarp();
      bdrain_wait(bar(L::kDrain), 0, p.f.err);
    }
   }
  } else if (warp < kTDrainWarp0) {
    // ------------------------------------------------------------ compute (P^T, dS^T), key rows
    // warp w: key rows 32 (w % 4) .. +31, queries 64 (w / 4) .. +63
    const int r = (warp & 3) * 32 + lane;
    const int qb = (warp >> 2) * 64;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float scale_log2 = p.f.scale_log2;
    const float bias_mul = kLog2e / p.f.scale_log2;
    uint32_t pit = 0, q_it = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0, snake); u < n_units && ok; u = snake_unit(++rnd, snake)) {
      const BUnit w = bwd_unit(p, u);
      if (w.n_pairs == 0) continue;
      const int key = w.kt * kTile + r;
      PairWalk pw;
      pw.begin(p, w);
      for (int i = 0; i < w.n_pairs && ok; ++i, pw.next(p, w)) {
        bool partial;
        const int qt = pw.qtile(p, w, &partial);
        const int h = pw.head(w);
        const int q0 = qt * kTile;
        const uint32_t X = (pit & 1) ? 128u : 0u, Y = L::kOwnY ? L::kColY : 128u - X;
        const uint32_t xcol = tmem + lane_off + X, ycol = tmem + lane_off + Y;
        const int s = q_it & 1;
        const float* nl = aux_f(s, 0);
        const float* dd = aux_f(s, 1);
        const int* iv = aux_i(s, 2);
        const uint8_t* mcol = nullptr;  // mask[b, h?, q, key] at q = 0
        const uint8_t* bcol = nullptr;
        int64_t msq = 0, bsq = 0;
        int bdt = 0;
        if (POLICY != kPolicyDflash) {
          if (p.f.has_mask) {
            const int hm = p.f.mask.head_per_query ? h : w.hk;
            mcol = reinterpret_cast<const uint8_t*>(p.f.mask.ptr) + w.b * p.f.mask.sb + hm * p.f.mask.sh +
                   aux_col(key, p.f.mask.kd);
            msq = p.f.mask.sq;
          }
          if (p.f.has_bias) {
            const int hb = p.f.bias.head_per_query ? h : w.hk;
            bdt = p.f.bias.dtype;
            const int esz = bdt == SMA_FP32 ? 4 : 2;
            bcol = reinterpret_cast<const uint8_t*>(p.f.bias.ptr) +
                   (w.b * p.f.bias.sb + hb * p.f.bias.sh + aux_col(key, p.f.bias.kd)) * esz;
            bsq = p.f.bias.sq * esz;
          }
        }
        if (!mbar_wait(bar(L::kAuxFull + s), (q_it >> 1) & 1, abort_flag, p.f.err)) { ok = false; break; }
        // S^T of pair pit completes SFull + (pit & 1) (one barrier per X region)
        if (!mbar_wait(bar(L::kSFull + (pit & 1)), (pit >> 1) & 1, abort_flag, p.f.err)) { ok = false; break; }
        tc_fence_after();
        // ---- phase A: P^T = exp2(S^T * scale * log2 e - lse * log2 e), packed into X
        // FULL and PARTIAL pairs run separate copies of the loop, so that a
        // FULL pair carries none of the mask evaluation.
        auto phase_a = [&](auto masked_tag) {
          constexpr bool MASKED = decltype(masked_tag)::value;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            const int cq = qb + 32 * c;  // first query column of the chunk
            uint32_t xr[32];
            tmem_ld32_at(xcol + cq, xr);
            // keep bits of the chunk's 32 queries (PARTIAL pairs only; the loads
            // are volatile so that FULL pairs never pay for them)
            uint32_t kbits = 0xffffffffu;
            if (MASKED) {
              kbits = 0u;
              if (POLICY == kPolicyDflash) {
                const uint32_t ivs = sbase + L::kAux + s * L::kAuxBytes + 2 * kTile * 4 + cq * 4;
  #pragma unroll
                for (int g4 = 0; g4 < 8; ++g4) {
                  const uint4 lo = ld_shared_v4(ivs + 16 * g4);
                  const uint4 hi = ld_shared_v4(ivs + kTile * 4 + 16 * g4);
                  const uint4 dl = ld_shared_v4(ivs + 2 * kTile * 4 + 16 * g4);
                  const uint4 dh = ld_shared_v4(ivs + 3 * kTile * 4 + 16 * g4);
                  const int l4[4] = {static_cast<int>(lo.x), static_cast<int>(lo.y), static_cast<int>(lo.z), static_cast<int>(lo.w)};
                  const int h4[4] = {static_cast<int>(hi.x), static_cast<int>(hi.y), static_cast<int>(hi.z), static_cast<int>(hi.w)};
                  const int a4[4] = {static_cast<int>(dl.x), static_cast<int>(dl.y), static_cast<int>(dl.z), static_cast<int>(dl.w)};
                  const int b4[4] = {static_cast<int>(dh.x), static_cast<int>(dh.y), static_cast<int>(dh.z), static_cast<int>(dh.w)};
  #pragma unroll
                  for (int z = 0; z < 4; ++z) {
                    const bool keep = (key >= l4[z] && key < h4[z]) || (key >= a4[z] && key < b4[z]);
                    kbits |= (keep ? 1u : 0u) << (4 * g4 + z);
                  }
                }
              } else {
                const volatile uint8_t* mv = mcol;
  #pragma unroll 4
                for (int z = 0; z < 32; ++z) {
                  const int q = q0 + cq + z;
                  const int qc = q < p.f.Lq ? q : 0;
                  const bool keep = q < w.lq && key < w.lk && (!p.f.causal || key <= q + w.lk - w.lq) &&
                                    (!p.f.has_mask || mv[qc * msq] != 0);
                  kbits |= (keep ? 1u : 0u) << z;
                }
              }
            }
            tc_wait_ld();
            uint32_t pk[16];
  #pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 n4 = *reinterpret_cast<const float4*>(nl + cq + e);
              const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
              float xs[4], pv[4];
  #pragma unroll
              for (int z = 0; z < 4; ++z) {
                xs[z] = __uint_as_float(xr[e + z]);
                if (POLICY != kPolicyDflash && p.f.has_bias) {
                  const int q = q0 + cq + e + z;
                  const int qc = q < p.f.Lq ? q : 0;  // rows past Lq read row 0 (their P is 0)
                  xs[z] = fmaf(load_any_as_float(bcol + qc * bsq, bdt, 0), bias_mul, xs[z]);
                }
              }
              // exponent arguments two at a time (packed fp32 pairs)
              const float2 sl2 = make_float2(scale_log2, scale_log2);
              const float2 t01 = fma2(make_float2(xs[0], xs[1]), sl2, make_float2(nn[0], nn[1]));
              const float2 t23 = fma2(make_float2(xs[2], xs[3]), sl2, make_float2(nn[2], nn[3]));
              const float ts[4] = {t01.x, t01.y, t23.x, t23.y};
  #pragma unroll
              for (int z = 0; z < 4; ++z) pv[z] = ((kbits >> (e + z)) & 1u) ? fast_exp2(ts[z]) : 0.f;
              pk[e >> 1] = DT == SMA_BF16 ? pack_bf16x2(pv[0], pv[1]) : pack_f16x2(pv[0], pv[1]);
              pk[(e >> 1) + 1] = DT == SMA_BF16 ? pack_bf16x2(pv[2], pv[3]) : pack_f16x2(pv[2], pv[3]);
            }
            tmem_st16_at(xcol + pcol(cq), pk);
          }
        };
        if (partial) phase_a(std::true_type{});
        else phase_a(std::false_type{});
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::kPDone));

        // ---- phase B: dS^T = P^T (dP^T - D), stored to shared memory
        if (!mbar_wait(bar(L::kDPFull), pit & 1, abort_flag, p.f.err)) { ok = false; break; }
        if (pit > 0 && !mbar_wait(bar(L::kDSFree), (pit - 1) & 1, abort_flag, p.f.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // dbias: this thread's key column of dS over its 64 queries, added
        // where the bias broadcasts (or stored where each element is its own)
        float* dbcol = nullptr;
        // (a dbias row of Lk columns has none for this thread's key past it)
        const bool db_key = key < p.db_kd;
        if (POLICY != kPolicyDflash && p.db_mode != kDbiasNone)
          dbcol = p.dbias + w.b * p.db_sb + (p.db_head_per_query ? h : w.hk) * p.db_sh +
                  (db_key ? key : 0);
        // the fixed-order mode stores the sum over the thread's 64 queries in
        // row (q0 + qb) / 64 of the partial buffer, if those start inside Lq
        const bool db_grp = q0 + qb < p.f.Lq;
        auto phase_b = [&](auto mode_tag) {
          constexpr int MODE = decltype(mode_tag)::value;
          float rsum = 0.f;
          // dS^T of query chunk c from its 32 dP^T columns yr
          auto chunk = [&](int c, const uint32_t* yr) {
            const int cq = qb + 32 * c;
            uint32_t pr[16];
            tmem_ld16_at(xcol + pcol(cq), pr);
            tc_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 d4 = *reinterpret_cast<const float4*>(dd + cq + e);
              const float2 p01 = unpack2<DT>(pr[e >> 1]);
              const float2 p23 = unpack2<DT>(pr[(e >> 1) + 1]);
              // dS = P (dP - D), two at a time (packed fp32 pairs)
              const float2 s01 = mul2(p01, sub2(make_float2(__uint_as_float(yr[e]), __uint_as_float(yr[e + 1])),
                                                make_float2(d4.x, d4.y)));
              const float2 s23 = mul2(p23, sub2(make_float2(__uint_as_float(yr[e + 2]), __uint_as_float(yr[e + 3])),
                                                make_float2(d4.z, d4.w)));
              const float s0 = s01.x, s1 = s01.y, s2 = s23.x, s3 = s23.y;
              pk[e >> 1] = DT == SMA_BF16 ? pack_bf16x2(s0, s1) : pack_f16x2(s0, s1);
              pk[(e >> 1) + 1] = DT == SMA_BF16 ? pack_bf16x2(s2, s3) : pack_f16x2(s2, s3);
              if (MODE == kDbiasRowSum || MODE == kDbiasGroupStore) {
                rsum += (s0 + s1) + (s2 + s3);  // rows past Lq have P = 0, so dS = 0
              } else if (MODE != kDbiasNone) {
                const float sv[4] = {s0, s1, s2, s3};
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                  const int q = q0 + cq + e + z;
                  if (q < p.f.Lq && db_key) {
                    if (MODE == kDbiasStore) dbcol[q * p.db_sq] = sv[z];
                    else atomicAdd(dbcol + q * p.db_sq, sv[z]);
                  }
                }
              }
            }
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              st_shared_v4(sw128_unit(sbase + L::kDS, r, cq / 8 + v4), pk[4 * v4], pk[4 * v4 + 1],
                           pk[4 * v4 + 2], pk[4 * v4 + 3]);
            // and packed into X beside P^T: dK's A operand
            tmem_st16_at(xcol + dscol(cq), pk);
          };
          // kEarlyY: all 64 of this thread's dP^T columns first, so that Y is
          // released (DPRead) for the next pair's S^T while dS is still being
          // formed.  Otherwise one 32-column chunk at a time.
          if (kEarlyY) {
            uint32_t yr2[64];
            tmem_ld32_at(ycol + qb, yr2);
            tmem_ld32_at(ycol + qb + 32, yr2 + 32);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(L::kDPRead));
            chunk(0, yr2);
            chunk(1, yr2 + 32);
          } else {
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t ych[32];
              tmem_ld32_at(ycol + qb + 32 * c, ych);
              chunk(c, ych);
            }
          }
          if (MODE == kDbiasRowSum && db_key) atomicAdd(dbcol, rsum);
          if (MODE == kDbiasGroupStore && db_key && db_grp) dbcol[((q0 + qb) >> 6) * p.db_sq] = rsum;
        };
        if (POLICY == kPolicyDflash || p.db_mode == kDbiasNone)
          phase_b(std::integral_constant<int, kDbiasNone>{});
        else if (p.db_mode == kDbiasStore)
          phase_b(std::integral_constant<int, kDbiasStore>{});
        else if (p.db_mode == kDbiasAdd)
          phase_b(std::integral_constant<int, kDbiasAdd>{});
        else if (p.db_mode == kDbiasGroupStore)
          phase_b(std::integral_constant<int, kDbiasGroupStore>{});
        else
          phase_b(std::integral_constant<int, kDbiasRowSum>{});
        fence_async_shared();
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::kDSDone));
        ++pit;
        ++q_it;
      }
    }
  } else {
    // ------------------------------------------------------------ dQ drain, dK / dV epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kTDrainRegs));
    const int wq = warp - kTDrainWarp0;
    const int r = wq * 32 + lane;  // dQ: query row; dK / dV: key row
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t dv_col = tmem + lane_off + L::kColDV;
    const uint32_t dk_col = tmem + lane_off + L::kColDK;
    typedef typename std::conditional<DT == SMA_BF16, __nv_bfloat16, __half>::type OutT;
    uint32_t pit = 0, uit = 0;
    bool ok = true;
    bool bulk_pending = false;
    for (int rnd = 0, u = snake_unit(0, snake); u < n_units && ok; u = snake_unit(++rnd, snake)) {
      const BUnit w = bwd_unit(p, u);
      const int key = w.kt * kTile + r;
      OutT* dvrow = reinterpret_cast<OutT*>(p.dv) + w.bt * p.dv_sb + static_cast<int64_t>(w.k_off + key) * p.dv_sr +
                    w.hk * p.dv_sh;
      OutT* dkrow = reinterpret_cast<OutT*>(p.dk) + w.bt * p.dk_sb + static_cast<int64_t>(w.k_off + key) * p.dk_sr +
                    w.hk * p.dk_sh;
      if (w.n_pairs == 0) {  // keys no query attends: zero gradients
        if (key < w.lk) {
          for (int e = 0; e < D / 8; ++e) {
            reinterpret_cast<uint4*>(dvrow)[e] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(dkrow)[e] = make_uint4(0, 0, 0, 0);
          }
        }
        continue;
      }
      PairWalk pw;
      pw.begin(p, w);
      for (int i = 0; i < w.n_pairs && ok; ++i, pw.next(p, w)) {
        bool partial;
        const int qt = pw.qtile(p, w, &partial);
        const int h = pw.head(w);
        const uint32_t X = (pit & 1) ? 128u : 0u;
        const uint32_t qcol = tmem + lane_off + X;
        if (!mbar_wait(bar(L::kDQFull), pit & 1, abort_flag, p.f.err)) { ok = false; break; }
        tc_fence_after();
        // dQ row q0 + r: all of it to registers, TMEM freed at once; then per
        // 32-column chunk the warp's 32 rows go through its 4 KB staging box
        // (128-byte swizzle) into a bulk tensor add on the fp32 accumulator.
        // Rows past Lq fall outside the map and are not written.
        uint32_t v[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32_at(qcol + 32 * c, v + 32 * c);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(L::kDQFree));
        const uint32_t stage = sbase + L::kStage + wq * L::kStageWarp;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          if (bulk_pending) {
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            st_shared_v4(stage + lane * 128 + ((u ^ (lane & 7)) << 4), v[32 * c + 4 * u],
                         v[32 * c + 4 * u + 1], v[32 * c + 4 * u + 2], v[32 * c + 4 * u + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            bulk_reduce_add_4d(&map_dq, stage, 32 * c, h, w.q_off + qt * kTile + 32 * wq, w.bt);
            bulk_commit();
          }
          bulk_pending = true;
        }
        ++pit;
      }
      if (!ok) break;
      if (!mbar_wait(bar(L::kAccDone), uit & 1, abort_flag, p.f.err)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? dv_col : dk_col;
        const float mul = which == 0 ? 1.f : p.scale;
        OutT* dst = which == 0 ? dvrow : dkrow;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_at(col + 32 * c, v);
          tc_wait_ld();
          if (key < w.lk) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float a = __uint_as_float(v[2 * e]) * mul;
              const float bq = __uint_as_float(v[2 * e + 1]) * mul;
              pk[e] = DT == SMA_BF16 ? pack_bf16x2(a, bq) : pack_f16x2(a, bq);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(L::kAccFree));
      ++uit;
    }
    // the staging boxes must stay valid until the reductions are done
    if (lane == 0) bulk_wait_all0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTMmaWarp) tmem_dealloc(tmem, kBTmemCols);
}

template <int D, int POLICY, int DT>
cudaError_t launch_bwd_t(const BwdProblem& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mdq,
                         cudaStream_t stream) {
  auto kern = attn_bwd_t_kernel<D, POLICY, DT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    // The setmaxnreg split assumes exactly kTLaunchRegs registers per thread.
    if (fa.numRegs != kTLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(TLayout<D>::kAlloc));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int n_units = p.f.B * p.f.KVH * p.f.KT;
  if (n_units == 0) return cudaSuccess;
  const int grid = n_units < num_sms() ? n_units : num_sms();
  kern<<<grid, kBwdTThreads, TLayout<D>::kAlloc, stream>>>(p, mq, mk, mv, mdo, mdq, n_units);
  return cudaGetLastError();
}

// n consecutive elements (2 or 4) of a row as floats, one vector load.
template <int DT>
__device__ __forceinline__ void load_vec_as_float(const void* base, int n, float (&f)[4]) {
  if (DT == SMA_FP32) {
    if (n == 4) {
      const float4 a = *reinterpret_cast<const float4*>(base);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    } else {
      const float2 a = *reinterpret_cast<const float2*>(base);
      f[0] = a.x; f[1] = a.y;
    }
  } else {
    uint32_t w[2];
    if (n == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(base);
      w[0] = a.x; w[1] = a.y;
    } else {
      w[0] = *reinterpret_cast<const uint32_t*>(base);
      w[1] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 v = unpack2<DT>(w[i]);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
}

// D = rowsum(dO * O) of one (b, q, h) row per warp, and the row's fp32 dQ
// accumulator zeroed.  At head dim 64 or 128 each lane takes d / 32
// consecutive elements with one vector load per operand (scalar loads if a
// row is not aligned for them) and zeroes its part of the accumulator with
// one vector store.
template <int DT>
__global__ void bwd_prep_kernel(const BwdProblem p) {
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.f.B) * p.f.Lq * p.f.H;
  if (gw >= rows) return;
  const int h = static_cast<int>(gw % p.f.H);
  const int64_t bq = gw / p.f.H;
  const int q = static_cast<int>(bq % p.f.Lq);
  const int b = static_cast<int>(bq / p.f.Lq);
  const int d = p.f.d;
  constexpr int kEs = DT == SMA_FP32 ? 4 : 2;
  const uint8_t* orow = reinterpret_cast<const uint8_t*>(p.f.o) +
                        (b * p.f.o_sb + static_cast<int64_t>(q) * p.f.o_sr + h * p.f.o_sh) * kEs;
  const uint8_t* grow = reinterpret_cast<const uint8_t*>(p.dout) +
                        (b * p.do_sb + static_cast<int64_t>(q) * p.do_sr + h * p.do_sh) * kEs;
  float* acc = p.dq_acc + gw * d;
  const int per = d >> 5;
  const bool vec = (d == 64 || d == 128) &&
                   ((reinterpret_cast<uintptr_t>(orow) | reinterpret_cast<uintptr_t>(grow)) &
                    static_cast<uintptr_t>(per * kEs - 1)) == 0;
  float s = 0.f;
  if (vec) {
    float of[4], gf[4];
    load_vec_as_float<DT>(orow + lane * per * kEs, per, of);
    load_vec_as_float<DT>(grow + lane * per * kEs, per, gf);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < per) s = fmaf(of[i], gf[i], s);
    if (per == 4) reinterpret_cast<float4*>(acc)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    else reinterpret_cast<float2*>(acc)[lane] = make_float2(0.f, 0.f);
  } else {
    for (int e = lane; e < d; e += 32) s += load_as_float<DT>(orow, e) * load_as_float<DT>(grow, e);
    for (int e = lane; e < d; e += 32) acc[e] = 0.f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) p.dvec[(static_cast<int64_t>(b) * p.f.H + h) * p.f.Lq + q] = s;
}

// codes[row][qt][kt] from the forward lists (2 = FULL, 1 = PARTIAL); the
// buffer is zeroed first.
__global__ void scatter_codes_kernel(const BwdProblem p, uint8_t* codes) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rows = static_cast<int64_t>(p.f.lists.LB) * p.f.lists.LH * p.f.QT;
  if (t >= rows * p.f.KT) return;
  const int64_t lrow = t / p.f.KT;  // (row, qt)
  const int j = static_cast<int>(t - lrow * p.f.KT);
  const int nf = p.f.lists.num_full[lrow], np = p.f.lists.num_part[lrow];
  uint8_t* c = codes + lrow * p.f.KT;
  if (j < nf) {
    const int kt = p.f.lists.full_idx[lrow * p.f.KT + j];
    if (kt >= 0 && kt < p.f.KT) c[kt] = 2;
  }
  if (j < np) {
    const int kt = p.f.lists.part_idx[lrow * p.f.KT + j];
    if (kt >= 0 && kt < p.f.KT) c[kt] = 1;
  }
}

// Per (row, key tile): ascending query tiles, FULL and PARTIAL lists.
constexpr int kTrThreads = 128;
__global__ void __launch_bounds__(kTrThreads) transpose_lists_kernel(const BwdProblem p,
                                                                      const uint8_t* codes) {
  const int kt = blockIdx.x;
  const int64_t row = blockIdx.y;
  __shared__ uint32_t s_warp[kTrThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t out = (row * p.f.KT + kt);
  int32_t* tf = const_cast<int32_t*>(p.t_full) + out * p.f.QT;
  int32_t* tp = const_cast<int32_t*>(p.t_part) + out * p.f.QT;
  uint32_t nf = 0, np = 0;
  for (int q0 = 0; q0 < p.f.QT; q0 += kTrThreads) {
    const int qt = q0 + threadIdx.x;
    const uint8_t code = qt < p.f.QT ? codes[(row * p.f.QT + qt) * p.f.KT + kt] : 0;
    const uint32_t v = (code == 2 ? 1u : 0u) | (code == 1 ? 0x10000u : 0u);
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t2 = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t2;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    uint32_t base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kTrThreads / 32; ++w) {
      base += w < warp ? s_warp[w] : 0u;
      tot += s_warp[w];
    }
    __syncthreads();
    const uint32_t ex = base + incl - v;
    if (code == 2) tf[nf + (ex & 0xffffu)] = qt;
    if (code == 1) tp[np + (ex >> 16)] = qt;
    nf += tot & 0xffffu;
    np += tot >> 16;
  }
  for (int i = nf + threadIdx.x; i < p.f.QT; i += kTrThreads) tf[i] = -1;
  for (int i = np + threadIdx.x; i < p.f.QT; i += kTrThreads) tp[i] = -1;
  if (threadIdx.x == 0) {
    const_cast<int32_t*>(p.t_num_full)[out] = static_cast<int32_t>(nf);
    const_cast<int32_t*>(p.t_num_part)[out] = static_cast<int32_t>(np);
  }
}

// dQ = scale * accumulator in the output dtype, one (b, q, h) row per warp:
// at head dim 64 or 128 each lane converts d / 32 consecutive elements with
// one vector load and one vector store (scalar stores if the dQ row is not
// aligned for them).
template <int DT>
__global__ void dq_convert_kernel(const BwdProblem p) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.f.B) * p.f.Lq * p.f.H;
  if (row >= rows) return;
  const int h = static_cast<int>(row % p.f.H);
  const int64_t bq = row / p.f.H;
  const int q = static_cast<int>(bq % p.f.Lq);
  const int b = static_cast<int>(bq / p.f.Lq);
  const int d = p.f.d;
  constexpr int kEs = DT == SMA_FP32 ? 4 : 2;
  const float* src = p.dq_acc + row * d;
  const int64_t off = b * p.dq_sb + static_cast<int64_t>(q) * p.dq_sr + h * p.dq_sh;
  uint8_t* dst = reinterpret_cast<uint8_t*>(p.dq) + off * kEs;
  const int per = d >> 5;
  const bool vec = (d == 64 || d == 128) &&
                   (reinterpret_cast<uintptr_t>(dst) & static_cast<uintptr_t>(per * kEs - 1)) == 0;
  if (vec) {
    float a[4];
    if (per == 4) {
      const float4 v = reinterpret_cast<const float4*>(src)[lane];
      a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
    } else {
      const float2 v = reinterpret_cast<const float2*>(src)[lane];
      a[0] = v.x; a[1] = v.y; a[2] = 0.f; a[3] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] *= p.scale;
    uint8_t* dl = dst + lane * per * kEs;
    if (DT == SMA_FP32) {
      if (per == 4) *reinterpret_cast<float4*>(dl) = make_float4(a[0], a[1], a[2], a[3]);
      else *reinterpret_cast<float2*>(dl) = make_float2(a[0], a[1]);
    } else {
      const uint32_t w0 = DT == SMA_BF16 ? pack_bf16x2(a[0], a[1]) : pack_f16x2(a[0], a[1]);
      const uint32_t w1 = DT == SMA_BF16 ? pack_bf16x2(a[2], a[3]) : pack_f16x2(a[2], a[3]);
      if (per == 4) *reinterpret_cast<uint2*>(dl) = make_uint2(w0, w1);
      else *reinterpret_cast<uint32_t*>(dl) = w0;
    }
  } else {
    for (int e = lane; e < d; e += 32) {
      const float v = src[e] * p.scale;
      if (DT == SMA_FP32) reinterpret_cast<float*>(dst)[e] = v;
      else if (DT == SMA_BF16) reinterpret_cast<__nv_bfloat16*>(dst)[e] = __float2bfloat16_rn(v);
      else reinterpret_cast<__half*>(dst)[e] = __float2half_rn(v);
    }
  }
}

}  // namespace

// Packed batches are one batch entry of total_q rows for the row-wise kernels
// (their per-query arrays are [H, total_q], the dQ accumulator [total_q, H, d]).
BwdProblem flat_view(const BwdProblem& p) {
  BwdProblem f = p;
  if (p.f.cu_q != nullptr) {
    f.f.B = 1;
    f.f.Lq = p.f.total_q;
  }
  return f;
}

cudaError_t launch_bwd_prep(const BwdProblem& pin, cudaStream_t stream) {
  const BwdProblem p = flat_view(pin);
  const int64_t rows = static_cast<int64_t>(p.f.B) * p.f.Lq * p.f.H;
  const int block = 256;
  const unsigned grid = static_cast<unsigned>((rows * 32 + block - 1) / block);
  if (p.f.dtype == SMA_BF16) bwd_prep_kernel<SMA_BF16><<<grid, block, 0, stream>>>(p);
  else if (p.f.dtype == SMA_FP16) bwd_prep_kernel<SMA_FP16><<<grid, block, 0, stream>>>(p);
  else bwd_prep_kernel<SMA_FP32><<<grid, block, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_transpose_lists(const BwdProblem& p, uint8_t* codes, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.f.lists.LB) * p.f.lists.LH;
  cudaError_t e = cudaMemsetAsync(codes, 0, static_cast<size_t>(rows * p.f.QT * p.f.KT), stream);
  if (e != cudaSuccess) return e;
  const int64_t n = rows * p.f.QT * p.f.KT;
  scatter_codes_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(p, codes);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  transpose_lists_kernel<<<dim3(p.f.KT, static_cast<unsigned>(rows)), kTrThreads, 0, stream>>>(p, codes);
  return cudaGetLastError();
}

// Fixed-order dbias (see kernels.h): one thread per output element, the
// partial rows summed in increasing (b, h, r) order.
__global__ void dbias_reduce_kernel(const float* __restrict__ part, int B, int H, int R,
                                    float* __restrict__ out, int nb, int nh, int nq, int kd) {
  const int64_t total = static_cast<int64_t>(nb) * nh * nq * kd;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const int k = static_cast<int>(t % kd);
  int64_t rest = t / kd;
  const int qo = static_cast<int>(rest % nq);
  rest /= nq;
  const int ho = static_cast<int>(rest % nh);
  const int bo = static_cast<int>(rest / nh);
  const int b0 = nb == 1 ? 0 : bo, b1 = nb == 1 ? B : bo + 1;
  const int g = H / nh;
  const int h0 = nh == 1 ? 0 : (nh == H ? ho : ho * g);
  const int h1 = nh == 1 ? H : (nh == H ? ho + 1 : ho * g + g);
  const int r0 = nq == 1 ? 0 : qo, r1 = nq == 1 ? R : qo + 1;
  float acc = 0.f;
  for (int b = b0; b < b1; ++b)
    for (int h = h0; h < h1; ++h)
      for (int r = r0; r < r1; ++r)
        acc += part[((static_cast<int64_t>(b) * H + h) * R + r) * kd + k];
  out[t] = acc;
}

cudaError_t launch_dbias_reduce(const float* part, int B, int H, int R, float* out, int nb, int nh,
                                int nq, int kd, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(nb) * nh * nq * kd;
  if (total == 0) return cudaSuccess;
  dbias_reduce_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
      part, B, H, R, out, nb, nh, nq, kd);
  return cudaGetLastError();
}

cudaError_t launch_dq_convert(const BwdProblem& pin, cudaStream_t stream) {
  const BwdProblem p = flat_view(pin);
  const int64_t rows = static_cast<int64_t>(p.f.B) * p.f.Lq * p.f.H;  // one warp each
  const unsigned grid = static_cast<unsigned>((rows * 32 + 255) / 256);
  if (p.f.dtype == SMA_BF16) dq_convert_kernel<SMA_BF16><<<grid, 256, 0, stream>>>(p);
  else if (p.f.dtype == SMA_FP16) dq_convert_kernel<SMA_FP16><<<grid, 256, 0, stream>>>(p);
  else dq_convert_kernel<SMA_FP32><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

int launch_attn_bwd(const BwdProblem& p, cudaStream_t stream, char* msg, size_t msg_len) {
  const AttnProblem& f = p.f;
  if (f.dtype == SMA_FP32) {  // FFMA path (no tensor maps)
    const cudaError_t e = launch_attn_bwd_simt(p, stream);
    if (e != cudaSuccess) {
      snprintf(msg, msg_len, "fp32 attention backward launch failed: %s", cudaGetErrorString(e));
      return SMA_ERR_CUDA;
    }
    return SMA_OK;
  }
  // packed batches: one batch entry of total_q (total_k) rows
  const bool packed = f.cu_q != nullptr;
  const int lq = packed ? f.total_q : f.Lq, lk = packed ? f.total_k : f.Lk, nb = packed ? 1 : f.B;
  CUtensorMap mq, mk, mv, mdo;
  if (!encode_map(&mq, f.q, f.dtype, f.d, f.H, lq, nb, f.q_sh, f.q_sr, f.q_sb, msg, msg_len) ||
      !encode_map(&mk, f.k, f.dtype, f.d, f.KVH, lk, nb, f.k_sh, f.k_sr, f.k_sb, msg, msg_len) ||
      !encode_map(&mv, f.v, f.dtype, f.d, f.KVH, lk, nb, f.v_sh, f.v_sr, f.v_sb, msg, msg_len) ||
      !encode_map(&mdo, p.dout, f.dtype, f.d, f.H, lq, nb, p.do_sh, p.do_sr, p.do_sb, msg, msg_len))
    return SMA_ERR_CUDA;
  CUtensorMap mdq;
  if (!encode_map_f32(&mdq, p.dq_acc, f.d, f.H, lq, nb, 32, 32, msg, msg_len)) return SMA_ERR_CUDA;
  cudaError_t e = cudaErrorInvalidValue;
  const bool bf = f.dtype == SMA_BF16;
  if (f.policy == kPolicyDflash) {
    if (f.d == 128) e = bf ? launch_bwd_t<128, kPolicyDflash, SMA_BF16>(p, mq, mk, mv, mdo, mdq, stream)
                           : launch_bwd_t<128, kPolicyDflash, SMA_FP16>(p, mq, mk, mv, mdo, mdq, stream);
    else e = bf ? launch_bwd_t<64, kPolicyDflash, SMA_BF16>(p, mq, mk, mv, mdo, mdq, stream)
                : launch_bwd_t<64, kPolicyDflash, SMA_FP16>(p, mq, mk, mv, mdo, mdq, stream);
  } else {
    if (f.d == 128) e = bf ? launch_bwd_t<128, kPolicyExplicit, SMA_BF16>(p, mq, mk, mv, mdo, mdq, stream)
                           : launch_bwd_t<128, kPolicyExplicit, SMA_FP16>(p, mq, mk, mv, mdo, mdq, stream);
    else e = bf ? launch_bwd_t<64, kPolicyExplicit, SMA_BF16>(p, mq, mk, mv, mdo, mdq, stream)
                : launch_bwd_t<64, kPolicyExplicit, SMA_FP16>(p, mq, mk, mv, mdo, mdq, stream);
  }
  if (e != cudaSuccess) {
    snprintf(msg, msg_len, "attention backward launch failed: %s", cudaGetErrorString(e));
    return SMA_ERR_CUDA;
  }
  return SMA_OK;
}

}  // namespace sma
