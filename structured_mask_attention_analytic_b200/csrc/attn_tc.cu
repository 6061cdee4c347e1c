// Attention forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent CTA per SM walks "units" (batch, KV head, pair of query
// heads, 128-row query tile).  The two query heads of a unit share the KV
// head, so they share every K/V tile and -- because both mask families here
// are identical across the heads of a group -- the same key-tile list.  Only
// tiles on that list are visited (empty tiles are skipped); the per-element
// mask is evaluated only on tiles flagged PARTIAL.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for query tile 0 (one thread per query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q tiles, K/V tiles into a ring of smem stages
//   warp  9    MMA issuer (one thread): S_i = Q_i K^T into TMEM (SS form),
//              O_i += P_i V with P_i read from TMEM (TS form)
//   warp  10   bias operand tiles when the bias goes through the tensor
//              cores (BTC, see AttnProblem::bias_tc); otherwise idle
//   warp  11   idle
// The kernel is launched with kLaunchRegs registers per thread; the producer
// warpgroup gives registers back (setmaxnreg.dec to kProducerRegs) and the two
// softmax warpgroups take them (setmaxnreg.inc to kSoftmaxRegs).  The shares
// add up to exactly the launch allocation:
//   2 * 128 * kSoftmaxRegs + 128 * kProducerRegs == 384 * kLaunchRegs
// and the host refuses to launch if the compiled register count differs.
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1; P_i (bf16/f16 pairs) overwrites
// the first half of S_i's columns once the softmax has read S_i.
//
// Online softmax in the log2 domain with a lazily rescaled reference max: O
// is rescaled in TMEM only when a row's max grows by more than 2^8.
//
// Mask sources (template policy):
//   DFlash   -- SpecForge issue #452 (Problem paragraph) and PR #905
//               (Motivation list; reply item 1 on the left-only window): a
//               row keeps its context prefix [clo, chi) and its own block's
//               slots [dlo, dhi); evaluated from the anchors.
//   Explicit -- flash-sparse-attention PR #190 (Design: boolean mask, True =
//               keep, additive bias, stride-0 broadcast dims), plus
//               bottom-right causal masking; the bias is added on every kept
//               tile, the mask read on PARTIAL tiles only.
//   Varlen   -- packed sequences: the explicit policy with each unit's rows
//               offset to its sequence and bounded by its lengths
//               (bottom-right causal per sequence); a mask / bias is read in
//               the padded per-sequence layout at sequence-local (q, k).
//   Gather   -- the explicit policy over keys compacted by a query-broadcast
//               mask (PR #197 top-k masks): K/V/bias are the compacted
//               operands and each row's causal bound is a limit on the
//               compacted index.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <type_traits>

#include "device_common.cuh"
#include "gather.cuh"
#include "kernels.h"
#include "tma_map.h"

namespace sma {
namespace {

constexpr int kThreads = 384;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBiasWarp = 10;  // bias operands of the tensor-core bias path
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kProducerRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kProducerRegs == kThreads * kLaunchRegs,
              "register split must equal the launch allocation");
constexpr uint32_t kTmemCols = 512;

// Exponentials of a softmax row run on MUFU ex2.  MUFU (16 per clock per
// SM) takes as long as the row's two products on the tensor cores, so a third
// of them once went to the FMA pipe (a cubic for 2^f and an integer add into
// the exponent field).  Since the units are dealt in snake order that is 1-2 %
// slower in short runs and 1 % slower over 50 steps under the power cap
// (measured), so every exponential is on MUFU.

template <int D, bool BTC = false>
struct Layout {
  // K runs ahead of V; with the bias on the tensor cores at d = 128 the K ring
  // gives up a stage to the bias operand tiles
  static constexpr int kKStages = D == 128 ? (BTC ? 2 : 3) : 4;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr uint32_t kChunkBytes = kTile * 128;  // 64 columns x 128 rows, 128B-swizzled
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + 2 * kTileBytes;
  static constexpr uint32_t kV = kK + kKStages * kTileBytes;
  // bias operand tiles (BTC): A (128 query rows x one K step) and one B
  // (128 keys x one K step) per K stage, 32-byte rows, 32-byte swizzle
  static constexpr uint32_t kXBytes = BTC ? kTile * 32 : 0;
  static constexpr uint32_t kAX = kV + kVStages * kTileBytes;
  static constexpr uint32_t kBX = kAX + kXBytes;
  static constexpr uint32_t kBars = kBX + kKStages * kXBytes;
  // barrier slots
  static constexpr int kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = kKFull + kKStages,
                       kVFull = kKEmpty + kKStages, kVEmpty = kVFull + kVStages,
                       kSBar = kVEmpty + kVStages, kPBar = kSBar + 2, kOBar = kPBar + 2,
                       kOFree = kOBar + 2, kDrain = kOFree + 2, kNumBars = kDrain + 1;
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kBytes = kAbort + 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // base is rounded up to 1024
  // TMEM columns
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct Unit {
  int b, hk, pair, qt, h0, h1valid;
  int q0, q1off, h1off;  // first query of tile 0; tile 1's query and head offsets
  int64_t list_row;
  int n_full, n_part;
  int split, j0, n;          // key-range segment: list entries [j0, j0 + n)
  int q_off, k_off, lq, lk;  // varlen: the sequence's first rows and lengths
};

template <int POLICY>
__device__ __forceinline__ Unit decode_unit(const AttnProblem& p, int u) {
  Unit w;
  // the segments of one unit are adjacent unit indices (adjacent CTAs);
  // packed sequences use neither the key-range split nor head packing
  constexpr bool kSplitPack = POLICY != kPolicyVarlen;
  w.split = kSplitPack ? u % p.n_split : 0;
  if (kSplitPack) u /= p.n_split;
  if (kSplitPack && p.pack > 1) {
    // head-packed tiles: tile i of the unit holds every head of the group
    // for queries [q0 + i * q1off, + 128 / pack); both blocks lie in one
    // 128-query tile, whose key-tile list they share
    const int rows = kTile / p.pack;
    const int qblocks = (p.Lq + rows - 1) / rows;
    const int per = p.B * p.KVH;
    const int pi = (qblocks + 1) / 2 - 1 - u / per;
    const int r = u % per;
    w.hk = r % p.KVH;
    w.b = r / p.KVH;
    w.pair = 0;
    w.h0 = w.hk * p.group;
    w.q0 = 2 * pi * rows;
    w.q1off = rows;
    w.h1off = 0;
    w.h1valid = w.q0 + rows < p.Lq;
    w.qt = w.q0 / kTile;
  } else {
    const int per_qt = p.B * p.KVH * p.npairs;
    w.qt = p.QT - 1 - u / per_qt;  // later query tiles first: they see the most keys
    int r = u % per_qt;
    w.pair = r % p.npairs;
    r /= p.npairs;
    w.hk = r % p.KVH;
    w.b = r / p.KVH;
    w.h0 = w.hk * p.group + 2 * w.pair;
    w.h1valid = (2 * w.pair + 1) < p.group;
    w.q0 = w.qt * kTile;
    w.q1off = 0;
    w.h1off = 1;
  }
  const int lb = p.lists.LB > 1 ? w.b : 0;
  int lh = 0;
  if (p.lists.head_mode == 1) lh = w.hk;
  else if (p.lists.head_mode == 2) lh = w.hk * p.npairs + w.pair;
  w.list_row = (static_cast<int64_t>(lb) * p.lists.LH + lh) * p.QT + w.qt;
  w.n_full = p.lists.num_full[w.list_row];
  w.n_part = p.lists.num_part[w.list_row];
  if (POLICY == kPolicyVarlen) {
    w.q_off = p.cu_q[w.b];
    w.lq = p.cu_q[w.b + 1] - w.q_off;
    w.k_off = p.cu_k[w.b];
    w.lk = p.cu_k[w.b + 1] - w.k_off;
    // malformed offsets (reported by the list kernel): the sequence is empty,
    // so no row of it is read or written
    if (w.lq < 0 || w.lq > p.Lq || w.q_off < 0 || w.q_off + w.lq > p.total_q || w.lk < 0 ||
        w.lk > p.Lk || w.k_off < 0 || w.k_off + w.lk > p.total_k) {
      w.q_off = w.k_off = w.lq = w.lk = 0;
      w.n_full = w.n_part = 0;
    }
  } else {
    w.q_off = 0;
    w.k_off = 0;
    w.lq = p.Lq;
    w.lk = p.Lk;
  }
  const int nt = w.n_full + w.n_part;
  const int ns = kSplitPack ? p.n_split : 1;
  const int seg = (nt + ns - 1) / ns;
  w.j0 = w.split * seg;
  w.n = max(0, min(seg, nt - w.j0));
  return w;
}

// Key tile of the segment's j-th entry (FULL entries precede PARTIAL ones).
__device__ __forceinline__ int tile_at(const AttnProblem& p, const Unit& w, int j, bool* partial) {
  j += w.j0;
  if (j < w.n_full) {
    *partial = false;
    return p.lists.full_idx[w.list_row * p.KT + j];
  }
  *partial = true;
  return p.lists.part_idx[w.list_row * p.KT + (j - w.n_full)];
}

// Waits that ignore the abort flag (used only while draining after an abort).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, int* err) {
  int never = 0;
  volatile int* nv = &never;
  mbar_wait(bar, parity, nv, err);
}

template <int D, int POLICY, int DT, bool BTC>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const AttnProblem p, const __grid_constant__ CUtensorMap map_q,
               const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
               int n_units) {
  using L = Layout<D, BTC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kQFull), 1);
    mbar_init(bar(L::kQEmpty), 1);
    for (int s = 0; s < L::kKStages; ++s) {
      // (with the bias on the tensor cores the bias warp's 32 lanes also
      // arrive, once its operand tile for the stage is written)
      mbar_init(bar(L::kKFull + s), BTC ? 1 + 32 : 1);
      mbar_init(bar(L::kKEmpty + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar(L::kVFull + s), 1);
      mbar_init(bar(L::kVEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kSBar + i), 1);
      mbar_init(bar(L::kPBar + i), 128);
      mbar_init(bar(L::kOBar + i), 1);
      mbar_init(bar(L::kOFree + i), 128);
    }
    mbar_init(bar(L::kDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
   if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; one elected lane issues the copies.
    if (elect_one()) {
      tma_prefetch_map(&map_q);
      tma_prefetch_map(&map_k);
      tma_prefetch_map(&map_v);
    }
    __syncwarp();
    uint32_t kv_k = 0, kv_v = 0, q_it = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0); u < n_units && ok; u = snake_unit(++rnd)) {
      const Unit w = decode_unit<POLICY>(p, u);
      const int n = w.n;
      if (n == 0) continue;
      if (q_it > 0 && !mbar_wait_warp(bar(L::kQEmpty), (q_it - 1) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(L::kQFull), (1 + w.h1valid) * L::kTileBytes);
        for (int i = 0; i < 1 + w.h1valid; ++i)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sbase + L::kQ + i * L::kTileBytes + c * L::kChunkBytes, &map_q,
                        bar(L::kQFull), c * 64, w.h0 + i * w.h1off,
                        w.q_off + w.q0 + i * w.q1off, POLICY == kPolicyVarlen ? 0 : w.b);
      }
      __syncwarp();
      ++q_it;
      bool partial_next = false;
      int kt_next = tile_at(p, w, 0, &partial_next);
      for (int j = 0; j < n && ok; ++j) {
        const int kt = kt_next;
        if (j + 1 < n) kt_next = tile_at(p, w, j + 1, &partial_next);
        const int kstage = kv_k % L::kKStages;
        const uint32_t kuse = kv_k / L::kKStages;
        if (kuse > 0 &&
            !mbar_wait_warp(bar(L::kKEmpty + kstage), (kuse - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::kKFull + kstage), L::kTileBytes);
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sbase + L::kK + kstage * L::kTileBytes + c * L::kChunkBytes, &map_k,
                        bar(L::kKFull + kstage), c * 64, w.hk, w.k_off + kt * kTile,
                        POLICY == kPolicyVarlen ? 0 : w.b);
        }
        __syncwarp();
        ++kv_k;
        const int vstage = kv_v % L::kVStages;
        const uint32_t vuse = kv_v / L::kVStages;
        if (vuse > 0 &&
            !mbar_wait_warp(bar(L::kVEmpty + vstage), (vuse - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(L::kVFull + vstage), L::kTileBytes);
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(sbase + L::kV + vstage * L::kTileBytes + c * L::kChunkBytes, &map_v,
                        bar(L::kVFull + vstage), c * 64, w.hk, w.k_off + kt * kTile,
                        POLICY == kPolicyVarlen ? 0 : w.b);
        }
        __syncwarp();
        ++kv_v;
      }
    }
    if (!ok) {
      // Drain: every copy this warp issued must land before the CTA exits.
      for (uint32_t t = 0; t < static_cast<uint32_t>(L::kKStages); ++t) {
        if (kv_k > t) {
          const uint32_t nn = kv_k - 1 - t;
          drain_wait(bar(L::kKFull + nn % L::kKStages), (nn / L::kKStages) & 1, p.err);
        }
      }
      for (uint32_t t = 0; t < static_cast<uint32_t>(L::kVStages); ++t) {
        if (kv_v > t) {
          const uint32_t nn = kv_v - 1 - t;
          drain_wait(bar(L::kVFull + nn % L::kVStages), (nn / L::kVStages) & 1, p.err);
        }
      }
      if (q_it > 0) drain_wait(bar(L::kQFull), (q_it - 1) & 1, p.err);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and waits; one elected lane issues every
    // tcgen05.mma and tcgen05.commit (commits track that lane's MMAs).
    constexpr uint32_t fmt = DT == SMA_BF16 ? 1u : 0u;
    constexpr uint32_t idesc_qk = mma_idesc_f16(fmt, 128, 128, 0, 0);
    constexpr uint32_t idesc_pv = mma_idesc_f16(fmt, 128, D, 0, 1);
    uint32_t kv_it = 0, q_it = 0;
    uint32_t pv_it0 = 0, pv_it1 = 0, units0 = 0, units1 = 0;
    bool ok = true;
    // Descriptors are built once per operand tile; a k-step only adds to the
    // start-address field (bits 0-13 of the low word, in 16-byte units), so
    // each MMA of the fully unrolled issue sequences costs one 32-bit add.
    auto with_lo = [](uint64_t d, uint32_t add) -> uint64_t {
      return (d & 0xffffffff00000000ull) | static_cast<uint32_t>(static_cast<uint32_t>(d) + add);
    };
    // With the bias on the tensor cores, one more K step adds b[k] / scale.
    auto issue_bias_step = [&](uint32_t d_col, int stage) {
      if (BTC)
        tc_mma_ss(d_col, smem_desc_sw32(sbase + L::kAX),
                  smem_desc_sw32(sbase + L::kBX + stage * L::kXBytes), idesc_qk, 1u);
    };
    auto issue_qk = [&](int i, int stage) {
      const uint64_t qd = smem_desc_sw128(sbase + L::kQ + i * L::kTileBytes, 16, 1024);
      const uint64_t kd = smem_desc_sw128(sbase + L::kK + stage * L::kTileBytes, 16, 1024);
      const uint32_t d_col = tmem + (i == 0 ? L::kColS0 : L::kColS1);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = ((s >> 2) * L::kChunkBytes + (s & 3) * 32) >> 4;
        tc_mma_ss(d_col, with_lo(qd, off), with_lo(kd, off), idesc_qk, s > 0 ? 1u : 0u);
      }
      issue_bias_step(d_col, stage);
    };
    // Both query tiles against one K tile, k-steps interleaved.
    auto issue_qk_pair = [&](int stage) {
      const uint64_t qd0 = smem_desc_sw128(sbase + L::kQ, 16, 1024);
      const uint64_t qd1 = smem_desc_sw128(sbase + L::kQ + L::kTileBytes, 16, 1024);
      const uint64_t kd = smem_desc_sw128(sbase + L::kK + stage * L::kTileBytes, 16, 1024);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = ((s >> 2) * L::kChunkBytes + (s & 3) * 32) >> 4;
        tc_mma_ss(tmem + L::kColS0, with_lo(qd0, off), with_lo(kd, off), idesc_qk, s > 0 ? 1u : 0u);
        tc_mma_ss(tmem + L::kColS1, with_lo(qd1, off), with_lo(kd, off), idesc_qk, s > 0 ? 1u : 0u);
      }
      issue_bias_step(tmem + L::kColS0, stage);
      issue_bias_step(tmem + L::kColS1, stage);
    };
    auto issue_pv = [&](int i, int stage, bool first) {
      const uint64_t vd =
          smem_desc_sw128(sbase + L::kV + stage * L::kTileBytes, L::kChunkBytes, 1024);
      const uint32_t d_col = tmem + (i == 0 ? L::kColO0 : L::kColO1);
      const uint32_t p_col = tmem + (i == 0 ? L::kColS0 : L::kColS1);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s) {
        tc_mma_ts(d_col, p_col + 8 * s, with_lo(vd, (s * 2048) >> 4), idesc_pv,
                  (first && s == 0) ? 0u : 1u);
      }
    };
    for (int rnd = 0, u = snake_unit(0); u < n_units && ok; u = snake_unit(++rnd)) {
      const Unit w = decode_unit<POLICY>(p, u);
      const int n = w.n;
      const int nq = 1 + w.h1valid;
      if (n > 0) {
        if (!mbar_wait_warp(bar(L::kQFull), q_it & 1, abort_flag, p.err)) { ok = false; break; }
        ++q_it;
        // S_i(0) = Q_i K(0)^T.  The previous unit's last PV_i read P_i from
        // S_i's columns; it was issued earlier by this lane, and the MMAs of
        // one issuing thread execute in order.
        {
          const int stage = kv_it % L::kKStages;
          if (!mbar_wait_warp(bar(L::kKFull + stage), (kv_it / L::kKStages) & 1, abort_flag,
                              p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            if (nq == 2) {
              issue_qk_pair(stage);
              tc_commit(bar(L::kSBar + 0));
              tc_commit(bar(L::kSBar + 1));
            } else {
              issue_qk(0, stage);
              tc_commit(bar(L::kSBar + 0));
            }
            tc_commit(bar(L::kKEmpty + stage));
            if (n == 1) tc_commit(bar(L::kQEmpty));
          }
          __syncwarp();
        }
        for (int j = 0; j < n && ok; ++j) {
          const int stage = kv_it % L::kVStages;
          const uint32_t ph = (kv_it / L::kVStages) & 1;
          const int nstage = (kv_it + 1) % L::kKStages;
          const uint32_t nph = ((kv_it + 1) / L::kKStages) & 1;
          if (!mbar_wait_warp(bar(L::kVFull + stage), ph, abort_flag, p.err)) { ok = false; break; }
          for (int i = 0; i < nq && ok; ++i) {
            const uint32_t pvi = i == 0 ? pv_it0 : pv_it1;
            const uint32_t uni = i == 0 ? units0 : units1;
            if (!mbar_wait_warp(bar(L::kPBar + i), pvi & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            if (j == 0 && uni > 0 &&
                !mbar_wait_warp(bar(L::kOFree + i), (uni - 1) & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            if (i == 0 && j + 1 < n &&
                !mbar_wait_warp(bar(L::kKFull + nstage), nph, abort_flag, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (elect_one()) {
              // O_i += P_i(j) V(j)
              issue_pv(i, stage, j == 0);
              tc_commit(bar(L::kOBar + i));
              // S_i(j+1) = Q_i K(j+1)^T right behind it: the MMAs of one
              // issuing thread execute in order, so PV_i(j) has read P_i(j)
              // before QK_i(j+1) rewrites those TMEM columns.
              if (j + 1 < n) {
                issue_qk(i, nstage);
                tc_commit(bar(L::kSBar + i));
              }
            }
            __syncwarp();
            if (i == 0) ++pv_it0; else ++pv_it1;
          }
          if (!ok) break;
          if (elect_one()) {
            tc_commit(bar(L::kVEmpty + stage));
            if (j + 1 < n) {
              tc_commit(bar(L::kKEmpty + nstage));
              if (j + 2 == n) tc_commit(bar(L::kQEmpty));
            }
          }
          __syncwarp();
          ++kv_it;
        }
      }
      units0 += 1;
      units1 += w.h1valid;
    }
    if (!ok) {
      if (elect_one()) tc_commit(bar(L::kDrain));
      __syncwarp();
      drain_wait(bar(L::kDrain), 0, p.err);
    }
   } else if (BTC && warp == kBiasWarp) {
    // ------------------------------------------------------------ bias operands
    // A: every query row [hi, lo, 0, ...] (1 / scale in the operand type); B
    // for each K stage: key row k [b[k], b[k], 0, ...].  Only the first
    // 16-byte half of a row ever holds data; the other half is zeroed once.
    // The bias row is shared by all queries and by both query tiles of a
    // unit (the launcher takes this path only then).  Lane l writes key rows
    // l, l + 32, l + 64, l + 96; the values of the next tile are loaded before
    // waiting for its stage to free up.
    const uint32_t ax = sbase + L::kAX;
    for (int r = lane; r < kTile; r += 32) {
      st_shared_v4(ax + sw32_chunk(r, 0), p.bias_tc_a, 0u, 0u, 0u);
      st_shared_v4(ax + sw32_chunk(r, 1), 0u, 0u, 0u, 0u);
      for (int s2 = 0; s2 < L::kKStages; ++s2)
        st_shared_v4(sbase + L::kBX + s2 * L::kXBytes + sw32_chunk(r, 1), 0u, 0u, 0u, 0u);
    }
    const uint16_t* bias16 = static_cast<const uint16_t*>(p.bias.ptr);
    const int kd = p.bias.kd;
    const uint32_t two_cols = (p.bias_tc_a >> 16) != 0u ? 1u : 0u;  // A has a nonzero lo column
    uint32_t kv_k = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0); u < n_units && ok; u = snake_unit(++rnd)) {
      const Unit w = decode_unit<POLICY>(p, u);
      const int n = w.n;
      if (n == 0) continue;
      const uint16_t* brow = bias16 + w.b * p.bias.sb + w.hk * p.bias.sh;
      bool partial;
      int kt = tile_at(p, w, 0, &partial);
      uint32_t v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = brow[aux_col(kt * kTile + lane + 32 * i, kd)];
      for (int j = 0; j < n && ok; ++j) {
        const int stage = kv_k % L::kKStages;
        const uint32_t kuse = kv_k / L::kKStages;
        if (kuse > 0 &&
            !mbar_wait_warp(bar(L::kKEmpty + stage), (kuse - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        const uint32_t bx = sbase + L::kBX + stage * L::kXBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(bx + sw32_chunk(lane + 32 * i, 0), v[i] | (v[i] << 16) * two_cols, 0u, 0u, 0u);
        fence_async_shared();
        mbar_arrive(bar(L::kKFull + stage));
        ++kv_k;
        if (j + 1 < n) {
          kt = tile_at(p, w, j + 1, &partial);
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = brow[aux_col(kt * kTile + lane + 32 * i, kd)];
        }
      }
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------------------------------------------------------ softmax
    const int qi = warp >> 2;        // which query tile of the unit
    const int quad = warp & 3;       // TMEM lane quadrant
    const int r = quad * 32 + lane;  // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = tmem + lane_off + (qi == 0 ? L::kColS0 : L::kColS1);
    const uint32_t o_col = tmem + lane_off + (qi == 0 ? L::kColO0 : L::kColO1);
    uint32_t it = 0;
    bool ok = true;
    for (int rnd = 0, u = snake_unit(0); u < n_units && ok; u = snake_unit(++rnd)) {
      const Unit w = decode_unit<POLICY>(p, u);
      if (qi == 1 && !w.h1valid) continue;
      const int qfirst = w.q0 + qi * w.q1off;  // first query of this tile
      int h, q;
      if (POLICY != kPolicyVarlen && p.pack > 1) {  // row r: head r % pack of query r / pack
        h = w.h0 + (r & (p.pack - 1));
        q = qfirst + (r >> (__ffs(p.pack) - 1));
      } else {
        h = w.h0 + qi;
        q = qfirst + r;
      }
      const bool row_valid = q < w.lq;
      const int n = w.n;

      // Per-row mask parameters.
      int clo = 0, chi = 0, dlo = 0, dhi = 0;  // DFlash keep intervals
      const uint8_t* mrow = nullptr;
      const uint8_t* brow = nullptr;
      int causal_lim = 0x7fffffff;
      if (POLICY == kPolicyDflash) {
        if (row_valid) {
          const int j = q / p.bs, i = q - j * p.bs;
          int a = p.anchors[static_cast<int64_t>(w.b) * p.N + j];
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
          const int hm = p.mask.head_per_query ? h : w.hk;
          mrow = reinterpret_cast<const uint8_t*>(p.mask.ptr) + w.b * p.mask.sb + hm * p.mask.sh +
                 static_cast<int64_t>(qq) * p.mask.sq;
        }
        if (p.has_bias) {
          const int hb = p.bias.head_per_query ? h : w.hk;
          const int esz = p.bias.dtype == SMA_FP32 ? 4 : 2;
          brow = reinterpret_cast<const uint8_t*>(p.bias.ptr) +
                 (w.b * p.bias.sb + hb * p.bias.sh + static_cast<int64_t>(qq) * p.bias.sq) * esz;
        }
        if (POLICY == kPolicyGather)  // compacted keys: the row's limit on the compacted index
          causal_lim = row_valid ? gather_row_limit(p, w.list_row / p.QT, q) - 1 : -1;
        else if (p.causal)
          causal_lim = q + w.lk - w.lq;
      }

      // Scores are scaled inside the exponent (one FFMA per element).  A bias
      // is added as b / scale beforehand, so that scale * (s + b / scale) *
      // log2(e) = (scale * s + b) * log2(e).
      const float exp_scale = p.scale_log2;
      const float bias_mul = kLog2e / p.scale_log2;
      // With compacted keys every PARTIAL tile is cut by the row limit.
      const int causal_off = POLICY == kPolicyGather ? -(1 << 30) : w.lk - w.lq;
      // explicit masks: the padded policy, and packed sequences (their mask in
      // the padded per-sequence layout, rows and columns sequence-local)
      constexpr bool kMasks = POLICY == kPolicyExplicit || POLICY == kPolicyVarlen;
      const bool mask_bcast_q = kMasks && p.has_mask && p.mask.sq == 0;
      // Mask / bias rows hold kd columns: round_up(Lk, 128), Lk, or 1.  Vector
      // loads start at most at the row's last aligned chunk (a 16-byte block
      // that holds column kd - 1), so none leaves the row's memory; columns
      // past Lk are never kept whatever is read for them.  A row of one column
      // holds one value for every key: a mask flag for the whole row, or a
      // bias that shifts every score of the row alike, which the softmax
      // ignores; it is added once, to the row's max (and so to lse).
      const bool bias_cols = !BTC && p.has_bias && p.bias.kd > 1;
      const int bias_vlast = (p.bias.kd - 1) & (p.bias.dtype == SMA_FP32 ? ~3 : ~7);
      const bool mask_row1 = p.has_mask && p.mask.kd == 1;
      const int mask_vlast16 = (p.mask.kd - 1) & ~15;
      const int mask_vlast4 = (p.mask.kd - 1) & ~3;
      const bool row_keep1 = mask_row1 && mrow[0] != 0;
      const float bias_row_log2 =
          (POLICY != kPolicyDflash && !BTC && p.has_bias && p.bias.kd == 1)
              ? load_any_as_float(brow, p.bias.dtype, 0) * kLog2e : 0.f;
      float m_ref = -INFINITY, l_sum = 0.f;
      bool partial_next = false;
      int kt_next = n > 0 ? tile_at(p, w, 0, &partial_next) : 0;
      for (int j = 0; j < n && ok; ++j) {
        const int kt = kt_next;
        const bool partial = partial_next;
        if (j + 1 < n) kt_next = tile_at(p, w, j + 1, &partial_next);  // prefetch
        const int k0 = kt * kTile;
        if (!mbar_wait(bar(L::kSBar + qi), it & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        float x[kTile];
        {
          uint32_t* xr = reinterpret_cast<uint32_t*>(x);
#pragma unroll
          for (int c = 0; c < kTile / 32; ++c) tmem_ld32_at(s_col + 32 * c, xr + 32 * c);
          tc_wait_ld();
        }
        if (POLICY != kPolicyDflash && bias_cols) {
          if (p.bias.dtype == SMA_FP32) {
#pragma unroll
            for (int c = 0; c < kTile; c += 4) {
              const float4 a = *reinterpret_cast<const float4*>(brow + min(k0 + c, bias_vlast) * 4);
              x[c] = fmaf(a.x, bias_mul, x[c]);
              x[c + 1] = fmaf(a.y, bias_mul, x[c + 1]);
              x[c + 2] = fmaf(a.z, bias_mul, x[c + 2]);
              x[c + 3] = fmaf(a.w, bias_mul, x[c + 3]);
            }
          } else if (p.bias.dtype == SMA_BF16) {
#pragma unroll
            for (int c = 0; c < kTile; c += 8) {
              const uint4 a = *reinterpret_cast<const uint4*>(brow + min(k0 + c, bias_vlast) * 2);
              const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                x[c + 2 * e] = fmaf(__uint_as_float(wv[e] << 16), bias_mul, x[c + 2 * e]);
                x[c + 2 * e + 1] =
                    fmaf(__uint_as_float(wv[e] & 0xffff0000u), bias_mul, x[c + 2 * e + 1]);
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < kTile; c += 8) {
              const uint4 a = *reinterpret_cast<const uint4*>(brow + min(k0 + c, bias_vlast) * 2);
              const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
                x[c + 2 * e] = fmaf(f.x, bias_mul, x[c + 2 * e]);
                x[c + 2 * e + 1] = fmaf(f.y, bias_mul, x[c + 2 * e + 1]);
              }
            }
          }
        }
        if (partial) {  // warp-uniform
          if (POLICY == kPolicyDflash) {
            const uint32_t wc = static_cast<uint32_t>(chi - clo);
            const uint32_t wd = static_cast<uint32_t>(dhi - dlo);
            const int ac = k0 - clo, ad = k0 - dlo;
#pragma unroll
            for (int c = 0; c < kTile; ++c) {
              const bool keep = static_cast<uint32_t>(c + ac) < wc ||
                                static_cast<uint32_t>(c + ad) < wd;
              x[c] = keep ? x[c] : -INFINITY;
            }
          } else {
            // Columns c >= lim fail the key-length or causal bound; both bounds
            // are checked only on tiles they can cut (uniform per tile).
            int lim = kTile;
            if (k0 + kTile > w.lk) lim = min(lim, w.lk - k0);
            if (p.causal && k0 + kTile - 1 > qfirst + causal_off)
              lim = min(lim, causal_lim - k0 + 1);
            if (kMasks && mask_row1) {
#pragma unroll
              for (int c = 0; c < kTile; ++c) x[c] = (row_keep1 && c < lim) ? x[c] : -INFINITY;
            } else if (mask_bcast_q) {
              // One mask row for every query row: 4 ballots turn the tile's 128
              // bytes into bits, bit l of word j = column 4 l + j.
              const uint32_t mw = *reinterpret_cast<const uint32_t*>(mrow + min(k0 + 4 * lane, mask_vlast4));
              uint32_t bits[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                bits[j] = __ballot_sync(0xffffffffu, ((mw >> (8 * j)) & 0xffu) != 0u);
#pragma unroll
              for (int c = 0; c < kTile; ++c) {
                const bool keep = ((bits[c & 3] >> (c >> 2)) & 1u) != 0u && c < lim;
                x[c] = keep ? x[c] : -INFINITY;
              }
            } else if (kMasks && p.has_mask) {
#pragma unroll
              for (int c = 0; c < kTile; c += 16) {
                const uint4 mv = *reinterpret_cast<const uint4*>(mrow + min(k0 + c, mask_vlast16));
                const uint32_t wv[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const bool keep = ((wv[e >> 2] >> (8 * (e & 3))) & 0xffu) != 0u && (c + e) < lim;
                  x[c + e] = keep ? x[c + e] : -INFINITY;
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < kTile; ++c) x[c] = c < lim ? x[c] : -INFINITY;
            }
          }
        }
        if (!row_valid) {
#pragma unroll
          for (int c = 0; c < kTile; ++c) x[c] = -INFINITY;
        }
        // Row max: eight independent chains, then a tree.
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = x[e];
#pragma unroll
        for (int c = 8; c < kTile; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
#pragma unroll
        for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int e = 0; e < w2; ++e) mx8[e] = fmaxf(mx8[e], mx8[e + w2]);
        const float m_new = fmaxf(m_ref, mx8[0] * exp_scale);
        // Lazy rescale of O: only when the max grew by more than 2^8.
        const bool need = (m_ref != -INFINITY) && (m_new > m_ref + 8.0f);
        if (__any_sync(0xffffffffu, need)) {
          if (!mbar_wait(bar(L::kOBar + qi), (it - 1) & 1, abort_flag, p.err)) { ok = false; }
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_col + 32 * c, o);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(o_col + 32 * c, o);
          }
          tc_wait_st();
          if (need) {
            l_sum *= alpha;
            m_ref = m_new;
          }
        }
        if (m_ref == -INFINITY) m_ref = m_new;
        const float msub = m_ref == -INFINITY ? 0.f : m_ref;
        float2 ls4[4];  // this tile's row sum, four chains of pairs
#pragma unroll
        for (int e = 0; e < 4; ++e) ls4[e] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 t = fma2(make_float2(x[32 * c + 2 * e], x[32 * c + 2 * e + 1]),
                                  make_float2(exp_scale, exp_scale), make_float2(-msub, -msub));
            float2 pp;
            pp.x = fast_exp2(t.x);
            pp.y = fast_exp2(t.y);
            ls4[e & 3] = add2(ls4[e & 3], pp);
            pk[e] = DT == SMA_BF16 ? pack_bf16x2(pp.x, pp.y) : pack_f16x2(pp.x, pp.y);
          }
          // P columns [16c, 16c+16) of the packed pairs
          asm volatile(
              "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
              "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(
                  s_col + 16 * c),
              "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]),
              "r"(pk[6]), "r"(pk[7]), "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]),
              "r"(pk[12]), "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
              : "memory");
        }
        {
          const float2 a2 = add2(add2(ls4[0], ls4[1]), add2(ls4[2], ls4[3]));
          l_sum += a2.x + a2.y;
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::kPBar + qi));
        ++it;
      }
      if (!ok) break;

      // Epilogue: O / l, lse.
      typedef typename std::conditional<DT == SMA_BF16, __nv_bfloat16, __half>::type OutT;
      OutT* orow = reinterpret_cast<OutT*>(p.o) + (POLICY == kPolicyVarlen ? 0 : w.b) * p.o_sb +
                   static_cast<int64_t>(w.q_off + q) * p.o_sr +
                   h * p.o_sh;
      // A row that kept no key has max -inf (and sum 0).
      const bool live = m_ref != -INFINITY;
      const float inv_l = live ? 1.0f / l_sum : 0.f;
      // Key-range segment: unnormalised O and (max, sum) go to the partials.
      const bool seg_out = POLICY != kPolicyVarlen && p.n_split > 1;
      const int64_t prow =
          (static_cast<int64_t>(w.split) * p.part_rows + (static_cast<int64_t>(w.b) * p.H + h) * p.Lq +
           q);
      if (n > 0) {
        if (!mbar_wait(bar(L::kOBar + qi), (it - 1) & 1, abort_flag, p.err)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_col + 32 * c, o);
          tc_wait_ld();
          if (seg_out) {
            if (row_valid) {
              uint4* dst = reinterpret_cast<uint4*>(p.part_o + prow * D + 32 * c);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
            }
          } else if (row_valid) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float a = __uint_as_float(o[2 * e]) * inv_l;
              const float bq = __uint_as_float(o[2 * e + 1]) * inv_l;
              pk[e] = DT == SMA_BF16 ? pack_bf16x2(a, bq) : pack_f16x2(a, bq);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      } else if (row_valid && !seg_out) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
        for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0, 0, 0, 0);
      }
      if (seg_out) {
        if (row_valid)
          *reinterpret_cast<float2*>(p.part_ml + 2 * prow) =
              make_float2(live ? m_ref + bias_row_log2 : -INFINITY, live ? l_sum : 0.f);
      } else if (row_valid && p.lse != nullptr) {
        p.lse[POLICY == kPolicyVarlen ? static_cast<int64_t>(h) * p.total_q + w.q_off + q
                                      : (static_cast<int64_t>(w.b) * p.H + h) * p.Lq + q] =
            live ? (m_ref + bias_row_log2 + __log2f(l_sum)) * kLn2 : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(bar(L::kOFree + qi));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Merge of the key-range segments.  Segment s holds, per row, O_s = sum of
// 2^(t - m_s) V over its keys (t = log2-domain score) and l_s = sum of
// 2^(t - m_s); with M = max m_s over the segments that kept a key,
//   O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,
//   lse = ln 2 * (M + log2 sum_s 2^(m_s - M) l_s).
// One warp per row: lane s reads segment s's (m_s, l_s) (at most 32
// segments) while every lane loads its D / 32 columns of all segments' O_s;
// the warp reduces M and the sum, then each lane accumulates its columns.  A
// segment that kept no key of the row (l_s = 0) may not have written O_s:
// its loaded values are discarded (weight 0, selected out).
template <int D, int DT>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnProblem p) {
  typedef typename std::conditional<DT == SMA_BF16, __nv_bfloat16, __half>::type OutT;
  constexpr int kPer = D / 32;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.part_rows) return;
  const int ns = p.n_split;
  const float2 v = lane < ns
                       ? reinterpret_cast<const float2*>(p.part_ml)[static_cast<int64_t>(lane) * p.part_rows + row]
                       : make_float2(-INFINITY, 0.f);
  // Every segment's O columns are loaded at once, before the weights are
  // known (one memory round trip for the whole row); a segment that kept no
  // key may not have written them, so its values are dropped by a select,
  // never multiplied.
  const float* src = p.part_o + row * D + lane * kPer;
  const int64_t seg_stride = p.part_rows * D;
  float vals[32][kPer];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
#pragma unroll
    for (int e = 0; e < kPer; ++e) vals[i][e] = 0.f;
    if (i < ns) {
      const float* sp = src + i * seg_stride;
      if (kPer == 4) {
        const float4 a = *reinterpret_cast<const float4*>(sp);
        vals[i][0] = a.x; vals[i][1] = a.y; vals[i][2] = a.z; vals[i][3] = a.w;
      } else {
        const float2 a = *reinterpret_cast<const float2*>(sp);
        vals[i][0] = a.x; vals[i][1] = a.y;
      }
    }
  }
  const bool live = v.y > 0.f;
  float mx = live ? v.x : -INFINITY;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float wgt = live ? fast_exp2(v.x - mx) : 0.f;
  float l = wgt * v.y;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float w_i = __shfl_sync(0xffffffffu, wgt, i);  // 0 for segments without keys
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w_i, w_i != 0.f ? vals[i][e] : 0.f, acc[e]);
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const int q = static_cast<int>(row % p.Lq);
  const int64_t bh = row / p.Lq;
  const int h = static_cast<int>(bh % p.H);
  const int b = static_cast<int>(bh / p.H);
  OutT* orow = reinterpret_cast<OutT*>(p.o) + b * p.o_sb + static_cast<int64_t>(q) * p.o_sr +
               h * p.o_sh + lane * kPer;
  uint32_t pk[kPer / 2];
#pragma unroll
  for (int e = 0; e < kPer / 2; ++e)
    pk[e] = DT == SMA_BF16 ? pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv)
                           : pack_f16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  if (kPer == 4) *reinterpret_cast<uint2*>(orow) = make_uint2(pk[0], pk[1]);
  else *reinterpret_cast<uint32_t*>(orow) = pk[0];
  if (lane == 0 && p.lse != nullptr)
    p.lse[row] = l > 0.f ? (mx + __log2f(l)) * kLn2 : -INFINITY;
}

// ------------------------------------------------------------------ host side

// bf16 bits of x rounded to nearest even (finite x), and back.
uint16_t float_to_bf16_bits(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}
float bf16_bits_to_float(uint16_t h) {
  const uint32_t u = static_cast<uint32_t>(h) << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

template <int D, int POLICY, int DT, bool BTC = false>
cudaError_t launch_typed(const AttnProblem& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, cudaStream_t stream) {
  using L = Layout<D, BTC>;
  static_assert(L::kAlloc <= 232448, "shared memory of one CTA");
  auto kern = attn_tc_kernel<D, POLICY, DT, BTC>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    // The setmaxnreg split assumes exactly kLaunchRegs registers per thread.
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L::kAlloc));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int n_units =
      static_cast<int>(fwd_units(p.B, p.KVH, p.npairs, p.QT, p.Lq, p.pack)) * p.n_split;
  if (n_units == 0) return cudaSuccess;
  const int grid = n_units < num_sms() ? n_units : num_sms();
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p, mq, mk, mv, n_units);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.n_split == 1) return e;
  const int64_t blocks = (p.part_rows + 7) / 8;
  attn_combine_kernel<D, DT><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// Tensor maps and the typed launch of one problem (pack already set).
int launch_problem(const AttnProblem& p, cudaStream_t stream, char* msg, size_t msg_len) {
  CUtensorMap mq, mk, mv;
  // packed sequences: one batch entry of total_q (total_k) rows
  const bool packed = p.policy == kPolicyVarlen;
  const int lq = packed ? p.total_q : p.Lq, lk = packed ? p.total_k : p.Lk, nb = packed ? 1 : p.B;
  if (!encode_map(&mq, p.q, p.dtype, p.d, p.H, lq, nb, p.q_sh, p.q_sr, p.q_sb, msg, msg_len,
                  p.pack) ||
      !encode_map(&mk, p.k, p.dtype, p.d, p.KVH, lk, nb, p.k_sh, p.k_sr, p.k_sb, msg, msg_len) ||
      !encode_map(&mv, p.v, p.dtype, p.d, p.KVH, lk, nb, p.v_sh, p.v_sr, p.v_sb, msg, msg_len))
    return SMA_ERR_CUDA;
  cudaError_t e = cudaErrorInvalidValue;
  const bool bf = p.dtype == SMA_BF16;
  if (p.policy == kPolicyDflash) {
    if (p.d == 128) e = bf ? launch_typed<128, kPolicyDflash, SMA_BF16>(p, mq, mk, mv, stream)
                           : launch_typed<128, kPolicyDflash, SMA_FP16>(p, mq, mk, mv, stream);
    else e = bf ? launch_typed<64, kPolicyDflash, SMA_BF16>(p, mq, mk, mv, stream)
                : launch_typed<64, kPolicyDflash, SMA_FP16>(p, mq, mk, mv, stream);
  } else if (p.policy == kPolicyGather) {
    if (p.d == 128) e = bf ? launch_typed<128, kPolicyGather, SMA_BF16>(p, mq, mk, mv, stream)
                           : launch_typed<128, kPolicyGather, SMA_FP16>(p, mq, mk, mv, stream);
    else e = bf ? launch_typed<64, kPolicyGather, SMA_BF16>(p, mq, mk, mv, stream)
                : launch_typed<64, kPolicyGather, SMA_FP16>(p, mq, mk, mv, stream);
  } else if (p.policy == kPolicyVarlen) {
    if (p.d == 128) e = bf ? launch_typed<128, kPolicyVarlen, SMA_BF16>(p, mq, mk, mv, stream)
                           : launch_typed<128, kPolicyVarlen, SMA_FP16>(p, mq, mk, mv, stream);
    else e = bf ? launch_typed<64, kPolicyVarlen, SMA_BF16>(p, mq, mk, mv, stream)
                : launch_typed<64, kPolicyVarlen, SMA_FP16>(p, mq, mk, mv, stream);
  } else if (p.bias_tc) {
    if (p.d == 128)
      e = bf ? launch_typed<128, kPolicyExplicit, SMA_BF16, true>(p, mq, mk, mv, stream)
             : launch_typed<128, kPolicyExplicit, SMA_FP16, true>(p, mq, mk, mv, stream);
    else e = bf ? launch_typed<64, kPolicyExplicit, SMA_BF16, true>(p, mq, mk, mv, stream)
                : launch_typed<64, kPolicyExplicit, SMA_FP16, true>(p, mq, mk, mv, stream);
  } else {
    if (p.d == 128) e = bf ? launch_typed<128, kPolicyExplicit, SMA_BF16>(p, mq, mk, mv, stream)
                           : launch_typed<128, kPolicyExplicit, SMA_FP16>(p, mq, mk, mv, stream);
    else e = bf ? launch_typed<64, kPolicyExplicit, SMA_BF16>(p, mq, mk, mv, stream)
                : launch_typed<64, kPolicyExplicit, SMA_FP16>(p, mq, mk, mv, stream);
  }
  if (e != cudaSuccess) {
    snprintf(msg, msg_len, "attention launch failed: %s", cudaGetErrorString(e));
    return SMA_ERR_CUDA;
  }
  return SMA_OK;
}

}  // namespace

int launch_attn_tc(const AttnProblem& p, cudaStream_t stream, char* msg, size_t msg_len) {
  // the combine kernel reads one segment per lane: at most 32 segments
  if (p.n_split < 1 || p.n_split > 32 ||
      (p.n_split > 1 && (p.policy == kPolicyVarlen || p.part_o == nullptr || p.part_ml == nullptr ||
                         p.part_rows != static_cast<int64_t>(p.B) * p.H * p.Lq))) {
    snprintf(msg, msg_len, "invalid key-range split");
    return SMA_ERR_INVALID_ARG;
  }
  AttnProblem pp = p;
  pp.pack = fwd_pack(p.Lq, p.group, p.lists.head_mode, p.policy);
  // The bias goes through the tensor cores when one bias row serves every
  // query and both query heads of a unit: query stride 0, head dim 1 or KVH
  // (or one head per KV head, or a head dim read with stride 0), more than
  // one key column, the operands' dtype.
  pp.bias_tc = 0;
  if (pp.policy == kPolicyExplicit && pp.has_bias && pp.bias.kd > 1 && pp.bias.sq == 0 &&
      pp.bias.dtype == pp.dtype &&
      (pp.bias.head_per_query == 0 || pp.group == 1 || pp.bias.sh == 0)) {
    pp.bias_tc = 1;
    // hi is 1 / scale rounded toward zero, so that lo = 1 / scale - hi >= 0:
    // a bias of -inf then gives -inf * hi + -inf * lo = -inf, never
    // -inf + inf.  When lo is 0 (1 / scale exact, e.g. 8 at head dim 64) the
    // operand has one column only, so that -inf never meets a zero factor.
    const float inv_scale = 1.4426950408889634f / pp.scale_log2;  // as the kernel's bias_mul
    uint16_t hi, lo;
    if (pp.dtype == SMA_BF16) {
      uint32_t u;
      memcpy(&u, &inv_scale, 4);
      hi = static_cast<uint16_t>(u >> 16);
      lo = float_to_bf16_bits(inv_scale - bf16_bits_to_float(hi));
    } else {
      hi = __half_as_ushort(__float2half_rz(inv_scale));
      lo = __half_as_ushort(__float2half_rn(inv_scale - __half2float(__ushort_as_half(hi))));
    }
    pp.bias_tc_a = static_cast<uint32_t>(hi) | (static_cast<uint32_t>(lo) << 16);
  }
  return launch_problem(pp, stream, msg, msg_len);
}

}  // namespace sma
