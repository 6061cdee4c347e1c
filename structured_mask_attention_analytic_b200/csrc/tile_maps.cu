// Tile classification kernels.
//
// * dfa_block_map_kernel -- full / partial / empty key-tile lists of the
//   DFlash draft-training mask, derived analytically from the anchors: each
//   query row keeps the union of two key intervals (its context prefix and
//   its own block's visible slots), so a 128x128 tile is classified by
//   interval arithmetic over its 128 rows.  The dense [B, H, Q, K] mask whose
//   materialisation runs out of memory in SpecForge issue #452 ("Tried to
//   allocate 256.00 GiB") is never formed, and there is no head dim (same
//   page, Expected Behavior: a head-independent mask with H=1).
// * mask_summary_kernel -- the same codes for an explicit boolean mask at its
//   own broadcast shape (flash-sparse-attention PR #190 contract), one
//   streaming pass over the mask.
// * explicit_lists_kernel -- lists for masked_attn_fwd from those codes plus
//   causal and key-length geometry (per sequence for packed batches with a
//   mask or bias).
#include "device_common.cuh"
#include "kernels.h"

namespace sma {

namespace {

constexpr int kMapThreads = 128;

// Block-wide exclusive scan of two 0/1 flags (128 threads = 4 warps).
struct FlagScan {
  int full_off, part_off, full_total, part_total;
};

__device__ __forceinline__ FlagScan scan_flags(int f, int p, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int fi = f, pi = p;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int a = __shfl_up_sync(0xffffffffu, fi, o);
    int c = __shfl_up_sync(0xffffffffu, pi, o);
    if (lane >= o) { fi += a; pi += c; }
  }
  if (lane == 31) { warp_sums[warp] = fi; warp_sums[4 + warp] = pi; }
  __syncthreads();
  int fo = 0, po = 0, ft = 0, pt = 0;
#pragma unroll
  for (int w = 0; w < kMapThreads / 32; ++w) {
    if (w < warp) { fo += warp_sums[w]; po += warp_sums[4 + w]; }
    ft += warp_sums[w];
    pt += warp_sums[4 + w];
  }
  __syncthreads();
  return {fo + fi - f, po + pi - p, ft, pt};
}

// Walks key tiles in chunks of 128, classifying with `code_of(kt)` and
// appending FULL / PARTIAL indices in ascending order; pads with -1.
template <class CodeFn>
__device__ void emit_lists(int KT, CodeFn code_of, int32_t* nf_out, int32_t* fi_row,
                           int32_t* np_out, int32_t* pi_row) {
  __shared__ int warp_sums[8];
  int nf = 0, np = 0;
  for (int base = 0; base < KT; base += kMapThreads) {
    const int kt = base + threadIdx.x;
    int code = kt < KT ? code_of(kt) : SMA_TILE_EMPTY;
    const int f = code == SMA_TILE_FULL, p = code == SMA_TILE_PARTIAL;
    FlagScan s = scan_flags(f, p, warp_sums);
    if (f) fi_row[nf + s.full_off] = kt;
    if (p) pi_row[np + s.part_off] = kt;
    nf += s.full_total;
    np += s.part_total;
  }
  for (int i = nf + threadIdx.x; i < KT; i += kMapThreads) fi_row[i] = -1;
  for (int i = np + threadIdx.x; i < KT; i += kMapThreads) pi_row[i] = -1;
  if (threadIdx.x == 0) { *nf_out = nf; *np_out = np; }
}

__device__ __forceinline__ int overlap(int lo, int hi, int a, int b) {
  const int l = lo > a ? lo : a;
  const int h = hi < b ? hi : b;
  return h > l ? h - l : 0;
}

__global__ void __launch_bounds__(kMapThreads)
dfa_block_map_kernel(DflashGeom g, const int32_t* __restrict__ anchors, int32_t* num_full,
                     int32_t* full_idx, int32_t* num_part, int32_t* part_idx, int* err) {
  const int qt = blockIdx.x, b = blockIdx.y;
  __shared__ int s_clo[kTile], s_chi[kTile], s_dlo[kTile], s_dhi[kTile];
  __shared__ int s_nvalid;

  // Row intervals: context [clo, chi) and own block [dlo, dhi).
  {
    const int r = threadIdx.x;
    const int q = qt * kTile + r;
    int clo = 0, chi = 0, dlo = 0, dhi = 0;
    if (q < g.Nq) {
      const int j = q / g.bs, i = q - j * g.bs;
      int a = anchors[static_cast<int64_t>(b) * g.N + j];
      if (a < 0 || a > g.Lc) {
        report_error(err, SMA_ERR_DEVICE_INPUT);
        a = a < 0 ? 0 : g.Lc;
      }
      chi = a;
      clo = g.window > 0 ? max(0, a + i - g.window + 1) : 0;
      if (clo > chi) clo = chi;
      const int base = g.Lc + j * g.bs;
      const int tlo = g.window > 0 ? max(0, i - g.window + 1) : 0;
      const int thi = g.causal ? i + 1 : g.bs;
      dlo = base + tlo;
      dhi = base + thi;
    }
    s_clo[r] = clo; s_chi[r] = chi; s_dlo[r] = dlo; s_dhi[r] = dhi;
    if (r == 0) s_nvalid = min(kTile, g.Nq - qt * kTile);
  }
  __syncthreads();
  const int nvalid = s_nvalid;

  auto code_of = [&](int kt) -> int {
    const int k0 = kt * kTile;
    const int k1 = min(k0 + kTile, g.Lk);
    const int width = k1 - k0;
    bool all_full = (k0 + kTile) <= g.Lk;
    bool any = false;
    for (int r = 0; r < nvalid; ++r) {
      const int c = overlap(s_clo[r], s_chi[r], k0, k1) + overlap(s_dlo[r], s_dhi[r], k0, k1);
      any |= c > 0;
      all_full &= c == width;
    }
    return !any ? SMA_TILE_EMPTY : (all_full ? SMA_TILE_FULL : SMA_TILE_PARTIAL);
  };
  const int64_t row = static_cast<int64_t>(b) * g.QT + qt;
  emit_lists(g.KT, code_of, num_full + row, full_idx + row * g.KT, num_part + row,
             part_idx + row * g.KT);
}

// One warp per (m0, m1, q-tile, k-tile) of the mask; rows of 128 bytes read as
// eight 16-byte vectors, four rows per warp instruction.
constexpr int kSummaryWarps = 8;

__global__ void __launch_bounds__(kSummaryWarps * 32)
mask_summary_kernel(const uint8_t* __restrict__ mask, int64_t m0, int64_t m1, int64_t m2,
                    int64_t s0, int64_t s1, int64_t s2, int kd, int Lk, int QT, int KT,
                    uint8_t* __restrict__ codes) {
  const int lane = threadIdx.x & 31;
  const int64_t tile = static_cast<int64_t>(blockIdx.x) * kSummaryWarps + (threadIdx.x >> 5);
  const int64_t n_tiles = m0 * m1 * QT * KT;
  if (tile >= n_tiles) return;
  const int kt = static_cast<int>(tile % KT);
  int64_t rest = tile / KT;
  const int qt = static_cast<int>(rest % QT);
  rest /= QT;
  const int64_t i1 = rest % m1, i0 = rest / m1;

  const int vec = lane & 7;             // which 16-byte column chunk of the row
  const int k0 = kt * kTile + vec * 16; // first column of that chunk
  // columns of this chunk that are < Lk, as a byte mask over the 16 bytes
  const int nvalid_cols = max(0, min(16, Lk - k0));
  const int64_t rows_left = m2 - static_cast<int64_t>(qt) * kTile;
  const int rows = static_cast<int>(rows_left < kTile ? rows_left : kTile);
  const uint8_t* base = mask + i0 * s0 + i1 * s1 + (static_cast<int64_t>(qt) * kTile) * s2;
  // rows of kd columns (round_up(Lk, 128), Lk, or 1 for every key): whole
  // 16-byte chunks as vectors, the rest column by column inside the row
  const bool whole = k0 + 16 <= kd;
  bool all_true = nvalid_cols == 16;
  bool any_true = false;
#pragma unroll 4
  for (int r = lane >> 3; r < rows; r += 4) {
    const uint8_t* mrow = base + r * s2;
    uint32_t w[4];
    if (whole) {
      const uint4 v = *reinterpret_cast<const uint4*>(mrow + k0);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[e] = 0u;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[e] |= static_cast<uint32_t>(mrow[aux_col(k0 + 4 * e + t, kd)]) << (8 * t);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // per-byte nonzero -> 0xff
      const uint32_t nz = __vcmpne4(w[e], 0u);
      const int first = e * 4;
      uint32_t valid = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (first + t < nvalid_cols) valid |= 0xffu << (8 * t);
      all_true &= (nz & valid) == valid;
      any_true |= (nz & valid) != 0u;
    }
  }
  all_true = __all_sync(0xffffffffu, all_true);
  any_true = __any_sync(0xffffffffu, any_true);
  if (lane == 0) {
    const bool in_range = (kt + 1) * kTile <= Lk;
    codes[tile] = !any_true ? SMA_TILE_EMPTY
                            : ((all_true && in_range) ? SMA_TILE_FULL : SMA_TILE_PARTIAL);
  }
}

__device__ __forceinline__ int combine_codes(int a, int b) {
  if (a == SMA_TILE_EMPTY || b == SMA_TILE_EMPTY) return SMA_TILE_EMPTY;
  if (a == SMA_TILE_FULL && b == SMA_TILE_FULL) return SMA_TILE_FULL;
  return SMA_TILE_PARTIAL;
}

// Union of two heads' codes for a tile both are computed on.
__device__ __forceinline__ int union_codes(int a, int b) {
  if (a == b) return a;
  return SMA_TILE_PARTIAL;
}

__global__ void __launch_bounds__(kMapThreads)
explicit_lists_kernel(AttnProblem p, const uint8_t* __restrict__ codes, int codes_qt,
                      int32_t* num_full, int32_t* full_idx, int32_t* num_part, int32_t* part_idx) {
  const int qt = blockIdx.x, lh = blockIdx.y, lb = blockIdx.z;
  // query / key lengths: the problem's, or for packed sequences (cu_q set;
  // list batch row lb is sequence lb) the sequence's, whose malformed
  // offsets are reported and leave it empty
  int Lq = p.Lq, Lk = p.Lk;
  if (p.cu_q != nullptr) {
    Lq = p.cu_q[lb + 1] - p.cu_q[lb];
    Lk = p.cu_k[lb + 1] - p.cu_k[lb];
    if (Lq < 0 || Lk < 0 || Lq > p.Lq || Lk > p.Lk || p.cu_q[lb] < 0 || p.cu_k[lb] < 0 ||
        p.cu_q[lb + 1] > p.total_q || p.cu_k[lb + 1] > p.total_k) {
      if (threadIdx.x == 0 && qt == 0 && lh == 0) report_error(p.err, SMA_ERR_DEVICE_INPUT);
      Lq = 0;
      Lk = 0;
    }
  }
  const int q0 = qt * kTile;
  const int q1 = min(q0 + kTile, Lq);
  const int off = Lk - Lq;
  // mask code rows used by this list
  int mh0 = 0, mh1 = -1;  // mask head indices (before stride folding)
  if (p.has_mask) {
    const int64_t mhs = p.mask.sizes[1];
    if (p.lists.head_mode == 2) {
      const int hk = lh / p.npairs, pr = lh - hk * p.npairs;
      const int h0 = hk * p.group + 2 * pr;
      mh0 = mhs == 1 ? 0 : h0;
      mh1 = (2 * pr + 1 < p.group) ? (mhs == 1 ? 0 : h0 + 1) : -1;
    } else if (p.lists.head_mode == 1) {
      mh0 = mhs == 1 ? 0 : lh;
    }
  }
  const int mb = (p.has_mask && p.mask.sizes[0] > 1) ? lb : 0;
  const int mq = (p.has_mask && p.mask.sizes[2] > 1) ? qt : 0;
  const int64_t mh_count = p.has_mask ? p.mask.sizes[1] : 1;

  auto code_of = [&](int kt) -> int {
    const int k0 = kt * kTile;
    if (q0 >= Lq || k0 >= Lk) return SMA_TILE_EMPTY;
    const int k1 = min(k0 + kTile, Lk);
    int c = ((kt + 1) * kTile <= Lk) ? SMA_TILE_FULL : SMA_TILE_PARTIAL;
    if (p.causal) {
      int cc;
      if (k1 - 1 <= q0 + off) cc = SMA_TILE_FULL;
      else if (k0 > (q1 - 1) + off) cc = SMA_TILE_EMPTY;
      else cc = SMA_TILE_PARTIAL;
      c = combine_codes(c, cc);
    }
    if (p.has_mask) {
      const int64_t rowbase = (static_cast<int64_t>(mb) * mh_count) * codes_qt;
      int mc = codes[((rowbase + static_cast<int64_t>(mh0) * codes_qt) + mq) * p.KT + kt];
      if (mh1 >= 0) {
        const int mc1 = codes[((rowbase + static_cast<int64_t>(mh1) * codes_qt) + mq) * p.KT + kt];
        mc = union_codes(mc, mc1);
      }
      c = combine_codes(c, mc);
    }
    return c;
  };
  const int64_t row = (static_cast<int64_t>(lb) * p.lists.LH + lh) * p.QT + qt;
  emit_lists(p.KT, code_of, num_full + row, full_idx + row * p.KT, num_part + row,
             part_idx + row * p.KT);
}

}  // namespace

cudaError_t launch_dfa_block_map(const DflashGeom& g, const int32_t* anchors, int32_t* num_full,
                                 int32_t* full_idx, int32_t* num_part, int32_t* part_idx, int* err,
                                 cudaStream_t stream) {
  dim3 grid(g.QT, g.B);
  dfa_block_map_kernel<<<grid, kMapThreads, 0, stream>>>(g, anchors, num_full, full_idx, num_part,
                                                          part_idx, err);
  return cudaGetLastError();
}

cudaError_t launch_mask_tile_summary(const uint8_t* mask, const int64_t sizes[4],
                                     const int64_t strides[4], int Lk, uint8_t* codes,
                                     cudaStream_t stream) {
  const int QT = static_cast<int>(ceil_div(sizes[2], kTile));
  const int KT = static_cast<int>(ceil_div(Lk, kTile));
  const int64_t n_tiles = sizes[0] * sizes[1] * QT * KT;
  if (n_tiles == 0) return cudaSuccess;
  const int64_t blocks = ceil_div(n_tiles, kSummaryWarps);
  mask_summary_kernel<<<static_cast<unsigned>(blocks), kSummaryWarps * 32, 0, stream>>>(
      mask, sizes[0], sizes[1], sizes[2], strides[0], strides[1], strides[2],
      static_cast<int>(sizes[3]), Lk, QT, KT, codes);
  return cudaGetLastError();
}

namespace {
// Lists of packed sequences: list row (b, qt) over the key tiles of sequence
// b, from its lengths cu[b+1] - cu[b]; causal is bottom-right per sequence.
__global__ void __launch_bounds__(kMapThreads)
varlen_lists_kernel(AttnProblem p, int32_t* num_full, int32_t* full_idx, int32_t* num_part,
                    int32_t* part_idx) {
  const int qt = blockIdx.x, b = blockIdx.z;
  int lq = p.cu_q[b + 1] - p.cu_q[b];
  int lk = p.cu_k[b + 1] - p.cu_k[b];
  if (lq < 0 || lk < 0 || lq > p.Lq || lk > p.Lk || p.cu_q[b] < 0 || p.cu_k[b] < 0 ||
      p.cu_q[b + 1] > p.total_q || p.cu_k[b + 1] > p.total_k) {
    if (threadIdx.x == 0 && qt == 0) report_error(p.err, SMA_ERR_DEVICE_INPUT);
    lq = 0;
    lk = 0;
  }
  const int q0 = qt * kTile;
  const int q1 = min(q0 + kTile, lq);
  const int off = lk - lq;
  auto code_of = [&](int kt) -> int {
    const int k0 = kt * kTile;
    if (q0 >= lq || k0 >= lk) return SMA_TILE_EMPTY;
    const int k1 = min(k0 + kTile, lk);
    int c = ((kt + 1) * kTile <= lk) ? SMA_TILE_FULL : SMA_TILE_PARTIAL;
    if (p.causal) {
      int cc;
      if (k1 - 1 <= q0 + off) cc = SMA_TILE_FULL;
      else if (k0 > (q1 - 1) + off) cc = SMA_TILE_EMPTY;
      else cc = SMA_TILE_PARTIAL;
      c = combine_codes(c, cc);
    }
    return c;
  };
  const int64_t row = static_cast<int64_t>(b) * p.QT + qt;
  emit_lists(p.KT, code_of, num_full + row, full_idx + row * p.KT, num_part + row,
             part_idx + row * p.KT);
}
}  // namespace

cudaError_t launch_varlen_lists(const AttnProblem& p, int32_t* num_full, int32_t* full_idx,
                                int32_t* num_part, int32_t* part_idx, cudaStream_t stream) {
  dim3 grid(p.QT, 1, p.B);
  varlen_lists_kernel<<<grid, kMapThreads, 0, stream>>>(p, num_full, full_idx, num_part, part_idx);
  return cudaGetLastError();
}

cudaError_t launch_explicit_lists(const AttnProblem& p, const uint8_t* codes, int codes_q_tiles,
                                  int32_t* num_full, int32_t* full_idx, int32_t* num_part,
                                  int32_t* part_idx, cudaStream_t stream) {
  dim3 grid(p.QT, p.lists.LH, p.lists.LB);
  explicit_lists_kernel<<<grid, kMapThreads, 0, stream>>>(p, codes, codes_q_tiles, num_full,
                                                           full_idx, num_part, part_idx);
  return cudaGetLastError();
}

}  // namespace sma
