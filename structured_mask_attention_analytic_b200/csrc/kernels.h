// Internal (non-ABI) description of the problems the kernels solve, and the
// host-side launchers the C ABI calls.  Plain C++ structs; no torch types.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace sma {

constexpr int kTile = 128;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t m) { return ceil_div(a, m) * m; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// DFlash mask geometry after is_causal / window resolution.
struct DflashGeom {
  int B, N, bs, Lc;  // batch, blocks, block size, context keys
  int Nq, Lk;        // queries, keys
  int QT, KT;        // 128-tiles of queries / keys
  int causal;        // 1: causal inside the block
  int window;        // left window W, 0 = none
};

// Mask or bias operand after stride-0 folding of its size-1 dims.
struct AuxView {
  const void* ptr = nullptr;
  int dtype = 0;        // bias dtype (SMA_BF16/FP16/FP32); unused for masks
  int64_t sb = 0, sh = 0, sq = 0;  // element strides, 0 for broadcast dims
  int head_per_query = 0;          // 1: head index is the query head, 0: the KV head
  int64_t sizes[4] = {0, 0, 0, 0};
  // Key columns each row holds: round_up(Lk, 128) (the padded form), Lk, or
  // 1 (one value for every key: the key dim broadcasts with stride 0).
  // Kernels read column min(k, kd - 1) for key k, so no access leaves a row.
  int kd = 0;
};

// Ascending key-tile lists; list row = (lb * LH + lh) * QT + qt.
struct TileLists {
  const int32_t* num_full = nullptr;
  const int32_t* full_idx = nullptr;
  const int32_t* num_part = nullptr;
  const int32_t* part_idx = nullptr;
  int LB = 1;         // batch rows (1 = shared by every batch entry)
  int LH = 1;         // head rows
  int head_mode = 0;  // 0: lh = 0; 1: lh = kv head; 2: lh = kv head * npairs + pair
};

// Gather: explicit policy over compacted keys (GatherView set, no mask).
// Varlen: packed sequences (cu_q / cu_k set), causal or not, no mask / bias.
enum MaskPolicy { kPolicyDflash = 0, kPolicyExplicit = 1, kPolicyGather = 2, kPolicyVarlen = 3 };

// Index-gather view of a query-broadcast keep mask: per gather row (batch
// row LB x head row LH of the mask, the same rows as the tile lists) the
// ascending original indices of the kept keys.  When set, the problem's k, v
// and bias are the compacted operands (compacted key j of a row is original
// key idx[row][j]) and Lk is the compacted capacity.
struct GatherView {
  const int32_t* idx = nullptr;    // [rows, cap]
  const int32_t* count = nullptr;  // [rows], <= cap
  int cap = 0;                     // multiple of 128
  int k_len = 0;                   // original key length
  int causal = 0;                  // bottom-right causal bound on original indices
};

// One attention forward problem: O[b, q, h] over keys of head h / group.
struct AttnProblem {
  int dtype;  // SMA_BF16 / SMA_FP16 / SMA_FP32 (q, k, v, out)
  int B, H, KVH, Lq, Lk, d;
  int group, npairs, QT, KT;
  float scale_log2;  // scale * log2(e)
  const void* q; int64_t q_sb, q_sr, q_sh;
  const void* k; int64_t k_sb, k_sr, k_sh;
  const void* v; int64_t v_sb, v_sr, v_sh;
  void* o; int64_t o_sb, o_sr, o_sh;
  float* lse;  // [B, H, Lq] contiguous or null
  TileLists lists;
  int policy;
  // DFlash policy
  const int32_t* anchors; int N, bs, Lc, causal_in_block, window;
  // explicit policy
  int causal;
  int has_mask, has_bias;
  AuxView mask, bias;
  // Bias on the tensor cores (tcgen05 explicit path, set by the launcher):
  // a bias shared by every query of a row of S, b[k], enters S = Q K^T as one
  // more K step whose A rows are [hi, lo, 0, ...] (1 / scale split into two
  // values of the operand type, packed hi | lo << 16 here) and whose B rows are
  // [b[k], b[k], 0, ...], so S holds q.k + b / scale and the softmax adds no
  // bias itself.
  int bias_tc = 0;
  uint32_t bias_tc_a = 0;
  GatherView gather;  // idx == nullptr: keys are not compacted
  // varlen policy: sequence b holds query rows [cu_q[b], cu_q[b+1]) of the
  // packed [total_q, H, d] operands (keys likewise); Lq / Lk are the maxima
  const int32_t* cu_q = nullptr;
  const int32_t* cu_k = nullptr;
  int total_q = 0, total_k = 0;
  // Key-range split (tcgen05 path, not varlen): each unit's key-tile list is
  // cut into n_split contiguous segments run as separate units.  Segment s
  // writes its rows' unnormalised O to part_o[s][row] and (running max in
  // log2 units, sum of exponentials) to part_ml[s][row]; a combine kernel
  // merges them into o and lse.  row = (b * H + h) * Lq + q, part_rows =
  // B * H * Lq.
  int n_split = 1;
  float* part_o = nullptr;   // [n_split, part_rows, d]
  float* part_ml = nullptr;  // [n_split, part_rows, 2]
  int64_t part_rows = 0;
  // Head packing (tcgen05 path; set by the launcher, see fwd_pack): with
  // pack = P > 1 a 128-row tile holds the P query heads of a KV head for
  // 128 / P consecutive queries (row r: head r % P, query r / P).
  int pack = 1;
  int* err;  // device error word
};

// Query heads per 128-row tile of the tcgen05 forward: the whole group when
// the queries are few (<= 64, so a head-per-tile layout would leave most rows
// empty), the group has 2, 4 or 8 heads and the tile lists are shared by the
// group's heads; 1 otherwise.
inline int fwd_pack(int Lq, int group, int head_mode, int policy) {
  if (policy == kPolicyVarlen || head_mode == 2 || Lq > 64) return 1;
  return (group == 2 || group == 4 || group == 8) ? group : 1;
}

// Units of the tcgen05 forward before any key-range split: (batch, KV head,
// pair of query heads, 128-query tile), or with head packing (batch, KV head,
// pair of 128 / pack-query blocks).
inline int64_t fwd_units(int B, int KVH, int npairs, int QT, int Lq, int pack) {
  if (pack == 1) return static_cast<int64_t>(B) * KVH * npairs * QT;
  const int rows = kTile / pack;
  const int qblocks = (Lq + rows - 1) / rows;
  return static_cast<int64_t>(B) * KVH * ((qblocks + 1) / 2);
}

// Backward of one attention problem.  `f` is the forward problem (q, k, v,
// geometry, policy, masks and the forward tile lists, f.o = the forward
// output O, f.lse = its log-sum-exp, read only); the transposed lists give,
// per list row and key tile, the query tiles that attend it.
struct BwdProblem {
  AttnProblem f;
  const void* dout; int64_t do_sb, do_sr, do_sh;   // upstream gradient dO [B, Lq, H, d]
  void* dq; int64_t dq_sb, dq_sr, dq_sh;           // [B, Lq, H, d]
  void* dk; int64_t dk_sb, dk_sr, dk_sh;           // [B, Lk, KVH, d]
  void* dv; int64_t dv_sb, dv_sr, dv_sh;
  float* dq_acc;   // [B, Lq, H, d] fp32, zeroed by the preparation kernel
  float* dvec;     // [B, H, Lq]: rowsum(dO * O)
  const int32_t* t_num_full; const int32_t* t_full;  // [rows, KT], [rows, KT, QT]
  const int32_t* t_num_part; const int32_t* t_part;
  float scale;     // softmax scale (dQ and dK carry it)
  // Gradient of the bias (explicit policy only): fp32, the bias's broadcast
  // shape (b', h', q', db_kd) with db_kd the bias's key dim (128-rounded Lk, or
  // Lk), zeroed before the kernel runs; element (b, h, q, k) of dS adds into
  // dbias[b * db_sb + hb * db_sh + q * db_sq + k] for k < db_kd (strides 0 on
  // broadcast dims; hb = h if db_head_per_query else h / group).
  float* dbias = nullptr;
  int64_t db_sb = 0, db_sh = 0, db_sq = 0;
  int db_kd = 0;
  int db_head_per_query = 0;
  int db_mode = 0;  // kDbias* below
};

#ifdef __CUDACC__
// Rows of one sequence (batch entry b): its first query / key row and its
// lengths.  Packed sequences (varlen) take them from the cumulative offsets;
// malformed offsets give an empty sequence (nothing of it is read or
// written; the list kernel reports them).  Padded batches: row 0, Lq, Lk.
struct SeqRows {
  int q_off, lq, k_off, lk;
};
template <int POLICY>
__device__ __forceinline__ SeqRows seq_rows(const AttnProblem& p, int b) {
  SeqRows s{0, p.Lq, 0, p.Lk};
  if (POLICY == kPolicyVarlen) {
    s.q_off = p.cu_q[b];
    s.lq = p.cu_q[b + 1] - s.q_off;
    s.k_off = p.cu_k[b];
    s.lk = p.cu_k[b + 1] - s.k_off;
    if (s.lq < 0 || s.lq > p.Lq || s.q_off < 0 || s.q_off + s.lq > p.total_q || s.lk < 0 ||
        s.lk > p.Lk || s.k_off < 0 || s.k_off + s.lk > p.total_k)
      s = SeqRows{0, 0, 0, 0};
  }
  return s;
}
// Index of (b, h, q) in the per-row float arrays (lse, rowsum(dO * O)):
// [B, H, Lq], or [H, total_q] for packed sequences.
template <int POLICY>
__device__ __forceinline__ int64_t row_index(const AttnProblem& p, int b, int h, const SeqRows& s,
                                             int q) {
  return POLICY == kPolicyVarlen ? static_cast<int64_t>(h) * p.total_q + s.q_off + q
                                 : (static_cast<int64_t>(b) * p.H + h) * p.Lq + q;
}
#endif

// How the backward writes dbias: not at all; one store per element (every
// element of dS has its own dbias element); one atomic add per element
// (several heads or batch rows share an element); one atomic add of each
// thread's sum over its queries (dbias broadcast over the queries); or, for
// the fixed-order (deterministic) dbias, one store of each thread's sum over
// its group of kDbiasGroupRows queries into row q / kDbiasGroupRows of a
// partial buffer (every partial element has exactly one writer).
enum DbiasMode { kDbiasNone = 0, kDbiasStore = 1, kDbiasAdd = 2, kDbiasRowSum = 3,
                 kDbiasGroupStore = 4 };
// Query rows summed per partial row by the tensor-core backward kernel (the
// transposed kernel, both head dims): each thread's 64 queries.
constexpr int dbias_group_rows(int) { return 64; }

// Single-query (decode) problem after the grouped-head swap: for each
// (b, kv head) the `group` query heads are the rows.
struct DecodeProblem {
  int dtype;
  int B, H, KVH, Lk, Kpad, d, group;
  float scale_log2;
  const void* q; int64_t q_sb, q_sh;
  const void* k; int64_t k_sb, k_sr, k_sh;
  const void* v; int64_t v_sb, v_sr, v_sh;
  void* o; int64_t o_sb, o_sh;
  float* lse;  // [B, H] (q_len 1) or null
  int has_mask, has_bias;
  AuxView mask, bias;
  // Bias on the tensor cores (tcgen05 explicit path, set by the launcher):
  // a bias shared by every query of a row of S, b[k], enters S = Q K^T as one
  // more K step whose A rows are [hi, lo, 0, ...] (1 / scale split into two
  // values of the operand type, packed hi | lo << 16 here) and whose B rows are
  // [b[k], b[k], 0, ...], so S holds q.k + b / scale and the softmax adds no
  // bias itself.
  int bias_tc = 0;
  uint32_t bias_tc_a = 0;
  int splits, chunk;       // split-KV: split s takes key tiles [s nt / splits, (s+1) nt / splits); chunk unused
  float* part_o;           // [B, H, splits, d]
  float* part_ml;          // [B, H, splits, 2]  (max in log2 units, sum)
  int* err;
};

struct TopkProblem {
  int bias_dtype;
  const void* bias; int64_t b_sizes[4]; int64_t b_strides[4];
  int Lk;
  int Kcols;  // columns of each bias / output row: round_up(Lk, 128) or Lk
  const uint8_t* pre; int64_t p_sizes[4]; int64_t p_strides[4];  // strides 0 on broadcast dims
  int window;
  uint8_t* out;
};

// ---- launchers (return cudaSuccess or the launch error)
cudaError_t launch_dfa_block_map(const DflashGeom& g, const int32_t* anchors, int32_t* num_full,
                                 int32_t* full_idx, int32_t* num_part, int32_t* part_idx, int* err,
                                 cudaStream_t stream);

cudaError_t launch_mask_tile_summary(const uint8_t* mask, const int64_t sizes[4],
                                     const int64_t strides[4], int Lk, uint8_t* codes,
                                     cudaStream_t stream);

// Tile lists of the explicit-mask path from the summary codes (may be null),
// causal flag and key length.  Writes LB*LH*QT lists.
cudaError_t launch_explicit_lists(const AttnProblem& p, const uint8_t* codes, int codes_q_tiles,
                                  int32_t* num_full, int32_t* full_idx, int32_t* num_part,
                                  int32_t* part_idx, cudaStream_t stream);

// Tile lists of packed sequences: per (sequence, query tile) the key tiles
// of that sequence, causal (bottom-right per sequence) or not.  Malformed
// offsets raise SMA_ERR_DEVICE_INPUT and give empty lists.
cudaError_t launch_varlen_lists(const AttnProblem& p, int32_t* num_full, int32_t* full_idx,
                                int32_t* num_part, int32_t* part_idx, cudaStream_t stream);

// Packed <-> padded copies of [total, heads, d] rows (pad zero-fills rows past
// each sequence's length).  esz: element size in bytes.
cudaError_t launch_varlen_pad(const void* packed, void* padded, const int32_t* cu, int batch,
                              int max_len, int heads, int d, int esz, int64_t p_row, int64_t p_head,
                              int64_t d_sb, int64_t d_sr, int64_t d_sh, cudaStream_t stream);
cudaError_t launch_varlen_unpad(const void* padded, void* packed, const int32_t* cu, int batch,
                                int max_len, int heads, int d, int esz, int64_t p_row,
                                int64_t p_head, int64_t s_sb, int64_t s_sr, int64_t s_sh,
                                cudaStream_t stream);

// tcgen05 forward (bf16 / fp16).  Returns a nonzero SMA status on a host-side
// failure (tensor map encoding) and writes a message to `msg`.
int launch_attn_tc(const AttnProblem& p, cudaStream_t stream, char* msg, size_t msg_len);

// fp32 FFMA forward.
cudaError_t launch_attn_simt(const AttnProblem& p, cudaStream_t stream);

cudaError_t launch_decode(const DecodeProblem& p, cudaStream_t stream);

// Index-gather preparation.  `mask` is a query-broadcast keep mask with
// element strides m_sb / m_sh (0 on broadcast dims) and m_kd columns per row
// (round_up(Lk, 128), Lk or 1); gather row (lb, lh) reads mask row
// lb * m_sb + lh * m_sh.
cudaError_t launch_select_keys(const uint8_t* mask, int64_t m_sb, int64_t m_sh, int m_kd, int LB,
                               int LH, int Lk, int cap, int32_t* idx, int32_t* count, int* err,
                               cudaStream_t stream);
// Compacted K and V ([B, cap, KVH, d], the strides in p.k/p.v) from the
// original operands; rows from count to the next multiple of 128 are zeroed.
cudaError_t launch_gather_kv(const AttnProblem& p, const void* k, const int64_t k_strides[3],
                             const void* v, const int64_t v_strides[3], cudaStream_t stream);
// Compacted bias (the view in p.bias, cap columns) from the original view.
cudaError_t launch_gather_bias(const AttnProblem& p, const AuxView& bias, int rows_h, int rows_q,
                               cudaStream_t stream);
// FULL / PARTIAL key-tile lists over the compacted keys.
cudaError_t launch_gather_lists(const AttnProblem& p, cudaStream_t stream);

cudaError_t launch_topk(const TopkProblem& p, cudaStream_t stream);

// Backward: rowsum(dO * O) and a zeroed dQ accumulator; the transposed tile
// lists (codes: scratch of rows * QT * KT bytes); the tcgen05 kernel (dK, dV
// and dQ partial sums); dQ = scale * accumulator in the output dtype.
cudaError_t launch_bwd_prep(const BwdProblem& p, cudaStream_t stream);
cudaError_t launch_transpose_lists(const BwdProblem& p, uint8_t* codes, cudaStream_t stream);
int launch_attn_bwd(const BwdProblem& p, cudaStream_t stream, char* msg, size_t msg_len);
cudaError_t launch_dq_convert(const BwdProblem& p, cudaStream_t stream);
// Fixed-order dbias: out[b', h', q', k] (the bias's broadcast shape, kd key
// columns) = the sum, in increasing (b, h, r) order, of part[b][h][r][k]
// ([B, H, R, kd]) over the batch rows, query heads and partial rows that
// element (b', h', q') gathers: every b when nb == 1, else b'; every head
// when nh == 1, heads [h' g, h' g + g) when nh is the KV head count and g =
// H / nh > 1, else h'; every r when nq == 1, else r = q'.
cudaError_t launch_dbias_reduce(const float* part, int B, int H, int R, float* out, int nb, int nh,
                                int nq, int kd, cudaStream_t stream);
// fp32 FFMA backward (dQ accumulator, dK, dV, dbias), after launch_bwd_prep
// and launch_transpose_lists; launch_dq_convert follows.
cudaError_t launch_attn_bwd_simt(const BwdProblem& p, cudaStream_t stream);

// Records `message` as the calling thread's last error (read back through
// sma_last_error) and returns `code`.
int set_last_error(int code, const char* message);

cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, int* err, int64_t* out,
                                         cudaStream_t stream);

// Device error word in the current context (looked up once per context).
int* device_error_word(cudaError_t* status);

// Unique id of the CUDA context current on the calling thread (ids are never
// reused within a process, so a context created after cudaDeviceReset, or a
// caller's own non-primary context, gets a new one); 0 if none is current.
unsigned long long current_context_id();

// Device addresses of a __device__ symbol per CUDA context.  A symbol's
// address belongs to the context the module is loaded in: it is not valid in
// another context of the same device, nor after the context is destroyed.
struct ContextAddressCache {
  static constexpr int kSlots = 64;
  std::mutex mutex;
  unsigned long long ids[kSlots] = {};
  void* ptrs[kSlots] = {};
  int count = 0;
  unsigned next_evict = 0;
  void* find(unsigned long long ctx_id);  // nullptr if not cached (or ctx_id 0)
  void insert(unsigned long long ctx_id, void* ptr);
};

int num_sms();

}  // namespace sma
