// C ABI of libsma (declared in include/sma.h): argument validation, stride-0
// folding of broadcast dims, workspace layout and stream-ordered launches.
// Nothing here allocates device memory or synchronises the stream (except
// sma_device_status, whose job is to synchronise).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "kernels.h"
#include "sma.h"

using namespace sma;

namespace {

thread_local std::string g_last_error;

sma_status fail(sma_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

sma_status ok() {
  g_last_error.clear();
  return SMA_OK;
}

sma_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SMA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int elem_size(int32_t dtype) { return dtype == SMA_FP32 ? 4 : 2; }

bool valid_dtype(int32_t dt) { return dt == SMA_BF16 || dt == SMA_FP16 || dt == SMA_FP32; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float resolve_scale(float scale, int d) {
  return scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
}

constexpr float kLog2eHost = 1.4426950408889634f;

// Q/K/V/O operand: [batch, len, heads, d], d contiguous.
sma_status check_operand(const char* name, const void* ptr, const int64_t* strides, int32_t dtype,
                         int64_t len) {
  if (ptr == nullptr) return fail(SMA_ERR_INVALID_ARG, "%s is NULL", name);
  if (strides == nullptr) return fail(SMA_ERR_INVALID_ARG, "%s strides are NULL", name);
  if (!aligned16(ptr)) return fail(SMA_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  const int es = elem_size(dtype);
  for (int i = 0; i < 3; ++i) {
    if (strides[i] < 0) return fail(SMA_ERR_INVALID_ARG, "%s stride %d is negative", name, i);
    if ((strides[i] * es) % 16 != 0)
      return fail(SMA_ERR_INVALID_ARG, "%s stride %d (%lld elements) is not a multiple of 16 bytes",
                  name, i, static_cast<long long>(strides[i]));
  }
  (void)len;
  return SMA_OK;
}

sma_status check_heads(int32_t heads, int32_t kv_heads, int32_t head_dim) {
  if (heads < 1 || kv_heads < 1) return fail(SMA_ERR_INVALID_ARG, "heads and kv_heads must be >= 1");
  if (heads % kv_heads != 0)
    return fail(SMA_ERR_INVALID_ARG, "heads (%d) must be a multiple of kv_heads (%d)", heads, kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(SMA_ERR_UNSUPPORTED, "head_dim %d is not supported (64 or 128)", head_dim);
  return SMA_OK;
}

// Mask/bias operand of the 4D broadcast contract; fills `view`.
sma_status check_aux(const char* name, const void* ptr, const int64_t* sizes,
                     const int64_t* strides, int esz, int32_t B, int32_t H, int32_t KVH,
                     int32_t Lq, int32_t Lk, bool allow_key_dim_1, AuxView* view) {
  if (sizes == nullptr || strides == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "%s sizes/strides are NULL", name);
  const int64_t kpad = round_up(Lk, kTile);
  if (sizes[0] != B && sizes[0] != 1)
    return fail(SMA_ERR_INVALID_ARG, "%s batch dim %lld must be %d or 1", name,
                static_cast<long long>(sizes[0]), B);
  if (sizes[1] != H && sizes[1] != KVH && sizes[1] != 1)
    return fail(SMA_ERR_INVALID_ARG, "%s head dim %lld must be %d, %d or 1", name,
                static_cast<long long>(sizes[1]), H, KVH);
  if (sizes[2] != Lq && sizes[2] != 1)
    return fail(SMA_ERR_INVALID_ARG, "%s query dim %lld must be %d or 1", name,
                static_cast<long long>(sizes[2]), Lq);
  // PR #190's interface pads the key dim to round_up(Lk, 128) and expands a
  // key dim of 1; the kernels read all three forms in place (no copy).
  if (sizes[3] != kpad && sizes[3] != Lk && sizes[3] != 1)
    return fail(SMA_ERR_INVALID_ARG,
                "%s key dim %lld must be round_up(k_len, 128) = %lld, k_len = %d or 1", name,
                static_cast<long long>(sizes[3]), static_cast<long long>(kpad), Lk);
  if (!allow_key_dim_1 && sizes[3] == 1 && Lk > 1)
    return fail(SMA_ERR_INVALID_ARG, "%s key dim 1 is not accepted here", name);
  if (sizes[3] != 1 && strides[3] != 1)
    return fail(SMA_ERR_INVALID_ARG, "%s last dim must be contiguous", name);
  // Rows of more than one column are read with 16-byte vector loads; a row
  // of one column is read one element at a time and needs only element
  // alignment.
  const bool one_col = sizes[3] == 1;
  if (!one_col && !aligned16(ptr))
    return fail(SMA_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  if (one_col && (reinterpret_cast<uintptr_t>(ptr) % esz) != 0)
    return fail(SMA_ERR_INVALID_ARG, "%s must be aligned to its element size", name);
  view->ptr = ptr;
  view->sb = sizes[0] == 1 ? 0 : strides[0];
  view->sh = sizes[1] == 1 ? 0 : strides[1];
  view->sq = sizes[2] == 1 ? 0 : strides[2];
  for (int64_t s : {view->sb, view->sh, view->sq}) {
    if (s < 0) return fail(SMA_ERR_INVALID_ARG, "%s has a negative stride", name);
    if (!one_col && (s * esz) % 16 != 0)
      return fail(SMA_ERR_INVALID_ARG, "%s strides must be multiples of 16 bytes", name);
  }
  view->head_per_query = sizes[1] == H ? 1 : 0;
  for (int i = 0; i < 4; ++i) view->sizes[i] = sizes[i];
  view->kd = static_cast<int>(sizes[3]);
  return SMA_OK;
}

sma_status check_desc(const dfa_mask_desc* d) {
  if (d == nullptr) return fail(SMA_ERR_INVALID_ARG, "desc is NULL");
  if (d->batch < 1 || d->n_blocks < 1 || d->block_size < 1 || d->ctx_len < 0)
    return fail(SMA_ERR_INVALID_ARG, "batch, n_blocks, block_size must be >= 1 and ctx_len >= 0");
  if (d->is_causal != SMA_IS_CAUSAL_UNSET && d->is_causal != 0 && d->is_causal != 1)
    return fail(SMA_ERR_INVALID_ARG, "is_causal must be -1, 0 or 1");
  if (d->layer_type != SMA_LAYER_FULL && d->layer_type != SMA_LAYER_SLIDING)
    return fail(SMA_ERR_INVALID_ARG, "layer_type must be 0 (full) or 1 (sliding)");
  if (d->layer_type == SMA_LAYER_SLIDING && d->sliding_window < 1)
    return fail(SMA_ERR_INVALID_ARG, "sliding layers need sliding_window >= 1");
  const int64_t nq = static_cast<int64_t>(d->n_blocks) * d->block_size;
  if (nq + d->ctx_len > (1LL << 30)) return fail(SMA_ERR_INVALID_ARG, "key length too large");
  return SMA_OK;
}

DflashGeom make_geom(const dfa_mask_desc* d) {
  DflashGeom g;
  g.B = d->batch;
  g.N = d->n_blocks;
  g.bs = d->block_size;
  g.Lc = d->ctx_len;
  g.Nq = d->n_blocks * d->block_size;
  g.Lk = g.Lc + g.Nq;
  g.QT = static_cast<int>(ceil_div(g.Nq, kTile));
  g.KT = static_cast<int>(ceil_div(g.Lk, kTile));
  // SpecForge PR #905, Motivation list.
  if (d->is_causal == SMA_IS_CAUSAL_UNSET) g.causal = d->layer_type == SMA_LAYER_SLIDING ? 1 : 0;
  else g.causal = d->is_causal;
  g.window = d->layer_type == SMA_LAYER_SLIDING ? d->sliding_window : 0;
  return g;
}

struct ListsLayout {
  size_t nf, np, fi, pi, end;
};

ListsLayout lists_layout(size_t base, int64_t rows, int KT) {
  ListsLayout l;
  l.nf = base;
  l.np = align256(l.nf + rows * 4);
  l.fi = align256(l.np + rows * 4);
  l.pi = align256(l.fi + rows * KT * 4);
  l.end = align256(l.pi + rows * KT * 4);
  return l;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---- key-range split of short-query forwards.  When the (batch, KV head,
// head pair, query tile) units of the tcgen05 forward fill at most half of
// the SMs, each unit's key-tile list is cut into n_split segments that run on
// separate SMs: as many segments per unit as whole units fit in one wave,
// at most one segment per 4 key tiles of a full list, and at most 32.  The
// partial results sit in the workspace after `base`.
struct SplitLayout {
  int n_split;
  size_t part_o, part_ml, end;
};

SplitLayout split_layout(size_t base, int B, int H, int KVH, int Lq, int d, int QT, int KT,
                         int head_mode, int policy) {
  SplitLayout s{1, base, base, base};
  const int group = H / KVH;
  const int64_t units =
      fwd_units(B, KVH, (group + 1) / 2, QT, Lq, fwd_pack(Lq, group, head_mode, policy));
  int64_t ns = units > 0 ? num_sms() / units : 1;
  if (ns > KT / 4) ns = KT / 4;
  if (ns > 32) ns = 32;
  if (ns < 2) return s;
  s.n_split = static_cast<int>(ns);
  const size_t rows = static_cast<size_t>(B) * H * Lq;
  s.part_o = align256(base);
  s.part_ml = align256(s.part_o + static_cast<size_t>(ns) * rows * d * 4);
  s.end = align256(s.part_ml + static_cast<size_t>(ns) * rows * 8);
  return s;
}

// Enables the split on a tensor-core problem whose workspace holds it.
void apply_split(AttnProblem& p, const SplitLayout& s, void* ws) {
  if (s.n_split < 2 || p.dtype == SMA_FP32) return;
  p.n_split = s.n_split;
  p.part_o = at<float>(ws, s.part_o);
  p.part_ml = at<float>(ws, s.part_ml);
  p.part_rows = static_cast<int64_t>(p.B) * p.H * p.Lq;
}

sma_status check_workspace(void* ws, size_t have, size_t need) {
  if (have < need)
    return fail(SMA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", have,
                need);
  if (need > 0 && ws == nullptr) return fail(SMA_ERR_INVALID_ARG, "workspace is NULL");
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(SMA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return SMA_OK;
}

// ---- masked path geometry
struct MaskedGeom {
  int LB, LH, head_mode, npairs, QT, KT, codes_qt;
  bool decode;
  int splits, chunk;
  size_t codes_bytes;
  ListsLayout lists;
  SplitLayout kv_split;  // key-range split of the tcgen05 forward
  size_t part_o, part_ml, total;
};

MaskedGeom masked_geom(int32_t B, int32_t H, int32_t KVH, int32_t Lq, int32_t Lk, int32_t d,
                       const int64_t* mask_sizes) {
  MaskedGeom g{};
  const int group = H / KVH;
  g.npairs = (group + 1) / 2;
  g.QT = static_cast<int>(ceil_div(Lq, kTile));
  g.KT = static_cast<int>(ceil_div(Lk, kTile));
  g.decode = Lq == 1;
  if (g.decode) {
    // split-KV: the kernel runs two CTAs per SM and a split takes an even
    // share of the key tiles (kernel side).  The split count minimises the
    // estimated time: waves of CTAs over the 2 x SM-count slots times the
    // 64-key steps of a split, plus two steps of fixed cost per CTA; splits
    // keep at least 512 keys, at most 64.
    const int rows_groups = (group + 7) / 8;
    const int64_t base_ctas = static_cast<int64_t>(B) * KVH * rows_groups;
    const int64_t slots = 2 * static_cast<int64_t>(num_sms());
    const int64_t steps = ceil_div(Lk, 64);
    const int max_splits = static_cast<int>(std::min<int64_t>(64, std::max<int64_t>(1, ceil_div(Lk, 512))));
    int splits = 1;
    int64_t best = -1;
    for (int sp = 1; sp <= max_splits; ++sp) {
      const int64_t cost = ceil_div(base_ctas * sp, slots) * (ceil_div(steps, sp) + 2);
      if (best < 0 || cost < best) {
        best = cost;
        splits = sp;
      }
    }
    g.splits = splits;
    g.chunk = 0;  // the kernel derives each split's key range
    g.part_o = 0;
    g.part_ml = align256(static_cast<size_t>(B) * H * splits * d * 4);
    g.total = align256(g.part_ml + static_cast<size_t>(B) * H * splits * 2 * 4);
    return g;
  }
  const bool has_mask = mask_sizes != nullptr;
  g.LB = (has_mask && mask_sizes[0] > 1) ? B : 1;
  if (!has_mask || mask_sizes[1] == 1) {
    g.head_mode = 0;
    g.LH = 1;
  } else if (mask_sizes[1] == H) {
    g.head_mode = 2;
    g.LH = KVH * g.npairs;
  } else {
    g.head_mode = 1;
    g.LH = KVH;
  }
  g.codes_qt = has_mask ? static_cast<int>(ceil_div(mask_sizes[2], kTile)) : 0;
  g.codes_bytes =
      has_mask ? align256(static_cast<size_t>(mask_sizes[0] * mask_sizes[1]) * g.codes_qt * g.KT) : 0;
  g.lists = lists_layout(g.codes_bytes, static_cast<int64_t>(g.LB) * g.LH * g.QT, g.KT);
  g.kv_split = split_layout(g.lists.end, B, H, KVH, Lq, d, g.QT, g.KT, g.head_mode, kPolicyExplicit);
  g.total = g.kv_split.end;
  return g;
}


// ---- backward workspace: forward tile lists (unless given), transposed
// lists, tile codes, rowsum(dO * O) and the fp32 dQ accumulator.
struct BwdLayout {
  ListsLayout fl;
  size_t tnf, tnp, tf, tp, codes, dvec, dqacc, total;
};

BwdLayout bwd_layout(size_t base, int64_t rows, int QT, int KT, int B, int H, int Lq, int d) {
  BwdLayout l;
  l.fl = lists_layout(base, rows * QT, KT);
  l.tnf = l.fl.end;
  l.tnp = align256(l.tnf + static_cast<size_t>(rows) * KT * 4);
  l.tf = align256(l.tnp + static_cast<size_t>(rows) * KT * 4);
  l.tp = align256(l.tf + static_cast<size_t>(rows) * KT * QT * 4);
  l.codes = align256(l.tp + static_cast<size_t>(rows) * KT * QT * 4);
  l.dvec = align256(l.codes + static_cast<size_t>(rows) * QT * KT);
  l.dqacc = align256(l.dvec + static_cast<size_t>(B) * H * Lq * 4);
  l.total = align256(l.dqacc + static_cast<size_t>(B) * Lq * H * d * 4);
  return l;
}

// Runs the backward launches for a filled problem (forward lists in place).
sma_status run_backward(BwdProblem& b, void* ws, const BwdLayout& l, cudaStream_t st) {
  b.t_num_full = at<int32_t>(ws, l.tnf);
  b.t_num_part = at<int32_t>(ws, l.tnp);
  b.t_full = at<int32_t>(ws, l.tf);
  b.t_part = at<int32_t>(ws, l.tp);
  b.dvec = at<float>(ws, l.dvec);
  b.dq_acc = at<float>(ws, l.dqacc);
  cudaError_t e = launch_bwd_prep(b, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward preparation launch failed");
  e = launch_transpose_lists(b, at<uint8_t>(ws, l.codes), st);
  if (e != cudaSuccess) return cuda_fail(e, "tile list transpose launch failed");
  char msg[256];
  const int rc = launch_attn_bwd(b, st, msg, sizeof(msg));
  if (rc != SMA_OK) return fail(rc, "%s", msg);
  e = launch_dq_convert(b, st);
  if (e != cudaSuccess) return cuda_fail(e, "dQ conversion launch failed");
  return SMA_OK;
}

sma_status check_grad_operands(int32_t dtype, int64_t lq, int64_t lk, const void* out,
                               const int64_t* o_strides, const float* lse, const void* dout,
                               const int64_t* do_strides, const void* dq, const int64_t* dq_strides,
                               const void* dk, const int64_t* dk_strides, const void* dv,
                               const int64_t* dv_strides) {
  sma_status s;
  if ((s = check_operand("out", out, o_strides, dtype, lq)) != SMA_OK) return s;
  if ((s = check_operand("dout", dout, do_strides, dtype, lq)) != SMA_OK) return s;
  if ((s = check_operand("dq", dq, dq_strides, dtype, lq)) != SMA_OK) return s;
  if ((s = check_operand("dk", dk, dk_strides, dtype, lk)) != SMA_OK) return s;
  if ((s = check_operand("dv", dv, dv_strides, dtype, lk)) != SMA_OK) return s;
  if (lse == nullptr) return fail(SMA_ERR_INVALID_ARG, "lse is NULL (the forward's log-sum-exp is required)");
  return SMA_OK;
}

void set_grads(BwdProblem& b, const void* dout, const int64_t* ds, void* dq, const int64_t* qs,
               void* dk, const int64_t* ks, void* dv, const int64_t* vs, float scale) {
  b.dout = dout; b.do_sb = ds[0]; b.do_sr = ds[1]; b.do_sh = ds[2];
  b.dq = dq; b.dq_sb = qs[0]; b.dq_sr = qs[1]; b.dq_sh = qs[2];
  b.dk = dk; b.dk_sb = ks[0]; b.dk_sr = ks[1]; b.dk_sh = ks[2];
  b.dv = dv; b.dv_sb = vs[0]; b.dv_sr = vs[1]; b.dv_sh = vs[2];
  b.scale = scale;
}

// ---- index-gather path geometry: kept-key lists, tile lists over the
// compacted keys, compacted K/V and bias, all in the workspace.
struct SparseGeom {
  int LB, LH, QT, KT, cap, Hc, Qc;
  size_t idx, count;
  ListsLayout lists;
  size_t kc, vc, bias;
  SplitLayout kv_split;
  size_t total;
};

sma_status sparse_geom(int32_t dtype, int32_t B, int32_t H, int32_t KVH, int32_t Lq, int32_t Lk,
                       int32_t d, const int64_t* mask_sizes, int32_t bias_dtype,
                       const int64_t* bias_sizes, int32_t max_keys, SparseGeom* g) {
  if (mask_sizes == nullptr) return fail(SMA_ERR_INVALID_ARG, "the index-gather path needs a mask");
  if (mask_sizes[2] != 1)
    return fail(SMA_ERR_UNSUPPORTED,
                "index-gather attention needs a mask broadcast over queries (size 1 in dim 2, "
                "got %lld); use masked_attn_fwd",
                static_cast<long long>(mask_sizes[2]));
  if (mask_sizes[1] != 1 && mask_sizes[1] != KVH)
    return fail(SMA_ERR_UNSUPPORTED,
                "index-gather attention needs mask rows shared by the query heads of a KV head "
                "(head dim 1 or %d, got %lld); use masked_attn_fwd",
                KVH, static_cast<long long>(mask_sizes[1]));
  if (mask_sizes[0] != 1 && mask_sizes[0] != B)
    return fail(SMA_ERR_INVALID_ARG, "mask batch dim must be %d or 1", B);
  g->LB = mask_sizes[0] > 1 ? B : 1;
  g->LH = mask_sizes[1] > 1 ? KVH : 1;
  g->QT = static_cast<int>(ceil_div(Lq, kTile));
  const int keys = (max_keys <= 0 || max_keys > Lk) ? Lk : max_keys;
  g->cap = static_cast<int>(round_up(keys, kTile));
  g->KT = g->cap / kTile;
  const int64_t rows = static_cast<int64_t>(g->LB) * g->LH;
  g->idx = 0;
  g->count = align256(static_cast<size_t>(rows) * g->cap * 4);
  g->lists = lists_layout(align256(g->count + rows * 4), rows * g->QT, g->KT);
  const size_t kv_bytes = static_cast<size_t>(B) * g->cap * KVH * d * elem_size(dtype);
  g->kc = g->lists.end;
  g->vc = align256(g->kc + kv_bytes);
  g->bias = align256(g->vc + kv_bytes);
  g->Hc = g->Qc = 0;
  g->total = g->bias;
  if (bias_sizes != nullptr) {
    if (bias_sizes[1] != H && bias_sizes[1] != KVH && bias_sizes[1] != 1)
      return fail(SMA_ERR_INVALID_ARG, "bias head dim must be %d, %d or 1", H, KVH);
    if (bias_sizes[2] != Lq && bias_sizes[2] != 1)
      return fail(SMA_ERR_INVALID_ARG, "bias query dim must be %d or 1", Lq);
    g->Hc = bias_sizes[1] == H ? H : KVH;
    g->Qc = static_cast<int>(bias_sizes[2]);
    g->total = align256(g->bias + static_cast<size_t>(B) * g->Hc * g->Qc * g->cap *
                                      elem_size(bias_dtype));
  }
  g->kv_split = split_layout(g->total, B, H, KVH, Lq, d, g->QT, g->KT, g->LH > 1 ? 1 : 0,
                             kPolicyGather);
  g->total = g->kv_split.end;
  return SMA_OK;
}

}  // namespace

int sma::set_last_error(int code, const char* message) {
  g_last_error = message;
  return code;
}

extern "C" {

const char* sma_last_error(void) { return g_last_error.c_str(); }

int32_t sma_abi_version(void) { return 1; }

sma_status sma_device_status(void* stream, int32_t* device_error) {
  if (device_error == nullptr) return fail(SMA_ERR_INVALID_ARG, "device_error is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronisation failed");
  int* word = device_error_word(&e);
  if (word == nullptr) return cuda_fail(e, "device error word unavailable");
  int v = 0;
  e = cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word failed");
  const int zero = 0;
  e = cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word failed");
  *device_error = v;
  return ok();
}

sma_status sma_selftest_wait_timeout(int64_t timeout_ns, int64_t* dev_out, void* stream) {
  if (dev_out == nullptr) return fail(SMA_ERR_INVALID_ARG, "dev_out is NULL");
  if (timeout_ns < 1000000 || timeout_ns > 2000000000)
    return fail(SMA_ERR_INVALID_ARG, "timeout_ns must be in [1 ms, 2 s]");
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  e = launch_wait_timeout_selftest(static_cast<uint64_t>(timeout_ns), err, dev_out,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch failed");
  return ok();
}

sma_status dfa_block_map_dims(const dfa_mask_desc* desc, int32_t* q_tiles, int32_t* kv_tiles) {
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  if (q_tiles == nullptr || kv_tiles == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "output pointers are NULL");
  const DflashGeom g = make_geom(desc);
  *q_tiles = g.QT;
  *kv_tiles = g.KT;
  return ok();
}

sma_status dfa_block_map(const dfa_mask_desc* desc, const int32_t* anchors, int32_t* num_full,
                         int32_t* full_idx, int32_t* num_part, int32_t* part_idx, void* stream) {
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  if (!anchors || !num_full || !full_idx || !num_part || !part_idx)
    return fail(SMA_ERR_INVALID_ARG, "a device pointer is NULL");
  const DflashGeom g = make_geom(desc);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  e = launch_dfa_block_map(g, anchors, num_full, full_idx, num_part, part_idx, err,
                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block map launch failed");
  return ok();
}

}  // extern "C"

namespace sma {
// Bytes of the DFlash forward's block map in its workspace (the minimum
// workspace of dfa_attn_fwd without a block map).
size_t dfa_fwd_map_bytes(const dfa_mask_desc* desc) {
  const DflashGeom g = make_geom(desc);
  return lists_layout(0, static_cast<int64_t>(g.B) * g.QT, g.KT).end;
}
}  // namespace sma

extern "C" {

sma_status dfa_attn_fwd_workspace_size(const dfa_mask_desc* desc, int32_t heads, int32_t kv_heads,
                                       int32_t head_dim, size_t* bytes) {
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  const DflashGeom g = make_geom(desc);
  const ListsLayout lay = lists_layout(0, static_cast<int64_t>(g.B) * g.QT, g.KT);
  *bytes = split_layout(lay.end, g.B, heads, kv_heads, g.Nq, head_dim, g.QT, g.KT, 0, kPolicyDflash).end;
  return ok();
}

sma_status dfa_attn_fwd(const dfa_mask_desc* desc, const int32_t* anchors, int32_t dtype,
                        int32_t heads, int32_t kv_heads, int32_t head_dim, float scale,
                        const void* q, const int64_t q_strides[3], const void* k,
                        const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                        void* out, const int64_t o_strides[3], float* lse,
                        const dfa_block_map_ptrs* block_map, void* workspace,
                        size_t workspace_bytes, void* stream) {
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (anchors == nullptr) return fail(SMA_ERR_INVALID_ARG, "anchors is NULL");
  const DflashGeom g = make_geom(desc);
  if ((s = check_operand("q", q, q_strides, dtype, g.Nq)) != SMA_OK) return s;
  if ((s = check_operand("k", k, k_strides, dtype, g.Lk)) != SMA_OK) return s;
  if ((s = check_operand("v", v, v_strides, dtype, g.Lk)) != SMA_OK) return s;
  if ((s = check_operand("out", out, o_strides, dtype, g.Nq)) != SMA_OK) return s;
  const ListsLayout lay = lists_layout(0, static_cast<int64_t>(g.B) * g.QT, g.KT);
  const SplitLayout sp = split_layout(lay.end, g.B, heads, kv_heads, g.Nq, head_dim, g.QT, g.KT, 0, kPolicyDflash);
  // The workspace must hold the block map (unless one is given); the
  // key-range split runs only when it also holds the split's partial results.
  if (block_map != nullptr) {
    if (!block_map->num_full || !block_map->full_idx || !block_map->num_part || !block_map->part_idx)
      return fail(SMA_ERR_INVALID_ARG, "block_map has a NULL pointer");
  } else if ((s = check_workspace(workspace, workspace_bytes, lay.end)) != SMA_OK) {
    return s;
  }
  const bool split_ok = workspace != nullptr && workspace_bytes >= sp.end &&
                        (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  const int32_t *nf, *np, *fi, *pi;
  if (block_map != nullptr) {
    nf = block_map->num_full;
    np = block_map->num_part;
    fi = block_map->full_idx;
    pi = block_map->part_idx;
  } else {
    int32_t* wnf = at<int32_t>(workspace, lay.nf);
    int32_t* wnp = at<int32_t>(workspace, lay.np);
    int32_t* wfi = at<int32_t>(workspace, lay.fi);
    int32_t* wpi = at<int32_t>(workspace, lay.pi);
    e = launch_dfa_block_map(g, anchors, wnf, wfi, wnp, wpi, err, st);
    if (e != cudaSuccess) return cuda_fail(e, "block map launch failed");
    nf = wnf; np = wnp; fi = wfi; pi = wpi;
  }

  AttnProblem p{};
  p.dtype = dtype;
  p.B = g.B; p.H = heads; p.KVH = kv_heads; p.Lq = g.Nq; p.Lk = g.Lk; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = (p.group + 1) / 2;
  p.QT = g.QT; p.KT = g.KT;
  p.scale_log2 = resolve_scale(scale, head_dim) * kLog2eHost;
  p.q = q; p.q_sb = q_strides[0]; p.q_sr = q_strides[1]; p.q_sh = q_strides[2];
  p.k = k; p.k_sb = k_strides[0]; p.k_sr = k_strides[1]; p.k_sh = k_strides[2];
  p.v = v; p.v_sb = v_strides[0]; p.v_sr = v_strides[1]; p.v_sh = v_strides[2];
  p.o = out; p.o_sb = o_strides[0]; p.o_sr = o_strides[1]; p.o_sh = o_strides[2];
  p.lse = lse;
  p.lists.num_full = nf; p.lists.full_idx = fi; p.lists.num_part = np; p.lists.part_idx = pi;
  p.lists.LB = g.B; p.lists.LH = 1; p.lists.head_mode = 0;
  p.policy = kPolicyDflash;
  p.anchors = anchors; p.N = g.N; p.bs = g.bs; p.Lc = g.Lc;
  p.causal_in_block = g.causal; p.window = g.window;
  p.err = err;
  if (split_ok) apply_split(p, sp, workspace);
  if (dtype == SMA_FP32) {
    e = launch_attn_simt(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch failed");
    return ok();
  }
  char msg[256];
  const int rc = launch_attn_tc(p, st, msg, sizeof(msg));
  if (rc != SMA_OK) return fail(rc, "%s", msg);
  return ok();
}

sma_status mask_tile_summary(const uint8_t* mask, const int64_t mask_sizes[4],
                             const int64_t mask_strides[4], int32_t k_len, uint8_t* codes,
                             void* stream) {
  if (mask == nullptr || codes == nullptr) return fail(SMA_ERR_INVALID_ARG, "NULL pointer");
  if (k_len < 1) return fail(SMA_ERR_INVALID_ARG, "k_len must be >= 1");
  if (mask_sizes == nullptr || mask_strides == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "mask sizes/strides are NULL");
  for (int i = 0; i < 3; ++i)
    if (mask_sizes[i] < 1) return fail(SMA_ERR_INVALID_ARG, "mask dims must be >= 1");
  AuxView view;
  // Shape checks that involve B/H/Lq do not apply here; use the mask's own dims.
  sma_status s = check_aux("mask", mask, mask_sizes, mask_strides, 1,
                           static_cast<int32_t>(mask_sizes[0]), static_cast<int32_t>(mask_sizes[1]),
                           static_cast<int32_t>(mask_sizes[1]), static_cast<int32_t>(mask_sizes[2]),
                           k_len, true, &view);
  if (s != SMA_OK) return s;
  const int64_t folded[4] = {view.sb, view.sh, view.sq, 1};
  cudaError_t e = launch_mask_tile_summary(mask, mask_sizes, folded, k_len, codes,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mask summary launch failed");
  return ok();
}

sma_status masked_attn_fwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                          int32_t q_len, int32_t k_len, int32_t head_dim,
                                          const int64_t mask_sizes[4], size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  *bytes = masked_geom(batch, heads, kv_heads, q_len, k_len, head_dim, mask_sizes).total;
  return ok();
}

sma_status masked_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                           int32_t is_causal, const void* q, const int64_t q_strides[3],
                           const void* k, const int64_t k_strides[3], const void* v,
                           const int64_t v_strides[3], const uint8_t* mask,
                           const int64_t mask_sizes[4], const int64_t mask_strides[4],
                           const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                           const int64_t bias_strides[4], void* out, const int64_t o_strides[3],
                           float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  if (is_causal != 0 && is_causal != 1) return fail(SMA_ERR_INVALID_ARG, "is_causal must be 0 or 1");
  if ((s = check_operand("q", q, q_strides, dtype, q_len)) != SMA_OK) return s;
  if ((s = check_operand("k", k, k_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_operand("v", v, v_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_operand("out", out, o_strides, dtype, q_len)) != SMA_OK) return s;
  AuxView mview, bview;
  const bool has_mask = mask != nullptr, has_bias = bias != nullptr;
  if (has_mask && (s = check_aux("mask", mask, mask_sizes, mask_strides, 1, batch, heads, kv_heads,
                                 q_len, k_len, true, &mview)) != SMA_OK)
    return s;
  if (has_bias) {
    if (!valid_dtype(bias_dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", bias_dtype);
    if ((s = check_aux("bias", bias, bias_sizes, bias_strides, elem_size(bias_dtype), batch, heads,
                       kv_heads, q_len, k_len, true, &bview)) != SMA_OK)
      return s;
    bview.dtype = bias_dtype;
  }
  const MaskedGeom mg =
      masked_geom(batch, heads, kv_heads, q_len, k_len, head_dim, has_mask ? mask_sizes : nullptr);
  if ((s = check_workspace(workspace, workspace_bytes, mg.total)) != SMA_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  const float scale_log2 = resolve_scale(scale, head_dim) * kLog2eHost;

  if (mg.decode) {
    // PR #190 swapped path: rows of one problem are the query heads of a KV head.
    DecodeProblem dp{};
    dp.dtype = dtype;
    dp.B = batch; dp.H = heads; dp.KVH = kv_heads; dp.Lk = k_len; dp.d = head_dim;
    dp.Kpad = static_cast<int>(round_up(k_len, kTile));
    dp.group = heads / kv_heads;
    dp.scale_log2 = scale_log2;
    dp.q = q; dp.q_sb = q_strides[0]; dp.q_sh = q_strides[2];
    dp.k = k; dp.k_sb = k_strides[0]; dp.k_sr = k_strides[1]; dp.k_sh = k_strides[2];
    dp.v = v; dp.v_sb = v_strides[0]; dp.v_sr = v_strides[1]; dp.v_sh = v_strides[2];
    dp.o = out; dp.o_sb = o_strides[0]; dp.o_sh = o_strides[2];
    dp.lse = lse;
    dp.has_mask = has_mask; dp.has_bias = has_bias;
    if (has_mask) dp.mask = mview;
    if (has_bias) dp.bias = bview;
    dp.splits = mg.splits;
    dp.chunk = mg.chunk;
    dp.part_o = at<float>(workspace, mg.part_o);
    dp.part_ml = at<float>(workspace, mg.part_ml);
    dp.err = err;
    e = launch_decode(dp, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch failed");
    return ok();
  }

  AttnProblem p{};
  p.dtype = dtype;
  p.B = batch; p.H = heads; p.KVH = kv_heads; p.Lq = q_len; p.Lk = k_len; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = mg.npairs;
  p.QT = mg.QT; p.KT = mg.KT;
  p.scale_log2 = scale_log2;
  p.q = q; p.q_sb = q_strides[0]; p.q_sr = q_strides[1]; p.q_sh = q_strides[2];
  p.k = k; p.k_sb = k_strides[0]; p.k_sr = k_strides[1]; p.k_sh = k_strides[2];
  p.v = v; p.v_sb = v_strides[0]; p.v_sr = v_strides[1]; p.v_sh = v_strides[2];
  p.o = out; p.o_sb = o_strides[0]; p.o_sr = o_strides[1]; p.o_sh = o_strides[2];
  p.lse = lse;
  p.policy = kPolicyExplicit;
  p.causal = is_causal;
  p.has_mask = has_mask;
  p.has_bias = has_bias;
  if (has_mask) p.mask = mview;
  if (has_bias) p.bias = bview;
  p.err = err;
  p.lists.LB = mg.LB;
  p.lists.LH = mg.LH;
  p.lists.head_mode = mg.head_mode;
  p.lists.num_full = at<int32_t>(workspace, mg.lists.nf);
  p.lists.num_part = at<int32_t>(workspace, mg.lists.np);
  p.lists.full_idx = at<int32_t>(workspace, mg.lists.fi);
  p.lists.part_idx = at<int32_t>(workspace, mg.lists.pi);
  apply_split(p, mg.kv_split, workspace);
  uint8_t* codes = has_mask ? at<uint8_t>(workspace, 0) : nullptr;
  if (has_mask) {
    const int64_t folded[4] = {mview.sb, mview.sh, mview.sq, 1};
    e = launch_mask_tile_summary(mask, mask_sizes, folded, k_len, codes, st);
    if (e != cudaSuccess) return cuda_fail(e, "mask summary launch failed");
  }
  e = launch_explicit_lists(p, codes, mg.codes_qt, at<int32_t>(workspace, mg.lists.nf),
                            at<int32_t>(workspace, mg.lists.fi), at<int32_t>(workspace, mg.lists.np),
                            at<int32_t>(workspace, mg.lists.pi), st);
  if (e != cudaSuccess) return cuda_fail(e, "tile list launch failed");
  if (dtype == SMA_FP32) {
    e = launch_attn_simt(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch failed");
    return ok();
  }
  char msg[256];
  const int rc = launch_attn_tc(p, st, msg, sizeof(msg));
  if (rc != SMA_OK) return fail(rc, "%s", msg);
  return ok();
}

sma_status dynamic_topk_mask(int32_t bias_dtype, const void* bias, const int64_t bias_sizes[4],
                             const int64_t bias_strides[4], int32_t k_len, const uint8_t* pre_mask,
                             const int64_t pre_mask_sizes[4], const int64_t pre_mask_strides[4],
                             int32_t window_size, uint8_t* out_mask, void* stream) {
  if (!valid_dtype(bias_dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", bias_dtype);
  if (bias == nullptr || out_mask == nullptr) return fail(SMA_ERR_INVALID_ARG, "NULL pointer");
  if (bias_sizes == nullptr || bias_strides == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "bias sizes/strides are NULL");
  if (k_len < 1) return fail(SMA_ERR_INVALID_ARG, "k_len must be >= 1");
  if (window_size < 1) return fail(SMA_ERR_INVALID_ARG, "window_size must be >= 1");
  for (int i = 0; i < 3; ++i)
    if (bias_sizes[i] < 1) return fail(SMA_ERR_INVALID_ARG, "bias dims must be >= 1");
  const int64_t kpad = round_up(k_len, kTile);
  // The padded key dim of PR #190's contract, or the true key length.  A key
  // dim of 1 (one value for every key) would rank every key equal; its
  // output would not have one column per key, so it is refused.
  if (bias_sizes[3] != kpad && bias_sizes[3] != k_len)
    return fail(SMA_ERR_INVALID_ARG,
                "bias key dim must be round_up(k_len, 128) = %lld or k_len = %d (the output mask "
                "has one column per key of the bias)",
                static_cast<long long>(kpad), k_len);
  if (bias_strides[3] != 1) return fail(SMA_ERR_INVALID_ARG, "bias last dim must be contiguous");
  if (!aligned16(bias)) return fail(SMA_ERR_INVALID_ARG, "bias must be 16-byte aligned");
  const int es = elem_size(bias_dtype);
  TopkProblem p{};
  p.bias_dtype = bias_dtype;
  p.bias = bias;
  for (int i = 0; i < 4; ++i) {
    p.b_sizes[i] = bias_sizes[i];
    p.b_strides[i] = (i < 3 && bias_sizes[i] == 1) ? 0 : bias_strides[i];
    if (p.b_strides[i] < 0 || (i < 3 && (p.b_strides[i] * es) % 16 != 0))
      return fail(SMA_ERR_INVALID_ARG, "bias strides must be non-negative multiples of 16 bytes");
  }
  p.Lk = k_len;
  p.Kcols = static_cast<int>(bias_sizes[3]);
  p.pre = pre_mask;
  if (pre_mask != nullptr) {
    if (pre_mask_sizes == nullptr || pre_mask_strides == nullptr)
      return fail(SMA_ERR_INVALID_ARG, "pre_mask sizes/strides are NULL");
    for (int i = 0; i < 3; ++i) {
      if (pre_mask_sizes[i] != 1 && pre_mask_sizes[i] != bias_sizes[i])
        return fail(SMA_ERR_INVALID_ARG, "pre_mask dim %d must be 1 or %lld", i,
                    static_cast<long long>(bias_sizes[i]));
    }
    if (pre_mask_sizes[3] < 1) return fail(SMA_ERR_INVALID_ARG, "pre_mask key dim must be >= 1");
    if (pre_mask_strides[3] != 1)
      return fail(SMA_ERR_INVALID_ARG, "pre_mask last dim must be contiguous");
    for (int i = 0; i < 4; ++i) {
      p.p_sizes[i] = pre_mask_sizes[i];
      p.p_strides[i] = (i < 3 && pre_mask_sizes[i] == 1) ? 0 : pre_mask_strides[i];
      if (p.p_strides[i] < 0) return fail(SMA_ERR_INVALID_ARG, "pre_mask strides must be >= 0");
    }
  }
  p.window = window_size;
  p.out = out_mask;
  if ((reinterpret_cast<uintptr_t>(out_mask) & 7u) != 0)
    return fail(SMA_ERR_INVALID_ARG, "out_mask must be 8-byte aligned");
  cudaError_t e = launch_topk(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch failed");
  return ok();
}

sma_status sparse_attn_fwd_workspace_size(int32_t dtype, int32_t batch, int32_t heads,
                                          int32_t kv_heads, int32_t q_len, int32_t k_len,
                                          int32_t head_dim, const int64_t mask_sizes[4],
                                          int32_t bias_dtype, const int64_t bias_sizes[4],
                                          int32_t max_keys, size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (bias_sizes != nullptr && !valid_dtype(bias_dtype))
    return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", bias_dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  SparseGeom g;
  if ((s = sparse_geom(dtype, batch, heads, kv_heads, q_len, k_len, head_dim, mask_sizes, bias_dtype,
                       bias_sizes, max_keys, &g)) != SMA_OK)
    return s;
  *bytes = g.total;
  return ok();
}

sma_status sparse_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                           int32_t is_causal, const void* q, const int64_t q_strides[3],
                           const void* k, const int64_t k_strides[3], const void* v,
                           const int64_t v_strides[3], const uint8_t* mask,
                           const int64_t mask_sizes[4], const int64_t mask_strides[4],
                           const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                           const int64_t bias_strides[4], int32_t max_keys, void* out,
                           const int64_t o_strides[3], float* lse, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  if (is_causal != 0 && is_causal != 1) return fail(SMA_ERR_INVALID_ARG, "is_causal must be 0 or 1");
  if ((s = check_operand("q", q, q_strides, dtype, q_len)) != SMA_OK) return s;
  if ((s = check_operand("k", k, k_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_operand("v", v, v_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_operand("out", out, o_strides, dtype, q_len)) != SMA_OK) return s;
  if (mask == nullptr) return fail(SMA_ERR_INVALID_ARG, "the index-gather path needs a mask");
  AuxView mview, bview;
  if ((s = check_aux("mask", mask, mask_sizes, mask_strides, 1, batch, heads, kv_heads, q_len, k_len,
                     true, &mview)) != SMA_OK)
    return s;
  const bool has_bias = bias != nullptr;
  if (has_bias) {
    if (!valid_dtype(bias_dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", bias_dtype);
    if ((s = check_aux("bias", bias, bias_sizes, bias_strides, elem_size(bias_dtype), batch, heads,
                       kv_heads, q_len, k_len, true, &bview)) != SMA_OK)
      return s;
    bview.dtype = bias_dtype;
  }
  SparseGeom g;
  if ((s = sparse_geom(dtype, batch, heads, kv_heads, q_len, k_len, head_dim, mask_sizes, bias_dtype,
                       has_bias ? bias_sizes : nullptr, max_keys, &g)) != SMA_OK)
    return s;
  if ((s = check_workspace(workspace, workspace_bytes, g.total)) != SMA_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");

  AttnProblem p{};
  p.dtype = dtype;
  p.B = batch; p.H = heads; p.KVH = kv_heads; p.Lq = q_len; p.Lk = g.cap; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = (p.group + 1) / 2;
  p.QT = g.QT; p.KT = g.KT;
  p.scale_log2 = resolve_scale(scale, head_dim) * kLog2eHost;
  p.q = q; p.q_sb = q_strides[0]; p.q_sr = q_strides[1]; p.q_sh = q_strides[2];
  // compacted K / V: [batch, cap, kv_heads, head_dim] contiguous
  p.k = at<uint8_t>(workspace, g.kc);
  p.v = at<uint8_t>(workspace, g.vc);
  p.k_sh = p.v_sh = head_dim;
  p.k_sr = p.v_sr = static_cast<int64_t>(kv_heads) * head_dim;
  p.k_sb = p.v_sb = static_cast<int64_t>(g.cap) * kv_heads * head_dim;
  p.o = out; p.o_sb = o_strides[0]; p.o_sr = o_strides[1]; p.o_sh = o_strides[2];
  p.lse = lse;
  p.policy = kPolicyGather;
  p.causal = 1;  // every PARTIAL tile is cut by its row's limit
  p.has_mask = 0;
  p.has_bias = has_bias;
  p.err = err;
  p.lists.LB = g.LB;
  p.lists.LH = g.LH;
  p.lists.head_mode = g.LH > 1 ? 1 : 0;
  p.lists.num_full = at<int32_t>(workspace, g.lists.nf);
  p.lists.num_part = at<int32_t>(workspace, g.lists.np);
  p.lists.full_idx = at<int32_t>(workspace, g.lists.fi);
  p.lists.part_idx = at<int32_t>(workspace, g.lists.pi);
  int32_t* idx = at<int32_t>(workspace, g.idx);
  int32_t* count = at<int32_t>(workspace, g.count);
  p.gather.idx = idx;
  p.gather.count = count;
  p.gather.cap = g.cap;
  p.gather.k_len = k_len;
  p.gather.causal = is_causal;
  apply_split(p, g.kv_split, workspace);
  if (has_bias) {
    AuxView cb;
    cb.ptr = at<uint8_t>(workspace, g.bias);
    cb.dtype = bias_dtype;
    cb.sq = g.Qc > 1 ? g.cap : 0;
    cb.sh = static_cast<int64_t>(g.Qc) * g.cap;
    cb.sb = static_cast<int64_t>(g.Hc) * g.Qc * g.cap;
    cb.head_per_query = g.Hc == heads && bview.head_per_query ? 1 : 0;
    cb.kd = g.cap;  // compacted rows hold every column up to cap
    p.bias = cb;
  }

  e = launch_select_keys(mask, mview.sb, mview.sh, mview.kd, g.LB, g.LH, k_len, g.cap, idx, count,
                         err, st);
  if (e != cudaSuccess) return cuda_fail(e, "key selection launch failed");
  e = launch_gather_kv(p, k, k_strides, v, v_strides, st);
  if (e != cudaSuccess) return cuda_fail(e, "K/V gather launch failed");
  if (has_bias) {
    e = launch_gather_bias(p, bview, g.Hc, g.Qc, st);
    if (e != cudaSuccess) return cuda_fail(e, "bias gather launch failed");
  }
  e = launch_gather_lists(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "tile list launch failed");
  if (dtype == SMA_FP32) {
    e = launch_attn_simt(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch failed");
    return ok();
  }
  char msg[256];
  const int rc = launch_attn_tc(p, st, msg, sizeof(msg));
  if (rc != SMA_OK) return fail(rc, "%s", msg);
  return ok();
}

sma_status dfa_attn_bwd_workspace_size(const dfa_mask_desc* desc, int32_t heads, int32_t kv_heads,
                                       int32_t head_dim, size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  if ((s = check_heads(heads, kv_heads, head_dim)) != SMA_OK) return s;
  const DflashGeom g = make_geom(desc);
  *bytes = bwd_layout(0, g.B, g.QT, g.KT, g.B, heads, g.Nq, head_dim).total;
  return ok();
}

sma_status dfa_attn_bwd(const dfa_mask_desc* desc, const int32_t* anchors, int32_t dtype,
                        int32_t heads, int32_t kv_heads, int32_t head_dim, float scale,
                        const void* q, const int64_t q_strides[3], const void* k,
                        const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                        const void* out, const int64_t o_strides[3], const float* lse,
                        const void* dout, const int64_t do_strides[3], void* dq,
                        const int64_t dq_strides[3], void* dk, const int64_t dk_strides[3],
                        void* dv, const int64_t dv_strides[3], void* workspace,
                        size_t workspace_bytes, void* stream) {
  sma_status s = check_desc(desc);
  if (s != SMA_OK) return s;
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if ((s = check_heads(heads, kv_heads, head_dim)) != SMA_OK) return s;
  if (anchors == nullptr) return fail(SMA_ERR_INVALID_ARG, "anchors is NULL");
  const DflashGeom g = make_geom(desc);
  if ((s = check_operand("q", q, q_strides, dtype, g.Nq)) != SMA_OK) return s;
  if ((s = check_operand("k", k, k_strides, dtype, g.Lk)) != SMA_OK) return s;
  if ((s = check_operand("v", v, v_strides, dtype, g.Lk)) != SMA_OK) return s;
  if ((s = check_grad_operands(dtype, g.Nq, g.Lk, out, o_strides, lse, dout, do_strides, dq,
                               dq_strides, dk, dk_strides, dv, dv_strides)) != SMA_OK)
    return s;
  const BwdLayout lay = bwd_layout(0, g.B, g.QT, g.KT, g.B, heads, g.Nq, head_dim);
  if ((s = check_workspace(workspace, workspace_bytes, lay.total)) != SMA_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  int32_t* nf = at<int32_t>(workspace, lay.fl.nf);
  int32_t* np = at<int32_t>(workspace, lay.fl.np);
  int32_t* fi = at<int32_t>(workspace, lay.fl.fi);
  int32_t* pi = at<int32_t>(workspace, lay.fl.pi);
  e = launch_dfa_block_map(g, anchors, nf, fi, np, pi, err, st);
  if (e != cudaSuccess) return cuda_fail(e, "block map launch failed");

  BwdProblem b{};
  AttnProblem& p = b.f;
  p.dtype = dtype;
  p.B = g.B; p.H = heads; p.KVH = kv_heads; p.Lq = g.Nq; p.Lk = g.Lk; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = (p.group + 1) / 2;
  p.QT = g.QT; p.KT = g.KT;
  const float sc = resolve_scale(scale, head_dim);
  p.scale_log2 = sc * kLog2eHost;
  p.q = q; p.q_sb = q_strides[0]; p.q_sr = q_strides[1]; p.q_sh = q_strides[2];
  p.k = k; p.k_sb = k_strides[0]; p.k_sr = k_strides[1]; p.k_sh = k_strides[2];
  p.v = v; p.v_sb = v_strides[0]; p.v_sr = v_strides[1]; p.v_sh = v_strides[2];
  p.o = const_cast<void*>(out); p.o_sb = o_strides[0]; p.o_sr = o_strides[1]; p.o_sh = o_strides[2];
  p.lse = const_cast<float*>(lse);
  p.lists.num_full = nf; p.lists.full_idx = fi; p.lists.num_part = np; p.lists.part_idx = pi;
  p.lists.LB = g.B; p.lists.LH = 1; p.lists.head_mode = 0;
  p.policy = kPolicyDflash;
  p.anchors = anchors; p.N = g.N; p.bs = g.bs; p.Lc = g.Lc;
  p.causal_in_block = g.causal; p.window = g.window;
  p.err = err;
  set_grads(b, dout, do_strides, dq, dq_strides, dk, dk_strides, dv, dv_strides, sc);
  if ((s = run_backward(b, workspace, lay, st)) != SMA_OK) return s;
  return ok();
}

sma_status masked_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                          int32_t q_len, int32_t k_len, int32_t head_dim,
                                          const int64_t mask_sizes[4], size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  // the prefill geometry (tile lists), whatever q_len is
  const MaskedGeom mg = masked_geom(batch, heads, kv_heads, q_len < 2 ? 2 : q_len, k_len, head_dim,
                                    mask_sizes);
  const int QT = static_cast<int>(ceil_div(q_len, kTile));
  const int KT = static_cast<int>(ceil_div(k_len, kTile));
  *bytes = bwd_layout(mg.codes_bytes, static_cast<int64_t>(mg.LB) * mg.LH, QT, KT, batch, heads,
                      q_len, head_dim).total;
  return ok();
}

// Partial buffer of the fixed-order dbias: [batch, heads, R, kd] fp32, R the
// partial rows per (batch, head): the query rows (a bias with a query dim, or
// the fp32 kernels, which store per element), else one row per group of
// dbias_group_rows(head_dim) queries.  0 bytes where every dbias element
// already has a single writer (a bias with its own element for each
// (batch, head, query)).
struct DetDbias {
  int R = 0;
  size_t bytes = 0;
};
static DetDbias det_dbias_layout(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                                 int32_t q_len, int32_t head_dim, const int64_t bias_sizes[4]) {
  DetDbias d;
  const int64_t nb = bias_sizes[0], nh = bias_sizes[1], nq = bias_sizes[2], kd = bias_sizes[3];
  const int group = heads / kv_heads;
  const bool own_head = heads == 1 || (nh > 1 && (nh == heads || group == 1));
  const bool own_batch = batch == 1 || nb > 1;
  if (nq > 1 && own_head && own_batch) return d;
  const int G = dbias_group_rows(head_dim);
  d.R = (nq > 1 || dtype == SMA_FP32) ? q_len : static_cast<int>(ceil_div(q_len, G));
  d.bytes = static_cast<size_t>(batch) * heads * d.R * kd * 4;
  return d;
}

sma_status masked_attn_bwd_dbias_workspace_size(int32_t dtype, int32_t batch, int32_t heads,
                                                int32_t kv_heads, int32_t q_len, int32_t head_dim,
                                                const int64_t bias_sizes[4], size_t* bytes) {
  if (bytes == nullptr || bias_sizes == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "bias_sizes / bytes is NULL");
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1) return fail(SMA_ERR_INVALID_ARG, "batch and q_len must be >= 1");
  for (int i = 0; i < 4; ++i)
    if (bias_sizes[i] < 1) return fail(SMA_ERR_INVALID_ARG, "bias sizes must be >= 1");
  *bytes = det_dbias_layout(dtype, batch, heads, kv_heads, q_len, head_dim, bias_sizes).bytes;
  return ok();
}

static sma_status masked_bwd_impl(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                                  int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                                  int32_t is_causal, const void* q, const int64_t q_strides[3],
                                  const void* k, const int64_t k_strides[3], const void* v,
                                  const int64_t v_strides[3], const uint8_t* mask,
                                  const int64_t mask_sizes[4], const int64_t mask_strides[4],
                                  const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                                  const int64_t bias_strides[4], const void* out,
                                  const int64_t o_strides[3], const float* lse, const void* dout,
                                  const int64_t do_strides[3], void* dq, const int64_t dq_strides[3],
                                  void* dk, const int64_t dk_strides[3], void* dv,
                                  const int64_t dv_strides[3], float* dbias, void* workspace,
                                  size_t workspace_bytes, bool deterministic, void* det_ws,
                                  size_t det_bytes, void* stream) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || q_len < 1 || k_len < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, q_len and k_len must be >= 1");
  if (is_causal != 0 && is_causal != 1) return fail(SMA_ERR_INVALID_ARG, "is_causal must be 0 or 1");
  if (dbias != nullptr && bias == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "dbias needs the bias (it takes the bias's shape)");
  if (dbias != nullptr && (reinterpret_cast<uintptr_t>(dbias) & 15u) != 0)
    return fail(SMA_ERR_INVALID_ARG, "dbias must be 16-byte aligned");
  if ((s = check_operand("q", q, q_strides, dtype, q_len)) != SMA_OK) return s;
  if ((s = check_operand("k", k, k_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_operand("v", v, v_strides, dtype, k_len)) != SMA_OK) return s;
  if ((s = check_grad_operands(dtype, q_len, k_len, out, o_strides, lse, dout, do_strides, dq,
                               dq_strides, dk, dk_strides, dv, dv_strides)) != SMA_OK)
    return s;
  AuxView mview, bview;
  const bool has_mask = mask != nullptr, has_bias = bias != nullptr;
  if (has_mask && (s = check_aux("mask", mask, mask_sizes, mask_strides, 1, batch, heads, kv_heads,
                                 q_len, k_len, true, &mview)) != SMA_OK)
    return s;
  if (has_bias) {
    if (!valid_dtype(bias_dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", bias_dtype);
    if ((s = check_aux("bias", bias, bias_sizes, bias_strides, elem_size(bias_dtype), batch, heads,
                       kv_heads, q_len, k_len, true, &bview)) != SMA_OK)
      return s;
    bview.dtype = bias_dtype;
  }
  const MaskedGeom mg = masked_geom(batch, heads, kv_heads, q_len < 2 ? 2 : q_len, k_len, head_dim,
                                    has_mask ? mask_sizes : nullptr);
  const int QT = static_cast<int>(ceil_div(q_len, kTile));
  const int KT = static_cast<int>(ceil_div(k_len, kTile));
  const BwdLayout lay = bwd_layout(mg.codes_bytes, static_cast<int64_t>(mg.LB) * mg.LH, QT, KT,
                                   batch, heads, q_len, head_dim);
  if ((s = check_workspace(workspace, workspace_bytes, lay.total)) != SMA_OK) return s;
  // fixed-order dbias partials (0 bytes: not used; a bias with a key dim of
  // 1 has the zero gradient, written without them)
  DetDbias det;
  if (deterministic && dbias != nullptr && bias != nullptr && (bias_sizes[3] > 1 || k_len == 1)) {
    det = det_dbias_layout(dtype, batch, heads, kv_heads, q_len, head_dim, bias_sizes);
    if ((s = check_workspace(det_ws, det_bytes, det.bytes)) != SMA_OK) return s;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  BwdProblem b{};
  AttnProblem& p = b.f;
  p.dtype = dtype;
  p.B = batch; p.H = heads; p.KVH = kv_heads; p.Lq = q_len; p.Lk = k_len; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = mg.npairs;
  p.QT = QT; p.KT = KT;
  const float sc = resolve_scale(scale, head_dim);
  p.scale_log2 = sc * kLog2eHost;
  p.q = q; p.q_sb = q_strides[0]; p.q_sr = q_strides[1]; p.q_sh = q_strides[2];
  p.k = k; p.k_sb = k_strides[0]; p.k_sr = k_strides[1]; p.k_sh = k_strides[2];
  p.v = v; p.v_sb = v_strides[0]; p.v_sr = v_strides[1]; p.v_sh = v_strides[2];
  p.o = const_cast<void*>(out); p.o_sb = o_strides[0]; p.o_sr = o_strides[1]; p.o_sh = o_strides[2];
  p.lse = const_cast<float*>(lse);
  p.policy = kPolicyExplicit;
  p.causal = is_causal;
  p.has_mask = has_mask;
  p.has_bias = has_bias;
  if (has_mask) p.mask = mview;
  if (has_bias) p.bias = bview;
  p.err = err;
  p.lists.LB = mg.LB;
  p.lists.LH = mg.LH;
  p.lists.head_mode = mg.head_mode;
  int32_t* nf = at<int32_t>(workspace, lay.fl.nf);
  int32_t* np = at<int32_t>(workspace, lay.fl.np);
  int32_t* fi = at<int32_t>(workspace, lay.fl.fi);
  int32_t* pi = at<int32_t>(workspace, lay.fl.pi);
  p.lists.num_full = nf; p.lists.num_part = np; p.lists.full_idx = fi; p.lists.part_idx = pi;
  uint8_t* codes = has_mask ? at<uint8_t>(workspace, 0) : nullptr;
  if (has_mask) {
    const int64_t folded[4] = {mview.sb, mview.sh, mview.sq, 1};
    e = launch_mask_tile_summary(mask, mask_sizes, folded, k_len, codes, st);
    if (e != cudaSuccess) return cuda_fail(e, "mask summary launch failed");
  }
  e = launch_explicit_lists(p, codes, mg.codes_qt, nf, fi, np, pi, st);
  if (e != cudaSuccess) return cuda_fail(e, "tile list launch failed");
  set_grads(b, dout, do_strides, dq, dq_strides, dk, dk_strides, dv, dv_strides, sc);
  if (dbias != nullptr) {
    // contiguous fp32 at the bias's sizes (b', h', q', kd), kd the bias's key
    // dim: round_up(Lk, 128), Lk, or 1
    const int64_t kd = bias_sizes[3];
    const int64_t nb = bias_sizes[0], nh = bias_sizes[1], nq = bias_sizes[2];
    e = cudaMemsetAsync(dbias, 0, static_cast<size_t>(nb * nh * nq * kd) * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "dbias zeroing failed");
    if (kd > 1 || k_len == 1) {
      b.dbias = dbias;
      b.db_sq = nq > 1 ? kd : 0;
      b.db_sh = nh > 1 ? nq * kd : 0;
      b.db_sb = nb > 1 ? nh * nq * kd : 0;
      b.db_kd = static_cast<int>(kd);
      // dbias has the bias's sizes: a head dim of `heads` is one row per
      // query head even where the bias itself is read with stride 0
      const int db_hpq = nh == heads ? 1 : 0;
      b.db_head_per_query = db_hpq;
      const bool own_head = heads == 1 || (nh > 1 && (db_hpq || p.group == 1));
      const bool own_batch = batch == 1 || nb > 1;
      b.db_mode = nq == 1 ? kDbiasRowSum : (own_head && own_batch ? kDbiasStore : kDbiasAdd);
      if (det.bytes > 0) {
        // every partial element has one writer; the reduce kernel then sums
        // the partials in a fixed order
        e = cudaMemsetAsync(det_ws, 0, det.bytes, st);
        if (e != cudaSuccess) return cuda_fail(e, "dbias partial zeroing failed");
        b.dbias = static_cast<float*>(det_ws);
        b.db_sq = kd;
        b.db_sh = static_cast<int64_t>(det.R) * kd;
        b.db_sb = static_cast<int64_t>(heads) * det.R * kd;
        b.db_head_per_query = 1;
        b.db_mode = nq == 1 && dtype != SMA_FP32 ? kDbiasGroupStore : kDbiasStore;
      }
    }
    // else: a bias with one value for every key adds the same amount to every
    // score of a row, which softmax ignores; its gradient, the sum of dS over
    // the row's keys, is exactly 0 (sum_k P (dP - D) = D - D), and the zeroed
    // dbias is the result.
  }
  if ((s = run_backward(b, workspace, lay, st)) != SMA_OK) return s;
  if (det.bytes > 0) {
    e = launch_dbias_reduce(static_cast<const float*>(det_ws), batch, heads, det.R, dbias,
                            static_cast<int>(bias_sizes[0]), static_cast<int>(bias_sizes[1]),
                            static_cast<int>(bias_sizes[2]), static_cast<int>(bias_sizes[3]), st);
    if (e != cudaSuccess) return cuda_fail(e, "dbias reduction launch failed");
  }
  return ok();
}

sma_status masked_attn_bwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                           int32_t is_causal, const void* q, const int64_t q_strides[3],
                           const void* k, const int64_t k_strides[3], const void* v,
                           const int64_t v_strides[3], const uint8_t* mask,
                           const int64_t mask_sizes[4], const int64_t mask_strides[4],
                           const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                           const int64_t bias_strides[4], const void* out,
                           const int64_t o_strides[3], const float* lse, const void* dout,
                           const int64_t do_strides[3], void* dq, const int64_t dq_strides[3],
                           void* dk, const int64_t dk_strides[3], void* dv,
                           const int64_t dv_strides[3], float* dbias, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return masked_bwd_impl(dtype, batch, heads, kv_heads, q_len, k_len, head_dim, scale, is_causal, q,
                         q_strides, k, k_strides, v, v_strides, mask, mask_sizes, mask_strides, bias,
                         bias_dtype, bias_sizes, bias_strides, out, o_strides, lse, dout, do_strides,
                         dq, dq_strides, dk, dk_strides, dv, dv_strides, dbias, workspace,
                         workspace_bytes, false, nullptr, 0, stream);
}

sma_status masked_attn_bwd_deterministic(
    int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads, int32_t q_len, int32_t k_len,
    int32_t head_dim, float scale, int32_t is_causal, const void* q, const int64_t q_strides[3],
    const void* k, const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
    const uint8_t* mask, const int64_t mask_sizes[4], const int64_t mask_strides[4],
    const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
    const int64_t bias_strides[4], const void* out, const int64_t o_strides[3], const float* lse,
    const void* dout, const int64_t do_strides[3], void* dq, const int64_t dq_strides[3], void* dk,
    const int64_t dk_strides[3], void* dv, const int64_t dv_strides[3], float* dbias,
    void* workspace, size_t workspace_bytes, void* dbias_workspace, size_t dbias_workspace_bytes,
    void* stream) {
  return masked_bwd_impl(dtype, batch, heads, kv_heads, q_len, k_len, head_dim, scale, is_causal, q,
                         q_strides, k, k_strides, v, v_strides, mask, mask_sizes, mask_strides, bias,
                         bias_dtype, bias_sizes, bias_strides, out, o_strides, lse, dout, do_strides,
                         dq, dq_strides, dk, dk_strides, dv, dv_strides, dbias, workspace,
                         workspace_bytes, true, dbias_workspace, dbias_workspace_bytes, stream);
}

// Mask / bias of a packed batch, in the padded per-sequence layout
// (b', h', q', kd) as masked_attn_fwd takes them for a [batch, max_q, ...,
// max_k] problem; rows and columns are sequence-local.  All NULL: none.
struct VarlenAux {
  const uint8_t* mask = nullptr;
  const int64_t* mask_sizes = nullptr;
  const int64_t* mask_strides = nullptr;
  const void* bias = nullptr;
  int32_t bias_dtype = 0;
  const int64_t* bias_sizes = nullptr;
  const int64_t* bias_strides = nullptr;
  float* dbias = nullptr;  // backward only
};

// List geometry of a packed batch: one list row per (sequence, list head,
// query tile); with a mask the list heads follow the mask's head dim as in
// masked_attn_fwd, and the tile codes of the mask lead the workspace.
struct VarlenLists {
  int LH = 1, head_mode = 0, codes_qt = 0;
  size_t codes_bytes = 0;
};
static VarlenLists varlen_lists_geom(int32_t batch, int32_t heads, int32_t kv_heads, int32_t max_q,
                                     int32_t max_k, int32_t head_dim, const int64_t* mask_sizes) {
  VarlenLists v;
  if (mask_sizes == nullptr) return v;
  const MaskedGeom mg = masked_geom(batch, heads, kv_heads, max_q < 2 ? 2 : max_q, max_k, head_dim,
                                    mask_sizes);
  v.LH = mg.LH;
  v.head_mode = mg.head_mode;
  v.codes_qt = mg.codes_qt;
  v.codes_bytes = mg.codes_bytes;
  return v;
}

// Validates the mask / bias of a packed batch against the padded
// per-sequence problem [batch, max_q, heads, max_k].
static sma_status check_varlen_aux(const VarlenAux& ax, int32_t batch, int32_t heads,
                                   int32_t kv_heads, int32_t max_q, int32_t max_k, AuxView* mview,
                                   AuxView* bview) {
  sma_status s;
  if (ax.mask != nullptr &&
      (s = check_aux("mask", ax.mask, ax.mask_sizes, ax.mask_strides, 1, batch, heads, kv_heads,
                     max_q, max_k, true, mview)) != SMA_OK)
    return s;
  if (ax.bias != nullptr) {
    if (!valid_dtype(ax.bias_dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown bias dtype %d", ax.bias_dtype);
    if ((s = check_aux("bias", ax.bias, ax.bias_sizes, ax.bias_strides, elem_size(ax.bias_dtype),
                       batch, heads, kv_heads, max_q, max_k, true, bview)) != SMA_OK)
      return s;
    bview->dtype = ax.bias_dtype;
  }
  return SMA_OK;
}

sma_status varlen_attn_fwd_workspace_size(int32_t batch, int32_t max_q, int32_t max_k, size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  if (batch < 1 || max_q < 1 || max_k < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, max_q and max_k must be >= 1");
  *bytes = lists_layout(0, static_cast<int64_t>(batch) * ceil_div(max_q, kTile),
                        static_cast<int>(ceil_div(max_k, kTile))).end;
  return ok();
}

// Tile lists of a packed batch: causal / length geometry per sequence, and
// with a mask its tile codes (summarised first into the workspace's head).
static cudaError_t launch_varlen_aux_lists(const AttnProblem& p, const VarlenAux& ax,
                                           const AuxView& mview, const VarlenLists& vl,
                                           void* workspace, const ListsLayout& lay,
                                           cudaStream_t st) {
  int32_t* nf = at<int32_t>(workspace, lay.nf);
  int32_t* np = at<int32_t>(workspace, lay.np);
  int32_t* fi = at<int32_t>(workspace, lay.fi);
  int32_t* pi = at<int32_t>(workspace, lay.pi);
  if (ax.mask == nullptr && ax.bias == nullptr) return launch_varlen_lists(p, nf, fi, np, pi, st);
  uint8_t* codes = nullptr;
  if (ax.mask != nullptr) {
    codes = at<uint8_t>(workspace, 0);
    const int64_t folded[4] = {mview.sb, mview.sh, mview.sq, 1};
    const cudaError_t e = launch_mask_tile_summary(ax.mask, ax.mask_sizes, folded, p.Lk, codes, st);
    if (e != cudaSuccess) return e;
  }
  return launch_explicit_lists(p, codes, vl.codes_qt, nf, fi, np, pi, st);
}

static sma_status varlen_fwd_impl(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                                  int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                                  int32_t max_k, float scale, int32_t is_causal,
                                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                  const void* q, const int64_t q_strides[2], const void* k,
                                  const int64_t k_strides[2], const void* v,
                                  const int64_t v_strides[2], void* out, const int64_t o_strides[2],
                                  float* lse, void* workspace, size_t workspace_bytes,
                                  const VarlenAux& ax, void* stream) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || total_q < 1 || total_k < 1 || max_q < 1 || max_k < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, totals and maxima must be >= 1");
  if (is_causal != 0 && is_causal != 1) return fail(SMA_ERR_INVALID_ARG, "is_causal must be 0 or 1");
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "cu_seqlens_q / cu_seqlens_k are NULL");
  if (q_strides == nullptr || k_strides == nullptr || v_strides == nullptr || o_strides == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "strides are NULL");
  const int64_t qs[3] = {0, q_strides[0], q_strides[1]};
  const int64_t ks[3] = {0, k_strides[0], k_strides[1]};
  const int64_t vs[3] = {0, v_strides[0], v_strides[1]};
  const int64_t os[3] = {0, o_strides[0], o_strides[1]};
  if ((s = check_operand("q", q, qs, dtype, total_q)) != SMA_OK) return s;
  if ((s = check_operand("k", k, ks, dtype, total_k)) != SMA_OK) return s;
  if ((s = check_operand("v", v, vs, dtype, total_k)) != SMA_OK) return s;
  if ((s = check_operand("out", out, os, dtype, total_q)) != SMA_OK) return s;
  AuxView mview, bview;
  if ((s = check_varlen_aux(ax, batch, heads, kv_heads, max_q, max_k, &mview, &bview)) != SMA_OK)
    return s;
  const bool has_mask = ax.mask != nullptr, has_bias = ax.bias != nullptr;
  const VarlenLists vl = varlen_lists_geom(batch, heads, kv_heads, max_q, max_k, head_dim,
                                           has_mask ? ax.mask_sizes : nullptr);
  const ListsLayout lay = lists_layout(vl.codes_bytes,
                                       static_cast<int64_t>(batch) * vl.LH * ceil_div(max_q, kTile),
                                       static_cast<int>(ceil_div(max_k, kTile)));
  if ((s = check_workspace(workspace, workspace_bytes, lay.end)) != SMA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  AttnProblem p{};
  p.dtype = dtype;
  p.B = batch; p.H = heads; p.KVH = kv_heads; p.Lq = max_q; p.Lk = max_k; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = (p.group + 1) / 2;
  p.QT = static_cast<int>(ceil_div(max_q, kTile));
  p.KT = static_cast<int>(ceil_div(max_k, kTile));
  p.scale_log2 = resolve_scale(scale, head_dim) * kLog2eHost;
  p.q = q; p.q_sb = 0; p.q_sr = q_strides[0]; p.q_sh = q_strides[1];
  p.k = k; p.k_sb = 0; p.k_sr = k_strides[0]; p.k_sh = k_strides[1];
  p.v = v; p.v_sb = 0; p.v_sr = v_strides[0]; p.v_sh = v_strides[1];
  p.o = out; p.o_sb = 0; p.o_sr = o_strides[0]; p.o_sh = o_strides[1];
  p.lse = lse;
  p.policy = kPolicyVarlen;
  p.causal = is_causal;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.err = err;
  p.has_mask = has_mask;
  p.has_bias = has_bias;
  if (has_mask) p.mask = mview;
  if (has_bias) p.bias = bview;
  p.lists.LB = batch; p.lists.LH = vl.LH; p.lists.head_mode = vl.head_mode;
  p.lists.num_full = at<int32_t>(workspace, lay.nf);
  p.lists.num_part = at<int32_t>(workspace, lay.np);
  p.lists.full_idx = at<int32_t>(workspace, lay.fi);
  p.lists.part_idx = at<int32_t>(workspace, lay.pi);
  if ((e = launch_varlen_aux_lists(p, ax, mview, vl, workspace, lay, st)) != cudaSuccess)
    return cuda_fail(e, "tile list launch failed");
  if (dtype == SMA_FP32) {
    e = launch_attn_simt(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch failed");
    return ok();
  }
  char msg[256];
  const int rc = launch_attn_tc(p, st, msg, sizeof(msg));
  if (rc != SMA_OK) return fail(rc, "%s", msg);
  return ok();
}

sma_status varlen_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                           int32_t max_k, float scale, int32_t is_causal, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, const void* q, const int64_t q_strides[2],
                           const void* k, const int64_t k_strides[2], const void* v,
                           const int64_t v_strides[2], void* out, const int64_t o_strides[2],
                           float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return varlen_fwd_impl(dtype, batch, heads, kv_heads, head_dim, total_q, total_k, max_q, max_k,
                         scale, is_causal, cu_seqlens_q, cu_seqlens_k, q, q_strides, k, k_strides, v,
                         v_strides, out, o_strides, lse, workspace, workspace_bytes, VarlenAux{},
                         stream);
}

sma_status varlen_masked_attn_fwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                                 int32_t max_q, int32_t max_k, int32_t head_dim,
                                                 const int64_t mask_sizes[4], size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || max_q < 1 || max_k < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, max_q and max_k must be >= 1");
  const VarlenLists vl = varlen_lists_geom(batch, heads, kv_heads, max_q, max_k, head_dim, mask_sizes);
  *bytes = lists_layout(vl.codes_bytes, static_cast<int64_t>(batch) * vl.LH * ceil_div(max_q, kTile),
                        static_cast<int>(ceil_div(max_k, kTile))).end;
  return ok();
}

sma_status varlen_masked_attn_fwd(
    int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads, int32_t head_dim, int32_t total_q,
    int32_t total_k, int32_t max_q, int32_t max_k, float scale, int32_t is_causal,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const void* q,
    const int64_t q_strides[2], const void* k, const int64_t k_strides[2], const void* v,
    const int64_t v_strides[2], const uint8_t* mask, const int64_t mask_sizes[4],
    const int64_t mask_strides[4], const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
    const int64_t bias_strides[4], void* out, const int64_t o_strides[2], float* lse,
    void* workspace, size_t workspace_bytes, void* stream) {
  VarlenAux ax;
  ax.mask = mask; ax.mask_sizes = mask_sizes; ax.mask_strides = mask_strides;
  ax.bias = bias; ax.bias_dtype = bias_dtype; ax.bias_sizes = bias_sizes; ax.bias_strides = bias_strides;
  return varlen_fwd_impl(dtype, batch, heads, kv_heads, head_dim, total_q, total_k, max_q, max_k,
                         scale, is_causal, cu_seqlens_q, cu_seqlens_k, q, q_strides, k, k_strides, v,
                         v_strides, out, o_strides, lse, workspace, workspace_bytes, ax, stream);
}

sma_status varlen_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t total_q,
                                          int32_t max_q, int32_t max_k, int32_t head_dim,
                                          size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  if (batch < 1 || heads < 1 || total_q < 1 || max_q < 1 || max_k < 1 || head_dim < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, heads, total_q, maxima and head_dim must be >= 1");
  const int QT = static_cast<int>(ceil_div(max_q, kTile));
  const int KT = static_cast<int>(ceil_div(max_k, kTile));
  // lists per sequence; per-query data and the dQ accumulator over the packed rows
  *bytes = bwd_layout(0, batch, QT, KT, 1, heads, total_q, head_dim).total;
  return ok();
}

static sma_status varlen_bwd_impl(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                                  int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                                  int32_t max_k, float scale, int32_t is_causal,
                                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                  const void* q, const int64_t q_strides[2], const void* k,
                                  const int64_t k_strides[2], const void* v,
                                  const int64_t v_strides[2], const void* out,
                                  const int64_t o_strides[2], const float* lse, const void* dout,
                                  const int64_t do_strides[2], void* dq, const int64_t dq_strides[2],
                                  void* dk, const int64_t dk_strides[2], void* dv,
                                  const int64_t dv_strides[2], void* workspace,
                                  size_t workspace_bytes, const VarlenAux& ax, void* stream) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || total_q < 1 || total_k < 1 || max_q < 1 || max_k < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, totals and maxima must be >= 1");
  if (is_causal != 0 && is_causal != 1) return fail(SMA_ERR_INVALID_ARG, "is_causal must be 0 or 1");
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "cu_seqlens_q / cu_seqlens_k are NULL");
  const int64_t* s2[7] = {q_strides, k_strides, v_strides, o_strides, do_strides, dq_strides, dk_strides};
  for (const int64_t* a : s2)
    if (a == nullptr) return fail(SMA_ERR_INVALID_ARG, "strides are NULL");
  if (dv_strides == nullptr) return fail(SMA_ERR_INVALID_ARG, "strides are NULL");
  // [rows, heads, d] operands as one batch entry: strides {0, row, head}
  const int64_t qs[3] = {0, q_strides[0], q_strides[1]}, ks[3] = {0, k_strides[0], k_strides[1]};
  const int64_t vs[3] = {0, v_strides[0], v_strides[1]}, os[3] = {0, o_strides[0], o_strides[1]};
  const int64_t gs[3] = {0, do_strides[0], do_strides[1]}, dqs[3] = {0, dq_strides[0], dq_strides[1]};
  const int64_t dks[3] = {0, dk_strides[0], dk_strides[1]}, dvs[3] = {0, dv_strides[0], dv_strides[1]};
  if ((s = check_operand("q", q, qs, dtype, total_q)) != SMA_OK) return s;
  if ((s = check_operand("k", k, ks, dtype, total_k)) != SMA_OK) return s;
  if ((s = check_operand("v", v, vs, dtype, total_k)) != SMA_OK) return s;
  if ((s = check_grad_operands(dtype, total_q, total_k, out, os, lse, dout, gs, dq, dqs, dk, dks, dv,
                               dvs)) != SMA_OK)
    return s;
  if (ax.dbias != nullptr && ax.bias == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "dbias needs the bias (it takes the bias's shape)");
  if (ax.dbias != nullptr && (reinterpret_cast<uintptr_t>(ax.dbias) & 15u) != 0)
    return fail(SMA_ERR_INVALID_ARG, "dbias must be 16-byte aligned");
  AuxView mview, bview;
  if ((s = check_varlen_aux(ax, batch, heads, kv_heads, max_q, max_k, &mview, &bview)) != SMA_OK)
    return s;
  const bool has_mask = ax.mask != nullptr, has_bias = ax.bias != nullptr;
  const VarlenLists vl = varlen_lists_geom(batch, heads, kv_heads, max_q, max_k, head_dim,
                                           has_mask ? ax.mask_sizes : nullptr);
  const int QT = static_cast<int>(ceil_div(max_q, kTile));
  const int KT = static_cast<int>(ceil_div(max_k, kTile));
  const BwdLayout lay = bwd_layout(vl.codes_bytes, static_cast<int64_t>(batch) * vl.LH, QT, KT, 1,
                                   heads, total_q, head_dim);
  if ((s = check_workspace(workspace, workspace_bytes, lay.total)) != SMA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  int* err = device_error_word(&e);
  if (err == nullptr) return cuda_fail(e, "device error word unavailable");
  BwdProblem b{};
  AttnProblem& p = b.f;
  p.dtype = dtype;
  p.B = batch; p.H = heads; p.KVH = kv_heads; p.Lq = max_q; p.Lk = max_k; p.d = head_dim;
  p.group = heads / kv_heads;
  p.npairs = (p.group + 1) / 2;
  p.QT = QT; p.KT = KT;
  const float sc = resolve_scale(scale, head_dim);
  p.scale_log2 = sc * kLog2eHost;
  p.q = q; p.q_sb = 0; p.q_sr = qs[1]; p.q_sh = qs[2];
  p.k = k; p.k_sb = 0; p.k_sr = ks[1]; p.k_sh = ks[2];
  p.v = v; p.v_sb = 0; p.v_sr = vs[1]; p.v_sh = vs[2];
  p.o = const_cast<void*>(out); p.o_sb = 0; p.o_sr = os[1]; p.o_sh = os[2];
  p.lse = const_cast<float*>(lse);
  p.policy = kPolicyVarlen;
  p.causal = is_causal;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.err = err;
  p.has_mask = has_mask;
  p.has_bias = has_bias;
  if (has_mask) p.mask = mview;
  if (has_bias) p.bias = bview;
  p.lists.LB = batch; p.lists.LH = vl.LH; p.lists.head_mode = vl.head_mode;
  int32_t* nf = at<int32_t>(workspace, lay.fl.nf);
  int32_t* np = at<int32_t>(workspace, lay.fl.np);
  int32_t* fi = at<int32_t>(workspace, lay.fl.fi);
  int32_t* pi = at<int32_t>(workspace, lay.fl.pi);
  p.lists.num_full = nf; p.lists.num_part = np; p.lists.full_idx = fi; p.lists.part_idx = pi;
  if ((e = launch_varlen_aux_lists(p, ax, mview, vl, workspace, lay.fl, st)) != cudaSuccess)
    return cuda_fail(e, "tile list launch failed");
  set_grads(b, dout, gs, dq, dqs, dk, dks, dv, dvs, sc);
  if (ax.dbias != nullptr) {
    // as masked_attn_bwd: contiguous fp32 at the bias's sizes, rows and
    // columns sequence-local
    const int64_t kd = ax.bias_sizes[3];
    const int64_t nb = ax.bias_sizes[0], nh = ax.bias_sizes[1], nq = ax.bias_sizes[2];
    e = cudaMemsetAsync(ax.dbias, 0, static_cast<size_t>(nb * nh * nq * kd) * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "dbias zeroing failed");
    if (kd > 1 || max_k == 1) {
      b.dbias = ax.dbias;
      b.db_sq = nq > 1 ? kd : 0;
      b.db_sh = nh > 1 ? nq * kd : 0;
      b.db_sb = nb > 1 ? nh * nq * kd : 0;
      b.db_kd = static_cast<int>(kd);
      const int db_hpq = nh == heads ? 1 : 0;
      b.db_head_per_query = db_hpq;
      const bool own_head = heads == 1 || (nh > 1 && (db_hpq || p.group == 1));
      const bool own_batch = batch == 1 || nb > 1;
      b.db_mode = nq == 1 ? kDbiasRowSum : (own_head && own_batch ? kDbiasStore : kDbiasAdd);
    }
  }
  if ((s = run_backward(b, workspace, lay, st)) != SMA_OK) return s;
  return ok();
}

sma_status varlen_attn_bwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                           int32_t max_k, float scale, int32_t is_causal, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, const void* q, const int64_t q_strides[2],
                           const void* k, const int64_t k_strides[2], const void* v,
                           const int64_t v_strides[2], const void* out, const int64_t o_strides[2],
                           const float* lse, const void* dout, const int64_t do_strides[2],
                           void* dq, const int64_t dq_strides[2], void* dk,
                           const int64_t dk_strides[2], void* dv, const int64_t dv_strides[2],
                           void* workspace, size_t workspace_bytes, void* stream) {
  return varlen_bwd_impl(dtype, batch, heads, kv_heads, head_dim, total_q, total_k, max_q, max_k,
                         scale, is_causal, cu_seqlens_q, cu_seqlens_k, q, q_strides, k, k_strides, v,
                         v_strides, out, o_strides, lse, dout, do_strides, dq, dq_strides, dk,
                         dk_strides, dv, dv_strides, workspace, workspace_bytes, VarlenAux{}, stream);
}

sma_status varlen_masked_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                                 int32_t total_q, int32_t max_q, int32_t max_k,
                                                 int32_t head_dim, const int64_t mask_sizes[4],
                                                 size_t* bytes) {
  if (bytes == nullptr) return fail(SMA_ERR_INVALID_ARG, "bytes is NULL");
  sma_status s = check_heads(heads, kv_heads, head_dim);
  if (s != SMA_OK) return s;
  if (batch < 1 || total_q < 1 || max_q < 1 || max_k < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, total_q and maxima must be >= 1");
  const VarlenLists vl = varlen_lists_geom(batch, heads, kv_heads, max_q, max_k, head_dim, mask_sizes);
  *bytes = bwd_layout(vl.codes_bytes, static_cast<int64_t>(batch) * vl.LH,
                      static_cast<int>(ceil_div(max_q, kTile)), static_cast<int>(ceil_div(max_k, kTile)),
                      1, heads, total_q, head_dim)
               .total;
  return ok();
}

sma_status varlen_masked_attn_bwd(
    int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads, int32_t head_dim, int32_t total_q,
    int32_t total_k, int32_t max_q, int32_t max_k, float scale, int32_t is_causal,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const void* q,
    const int64_t q_strides[2], const void* k, const int64_t k_strides[2], const void* v,
    const int64_t v_strides[2], const uint8_t* mask, const int64_t mask_sizes[4],
    const int64_t mask_strides[4], const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
    const int64_t bias_strides[4], const void* out, const int64_t o_strides[2], const float* lse,
    const void* dout, const int64_t do_strides[2], void* dq, const int64_t dq_strides[2], void* dk,
    const int64_t dk_strides[2], void* dv, const int64_t dv_strides[2], float* dbias,
    void* workspace, size_t workspace_bytes, void* stream) {
  VarlenAux ax;
  ax.mask = mask; ax.mask_sizes = mask_sizes; ax.mask_strides = mask_strides;
  ax.bias = bias; ax.bias_dtype = bias_dtype; ax.bias_sizes = bias_sizes; ax.bias_strides = bias_strides;
  ax.dbias = dbias;
  return varlen_bwd_impl(dtype, batch, heads, kv_heads, head_dim, total_q, total_k, max_q, max_k,
                         scale, is_causal, cu_seqlens_q, cu_seqlens_k, q, q_strides, k, k_strides, v,
                         v_strides, out, o_strides, lse, dout, do_strides, dq, dq_strides, dk,
                         dk_strides, dv, dv_strides, workspace, workspace_bytes, ax, stream);
}

static sma_status check_pad_args(int32_t dtype, int32_t batch, int32_t max_len, int32_t heads,
                                 int32_t head_dim, const int32_t* cu, const void* packed,
                                 const int64_t* p_strides, const void* padded,
                                 const int64_t* d_strides) {
  if (!valid_dtype(dtype)) return fail(SMA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (batch < 1 || max_len < 0 || heads < 1 || head_dim < 1)
    return fail(SMA_ERR_INVALID_ARG, "batch, heads and head_dim must be >= 1, max_len >= 0");
  const int es = elem_size(dtype);
  if ((head_dim * es) % 16 != 0) return fail(SMA_ERR_INVALID_ARG, "rows must be multiples of 16 bytes");
  if (cu == nullptr || packed == nullptr || padded == nullptr || p_strides == nullptr ||
      d_strides == nullptr)
    return fail(SMA_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(packed) || !aligned16(padded))
    return fail(SMA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  for (int i = 0; i < 2; ++i)
    if (p_strides[i] < 0 || (p_strides[i] * es) % 16 != 0)
      return fail(SMA_ERR_INVALID_ARG, "packed strides must be non-negative multiples of 16 bytes");
  for (int i = 0; i < 3; ++i)
    if (d_strides[i] < 0 || (d_strides[i] * es) % 16 != 0)
      return fail(SMA_ERR_INVALID_ARG, "padded strides must be non-negative multiples of 16 bytes");
  return SMA_OK;
}

sma_status varlen_pad(int32_t dtype, int32_t batch, int32_t max_len, int32_t heads,
                      int32_t head_dim, const int32_t* cu_seqlens, const void* packed,
                      const int64_t packed_strides[2], void* padded,
                      const int64_t padded_strides[3], void* stream) {
  sma_status s = check_pad_args(dtype, batch, max_len, heads, head_dim, cu_seqlens, packed,
                                packed_strides, padded, padded_strides);
  if (s != SMA_OK) return s;
  cudaError_t e = launch_varlen_pad(packed, padded, cu_seqlens, batch, max_len, heads, head_dim,
                                    elem_size(dtype), packed_strides[0], packed_strides[1],
                                    padded_strides[0], padded_strides[1], padded_strides[2],
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pad launch failed");
  return ok();
}

sma_status varlen_unpad(int32_t dtype, int32_t batch, int32_t max_len, int32_t heads,
                        int32_t head_dim, const int32_t* cu_seqlens, const void* padded,
                        const int64_t padded_strides[3], void* packed,
                        const int64_t packed_strides[2], void* stream) {
  sma_status s = check_pad_args(dtype, batch, max_len, heads, head_dim, cu_seqlens, packed,
                                packed_strides, padded, padded_strides);
  if (s != SMA_OK) return s;
  cudaError_t e = launch_varlen_unpad(padded, packed, cu_seqlens, batch, max_len, heads, head_dim,
                                      elem_size(dtype), packed_strides[0], packed_strides[1],
                                      padded_strides[0], padded_strides[1], padded_strides[2],
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "unpad launch failed");
  return ok();
}

}  // extern "C"
