/*
 * sma.h -- C ABI of libsma: scaled-dot-product attention under structured
 * masks on NVIDIA B200 (sm_100a).
 *
 * Operations, all asynchronous on the caller's CUDA stream:
 *
 *   dfa_block_map      full / partial / empty key-tile lists of the DFlash
 *                      draft-training mask, computed from the block anchors
 *                      alone (no dense mask is ever built).
 *   dfa_attn_fwd       attention forward under that mask (also the DFlash
 *                      inference mask: one block, anchor = context length).
 *   masked_attn_fwd    attention forward with a broadcastable 4D boolean mask
 *                      and/or additive bias, optional causal masking, and the
 *                      single-query grouped-head ("swapped") decode path.
 *   dynamic_topk_mask  boolean keep mask of the window_size largest entries
 *                      of an attention bias per row, after a pre-mask.
 *   sparse_attn_fwd    masked_attn_fwd over only the keys a query-broadcast
 *                      mask keeps (index gather), e.g. a top-k mask.
 *   dfa_attn_bwd,      gradients dQ, dK, dV of the two attention forwards.
 *   masked_attn_bwd    (and masked_attn_bwd_deterministic: dbias summed in a
 *                      fixed order)
 *   varlen_attn_fwd    attention over packed variable-length sequences, with
 *                      varlen_pad / varlen_unpad.
 *
 * plus mask_tile_summary (the tile classifier masked_attn_fwd runs on an
 * explicit mask), workspace queries and error reporting.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor arguments are DEVICE pointers owned by the caller; the library
 *   allocates no device memory and keeps no state besides a thread-local
 *   error string and one device error word per device.
 * - Strides are in ELEMENTS.  Q/K/V/O are [batch, length, heads, head_dim]
 *   with head_dim contiguous; their strides arrays give the batch, length and
 *   head strides in that order.  Every stride and base address must be a
 *   multiple of 16 bytes (TMA requirement) for bf16/fp16 inputs.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 * - Arguments are validated on the host before anything is launched; an
 *   invalid call returns a nonzero status and launches nothing.  The message
 *   is available from sma_last_error() on the calling thread.
 * - Faults found on the device (an anchor out of range, a pipeline wait that
 *   ran out of time) set the device error word; read and clear it with
 *   sma_device_status().  Kernels never trap.
 * - Query head h uses key/value head h / (heads / kv_heads) (contiguous
 *   groups).
 * - scale <= 0 selects 1/sqrt(head_dim).
 * - lse (nullable) receives the natural-log log-sum-exp of each row's kept
 *   scores, float32 [batch, heads, q_len] contiguous; a row with no kept key
 *   gets -inf and a zero output row.
 */
#ifndef SMA_H_
#define SMA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t sma_status;

#define SMA_OK 0
#define SMA_ERR_INVALID_ARG 1    /* shape, stride, pointer or value rejected */
#define SMA_ERR_UNSUPPORTED 2    /* valid but not implemented (e.g. head_dim 96) */
#define SMA_ERR_CUDA 3           /* a CUDA runtime/driver call failed */
#define SMA_ERR_WORKSPACE 4      /* workspace smaller than the size query says */
#define SMA_ERR_DEVICE_TIMEOUT 5 /* a kernel's bounded pipeline wait expired */
#define SMA_ERR_DEVICE_INPUT 6   /* a device-resident input was out of range */

#define SMA_BF16 0
#define SMA_FP16 1
#define SMA_FP32 2

/* Tiles of the block maps and summaries are SMA_TILE x SMA_TILE
 * (queries x keys). */
#define SMA_TILE 128
#define SMA_TILE_EMPTY 0
#define SMA_TILE_PARTIAL 1
#define SMA_TILE_FULL 2

#define SMA_IS_CAUSAL_UNSET (-1)
#define SMA_LAYER_FULL 0
#define SMA_LAYER_SLIDING 1

/* Message for the last nonzero status returned on this thread ("" if none). */
const char* sma_last_error(void);

/* ABI version of this header (bumped on any signature change). */
int32_t sma_abi_version(void);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device into *device_error (SMA_OK if no kernel reported a fault).
 * Returns SMA_ERR_CUDA if the synchronisation itself failed. */
sma_status sma_device_status(void* stream, int32_t* device_error);

/* Diagnostic: launches one tiny kernel that waits, with the bounded wait every
 * pipeline kernel of the library uses, on a barrier that nothing completes.
 * After `timeout_ns` (1 ms .. 2 s) the wait gives up, the kernel records
 * SMA_ERR_DEVICE_TIMEOUT in the device error word and returns normally, so
 * the CUDA context stays usable.  dev_out (device, int64[2]) receives
 * {1 if the wait gave up else 0, nanoseconds waited}.  Not part of the
 * method; it checks the failure-reporting path without faulting the GPU. */
sma_status sma_selftest_wait_timeout(int64_t timeout_ns, int64_t* dev_out, void* stream);

/* ------------------------------------------------------------------------
 * DFlash mask description.
 *
 * Source: SpecForge issue #452 "flex_attention BlockMask incorrectly created
 * with H=num_heads", Problem paragraph -- every draft query sees the context
 * that precedes its block plus the tokens of its own block, identically for
 * every head (so the maps here have no head dimension).  SpecForge PR #905
 * "Fix DFlash attention masking", Motivation list -- is_causal absent:
 * bidirectional inside the block on full-attention layers, causal on
 * sliding-attention layers; False: bidirectional on both; True: causal on
 * both.  Same page, reply item 1 (#934): the in-block sliding window keeps
 * only its left bound.
 *
 * Keys are laid out as [context 0..ctx_len) [block 0] ... [block N-1], so
 * k_len = ctx_len + n_blocks * block_size and q_len = n_blocks * block_size.
 * Query i of block j sits at position anchor[b][j] + i, context key k at
 * position k.  Query (j, i) keeps
 *   context key k  iff k < anchor[b][j]  and (sliding: anchor[b][j]+i-k < W)
 *   draft key of block j' at offset t  iff j' == j and (causal: t <= i)
 *                                        and (sliding: i - t < W).
 * ---------------------------------------------------------------------- */
typedef struct dfa_mask_desc {
  int32_t batch;          /* B >= 1 */
  int32_t n_blocks;       /* N >= 1 draft blocks per sequence */
  int32_t block_size;     /* tokens per draft block, >= 1 */
  int32_t ctx_len;        /* context keys, >= 0 */
  int32_t is_causal;      /* SMA_IS_CAUSAL_UNSET, 0 or 1 */
  int32_t layer_type;     /* SMA_LAYER_FULL or SMA_LAYER_SLIDING */
  int32_t sliding_window; /* W >= 1; read only when layer_type is sliding */
} dfa_mask_desc;

/* Tile-grid size of the block map: q_tiles = ceil(q_len/128),
 * kv_tiles = ceil(k_len/128). */
sma_status dfa_block_map_dims(const dfa_mask_desc* desc, int32_t* q_tiles, int32_t* kv_tiles);

/* DFlash block map, computed analytically from the anchors.
 *
 * anchors   int32 [batch, n_blocks] device, row-major; each in [0, ctx_len]
 *           (need not be sorted or distinct).  Out-of-range anchors are
 *           clamped and raise SMA_ERR_DEVICE_INPUT in the device error word.
 * num_full  int32 [batch, q_tiles]           number of FULL key tiles
 * full_idx  int32 [batch, q_tiles, kv_tiles] their indices, ascending, then -1
 * num_part  int32 [batch, q_tiles]           number of PARTIAL key tiles
 * part_idx  int32 [batch, q_tiles, kv_tiles] their indices, ascending, then -1
 * A tile is FULL iff it lies inside [0, k_len) and every (valid query, key)
 * pair in it is kept, EMPTY iff none is, PARTIAL otherwise.  This is the
 * flex_attention BlockMask with a head dim of 1 that issue #452 asks for. */
sma_status dfa_block_map(const dfa_mask_desc* desc, const int32_t* anchors, int32_t* num_full,
                         int32_t* full_idx, int32_t* num_part, int32_t* part_idx, void* stream);

/* A block map produced by dfa_block_map for the same descriptor (device
 * pointers, layouts as documented there). */
typedef struct dfa_block_map_ptrs {
  const int32_t* num_full;
  const int32_t* full_idx;
  const int32_t* num_part;
  const int32_t* part_idx;
} dfa_block_map_ptrs;

/* Workspace bytes dfa_attn_fwd uses for this problem: the block map (when
 * the call computes it) and, for problems with too few (batch, KV head, head
 * pair, 128-query tile) units to fill the SMs, the partial results of the
 * key-range split (per segment and query row: fp32 O and the running max and
 * sum).  The caller allocates it; it may be reused across calls ordered on
 * one stream. */
sma_status dfa_attn_fwd_workspace_size(const dfa_mask_desc* desc, int32_t heads, int32_t kv_heads,
                                       int32_t head_dim, size_t* bytes);

/* Attention forward under the DFlash mask.
 *
 * block_map  NULL: the map is computed into `workspace` first (one extra
 *            kernel).  Otherwise a map from dfa_block_map for the same desc
 *            and anchors, e.g. shared by the layers of one training step;
 *            `workspace` may then be NULL with 0 bytes.
 * workspace  at least the block map's bytes when block_map is NULL
 *            (SMA_ERR_WORKSPACE otherwise).  Short-query problems (e.g. one
 *            draft block after a long context) cut each unit's key tiles
 *            into contiguous segments run on separate SMs and merge the
 *            segments' partial results in a second kernel; they do so only
 *            when `workspace` holds dfa_attn_fwd_workspace_size bytes.  The
 *            split changes the fp32 summation order, not the result beyond
 *            rounding.
 * q    [batch, q_len, heads, head_dim]     strides q_strides (batch, row, head)
 * k, v [batch, k_len, kv_heads, head_dim]  strides k_strides / v_strides
 * out  [batch, q_len, heads, head_dim]     strides o_strides; same dtype as q
 * dtype SMA_BF16 / SMA_FP16 (tensor cores, fp32 accumulation and softmax) or
 *       SMA_FP32 (fp32 FFMA throughout).  head_dim 64 or 128; heads a
 *       multiple of kv_heads.
 * Only key tiles the block map marks FULL or PARTIAL are computed; the mask is
 * evaluated per element on PARTIAL tiles only. */
sma_status dfa_attn_fwd(const dfa_mask_desc* desc, const int32_t* anchors, int32_t dtype,
                        int32_t heads, int32_t kv_heads, int32_t head_dim, float scale,
                        const void* q, const int64_t q_strides[3], const void* k,
                        const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                        void* out, const int64_t o_strides[3], float* lse,
                        const dfa_block_map_ptrs* block_map, void* workspace,
                        size_t workspace_bytes, void* stream);

/* dfa_attn_fwd for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot give the library a device workspace -- a plain C host program
 * without a CUDA memory manager of its own, or a runtime whose device memory
 * is fully pre-reserved by another allocator, where one more cudaMalloc
 * would fail or fragment that pool.
 *
 * Same arguments and result as dfa_attn_fwd, without block_map and
 * workspace: the block map goes to a fixed 4 MiB device array inside the
 * library (held by every GPU that loads the library until process exit).
 * Problems whose block map needs more than 4 MiB return SMA_ERR_WORKSPACE
 * (about batch * q_tiles * (kv_tiles + 1) * 8 bytes; the 32768-query,
 * 65536-key long-context problem needs 1.05 MB).  Calls share the array:
 * calls that may overlap on the GPU (unordered streams) race, so order them
 * on one stream.  The first call in a CUDA context looks up the array's
 * address with that context current and caches it per context; make it
 * before any stream capture starts.  A new context (after cudaDeviceReset,
 * or a caller's own non-primary context) repeats the lookup on its first
 * call.  No device memory is allocated or freed. */
sma_status dfa_attn_fwd_noalloc(const dfa_mask_desc* desc, const int32_t* anchors, int32_t dtype,
                                int32_t heads, int32_t kv_heads, int32_t head_dim, float scale,
                                const void* q, const int64_t q_strides[3], const void* k,
                                const int64_t k_strides[3], const void* v,
                                const int64_t v_strides[3], void* out, const int64_t o_strides[3],
                                float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Broadcastable 4D mask / bias contract.
 *
 * Source: flash-sparse-attention PR #190 "Broadcastable 4D mask/bias,
 * 128-rounded key length, stride-0 broadcasting, and dbias reductions",
 * Design and Changes sections.  mask (uint8 0/1, True = keep) and bias
 * (additive, SMA_BF16/SMA_FP16/SMA_FP32) are rank 4 with sizes
 *   ({batch|1}, {heads|kv_heads|1}, {q_len|1}, {round_up(k_len, 128)|k_len|1})
 * and a contiguous last dim (stride 1).  Size-1 dims broadcast with stride 0
 * whatever stride is passed; there is no implicit 3D form.  A head dim of
 * kv_heads (when kv_heads != heads) is indexed by the query head's KV head.
 * Key dim: the page's interface pads it to round_up(k_len, 128) and expands
 * a key dim of 1 before its kernels run; here all three forms are read in
 * place, with no copy.  Columns in [k_len, round_up(k_len,128)) are never
 * read as meaningful: they are never attended whatever they hold.  A key dim
 * of 1 is one value for every key (its last-dim stride is ignored).
 * Alignment: base address and the batch / head / query strides must be
 * multiples of 16 bytes (vector loads), except for a key dim of 1, which is
 * read one element at a time and needs only element alignment.
 * ---------------------------------------------------------------------- */

/* Tile codes of an explicit mask at its own broadcast shape:
 * codes uint8 [m0, m1, ceil(m2/128), ceil(k_len/128)] contiguous (device),
 * where (m0, m1, m2, m3) = mask_sizes; columns >= k_len count as not kept.
 * mask must be 16-byte aligned with 16-byte-multiple strides (or 0). */
sma_status mask_tile_summary(const uint8_t* mask, const int64_t mask_sizes[4],
                             const int64_t mask_strides[4], int32_t k_len, uint8_t* codes,
                             void* stream);

/* Workspace bytes masked_attn_fwd needs (tile summary, tile lists, the
 * split-KV partials of the single-query path, and for other short-query
 * problems the partials of the key-range split: each unit's key tiles cut
 * into segments run on separate SMs, merged by a second kernel).  mask_sizes may be NULL when
 * no mask will be passed.  The single-query split count follows the current
 * device's SM count (148 when no device is current), so query the size with
 * the device that will run the call current; a smaller workspace is refused
 * with SMA_ERR_WORKSPACE. */
sma_status masked_attn_fwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                          int32_t q_len, int32_t k_len, int32_t head_dim,
                                          const int64_t mask_sizes[4], size_t* bytes);

/* Attention forward with optional mask, bias and causal masking.
 *
 * s = scale * q.k + bias[...];  key k is kept iff k < k_len and
 * mask[...] (when given) and (is_causal -> k <= q + k_len - q_len, i.e.
 * bottom-right aligned).
 * mask / bias: NULL or the 4D contract above; their sizes/strides arrays are
 * ignored when the pointer is NULL.
 * When q_len == 1 (decode) the grouped query heads of each KV head are
 * processed together as rows of one problem (the "swapped" path of PR #190,
 * Swapped path bullets); mask/bias keep their original batch/head meaning.
 * The result is the same as the unswapped definition. */
sma_status masked_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                           int32_t is_causal, const void* q, const int64_t q_strides[3],
                           const void* k, const int64_t k_strides[3], const void* v,
                           const int64_t v_strides[3], const uint8_t* mask,
                           const int64_t mask_sizes[4], const int64_t mask_strides[4],
                           const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                           const int64_t bias_strides[4], void* out, const int64_t o_strides[3],
                           float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dynamic top-k keep mask.
 *
 * Source: flash-sparse-attention PR #197 "Centralize dynamic mask creation
 * for FDMA" -- Design (dynamic_mask / create_mask) and Implementation Notes:
 * positions the pre-mask marks invalid are set to the minimum finite value of
 * the BIAS dtype before choosing the window_size largest entries of each row,
 * so they are never selected.
 *
 * bias      [b, h, q, kc] dtype bias_dtype, strides given, last dim
 *           contiguous, kc = round_up(k_len,128) or k_len (a key dim of 1 is
 *           refused: the output has one column per key).  Only columns
 *           < k_len take part.
 * pre_mask  NULL or uint8 0/1 4D with sizes (pb, ph, pq, pk): pb in {1, b},
 *           ph in {1, h}, pq in {1, q}, pk >= 1, last stride 1; columns
 *           >= pk are invalid.  A 2D (batch, k_len) pre-mask is passed as
 *           sizes (batch, 1, 1, k_len).
 * out_mask  uint8 [b, h, q, kc] contiguous (device), 8-byte aligned; columns
 *           >= k_len are written 0.
 * Per row: entry k is kept iff it is among the window_size largest masked
 * values (equal values: lower k first; -0 equals +0) and the pre-mask keeps
 * it.  window_size >= k_len keeps exactly the pre-mask. */
sma_status dynamic_topk_mask(int32_t bias_dtype, const void* bias, const int64_t bias_sizes[4],
                             const int64_t bias_strides[4], int32_t k_len, const uint8_t* pre_mask,
                             const int64_t pre_mask_sizes[4], const int64_t pre_mask_strides[4],
                             int32_t window_size, uint8_t* out_mask, void* stream);

/* ------------------------------------------------------------------------
 * Backward (gradients) of the two attention entry points.
 *
 * Source: flash-sparse-attention PR #190, Changes (mha_bwd): the backward
 * returns dQ, dK, dV under the same 4D mask/bias contract; SpecForge issue
 * #452 (Problem) for the DFlash mask it is trained with.  With the forward's
 * P (softmax over the kept keys) and O, and the upstream gradient dO:
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *   dQ = scale * dS K,  dK = scale * dS^T Q
 * (dK, dV summed over the query heads of each KV head).  Keys that no query
 * attends get zero gradients; rows with no kept key contribute nothing.
 *
 * out, lse  the forward's output and log-sum-exp (natural log, [B, H, Lq]
 *           contiguous float32, -inf for rows with no kept key), as the
 *           forward call wrote them with the same arguments.
 * dout      the upstream gradient, [B, Lq, H, d] like out.
 * dq        [B, Lq, H, d]; dk, dv [B, Lk, KVH, d]: written, caller-owned,
 *           strides as for q/k/v (last dim contiguous, 16-byte multiples).
 * dtype     SMA_BF16 or SMA_FP16 (tensor cores, fp32 accumulation; dQ is
 *           accumulated in fp32 in the workspace), or SMA_FP32 (fp32 FFMA
 *           throughout, the gradients of the fp32 forward; no tensor cores,
 *           a correctness path).  head_dim 64 or 128.
 * The workspace holds the tile lists, rowsum(dO * O) and the fp32 dQ
 * accumulator (B * Lq * H * d * 4 bytes); query its size first.
 * ---------------------------------------------------------------------- */

sma_status dfa_attn_bwd_workspace_size(const dfa_mask_desc* desc, int32_t heads, int32_t kv_heads,
                                       int32_t head_dim, size_t* bytes);

sma_status dfa_attn_bwd(const dfa_mask_desc* desc, const int32_t* anchors, int32_t dtype,
                        int32_t heads, int32_t kv_heads, int32_t head_dim, float scale,
                        const void* q, const int64_t q_strides[3], const void* k,
                        const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                        const void* out, const int64_t o_strides[3], const float* lse,
                        const void* dout, const int64_t do_strides[3], void* dq,
                        const int64_t dq_strides[3], void* dk, const int64_t dk_strides[3],
                        void* dv, const int64_t dv_strides[3], void* workspace,
                        size_t workspace_bytes, void* stream);

sma_status masked_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                          int32_t q_len, int32_t k_len, int32_t head_dim,
                                          const int64_t mask_sizes[4], size_t* bytes);

/* mask / bias / is_causal / scale exactly as given to masked_attn_fwd (any
 * q_len; single-query problems run the general kernel).
 *
 * dbias (nullable; device, 16-byte aligned, caller-owned): the bias gradient
 * of PR #190 (Changes, mha_bwd), written as contiguous float32 with the
 * bias's own sizes (b', h', q', kd), kd the bias's key dim.  Element
 * (b, h, q, k) of dS = P * (dP - D) (the gradient of the score, bias
 * included) is summed into the dbias element its bias element broadcast
 * from: over the batch when b' = 1, over the heads of a group when
 * h' = kv_heads, over all heads when h' = 1, over the queries when q' = 1,
 * over the keys when kd = 1.  Columns >= k_len come out 0.  With kd = 1 (one
 * bias value for every key of a row) the sum over the row's keys is exactly
 * 0 (sum_k P (dP - D) = D - D): the call writes zeros.
 * The call zeroes dbias first; sums over broadcast dims use fp32 atomic
 * adds, so their rounding order is not fixed (masked_attn_bwd_deterministic
 * fixes it).  Needs a bias (SMA_ERR_INVALID_ARG otherwise). */
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
                           size_t workspace_bytes, void* stream);

/* Bytes of the second workspace masked_attn_bwd_deterministic needs for a
 * bias of sizes bias_sizes (b', h', q', kd): the fixed-order partial sums,
 * batch * heads * R * kd * 4 with R = q_len for a bias with a query dim (or
 * dtype SMA_FP32), else ceil(q_len / 64) (query groups of 64 rows).
 * 0 when every dbias element already has a single writer (a bias with its
 * own element for each batch row, query head and query). */
sma_status masked_attn_bwd_dbias_workspace_size(int32_t dtype, int32_t batch, int32_t heads,
                                                int32_t kv_heads, int32_t q_len, int32_t head_dim,
                                                const int64_t bias_sizes[4], size_t* bytes);

/* masked_attn_bwd with a dbias that is bitwise the same on every call with
 * the same inputs.  The page (PR #190, Changes: dbias reduced over the
 * broadcast dims) fixes the sums but no order; this entry point fixes one:
 * every element of the partial buffer (dbias_workspace, device, at least
 * masked_attn_bwd_dbias_workspace_size bytes, caller-owned) has exactly one
 * writer, per batch row, query head and query (or group of G queries), and
 * one kernel then adds the partials of each dbias element in increasing
 * (batch, head, partial row) order.  dQ / dK / dV are those of
 * masked_attn_bwd.  SMA_ERR_WORKSPACE if dbias_workspace is smaller than the
 * query says. */
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
    void* stream);

/* ------------------------------------------------------------------------
 * Variable-length (packed) batches.
 *
 * Source: flash-sparse-attention PR #197, Changes list: the integration's
 * loader returns a varlen attention function and pad / unpad helpers next to
 * the padded one; the pages give no interface, so this follows the packed
 * layout those names denote.  Sequence b owns rows [cu_seqlens_q[b],
 * cu_seqlens_q[b+1]) of the packed queries and [cu_seqlens_k[b],
 * cu_seqlens_k[b+1]) of the packed keys (int32 [batch + 1], ascending, on the
 * device); it attends only its own keys, bottom-right causal per sequence
 * when is_causal (key k kept iff k <= q + len_k - len_q).  No mask or bias
 * here (varlen_masked_attn_fwd below takes them).
 *
 * q, out   [total_q, heads, d]; k, v [total_k, kv_heads, d]; strides[2] =
 *          {row, head} in elements, d contiguous, 16-byte multiples.
 * lse      NULL or float32 [heads, total_q] (natural log; -inf for rows
 *          with no kept key, e.g. causal rows when len_q > len_k).
 * max_q / max_k bound every sequence's lengths (host values, size the tile
 *          lists); offsets that break a bound, are not ascending or exceed
 *          the totals raise SMA_ERR_DEVICE_INPUT in the device error word and
 *          leave that sequence's rows unwritten.
 * dtype    SMA_BF16 / SMA_FP16 (tensor cores) or SMA_FP32 (FFMA
 *          arithmetic, no TF32); head_dim 64 or 128.
 * ---------------------------------------------------------------------- */

sma_status varlen_attn_fwd_workspace_size(int32_t batch, int32_t max_q, int32_t max_k, size_t* bytes);

sma_status varlen_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                           int32_t max_k, float scale, int32_t is_causal, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, const void* q, const int64_t q_strides[2],
                           const void* k, const int64_t k_strides[2], const void* v,
                           const int64_t v_strides[2], void* out, const int64_t o_strides[2],
                           float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes varlen_attn_bwd needs: the per-sequence tile lists and
 * their transpose, rowsum(dO * O) [heads, total_q] and the fp32 dQ
 * accumulator [total_q, heads, head_dim]. */
sma_status varlen_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t total_q,
                                          int32_t max_q, int32_t max_k, int32_t head_dim,
                                          size_t* bytes);

/* Gradients of varlen_attn_fwd for an upstream gradient dout (the packed
 * counterpart of masked_attn_bwd; the derivative of softmax attention as in
 * flash-sparse-attention PR #190, Changes: mha_bwd, per sequence).  out and
 * lse are that forward's results for the same arguments (lse required);
 * dout, dq [total_q, heads, d], dk, dv [total_k, kv_heads, d] with strides[2]
 * = {row, head}.  Keys of a sequence that none of its queries keeps get zero
 * dK / dV; rows with no kept key get zero dQ.  bf16 / fp16 on the tensor
 * cores, fp32 with FFMA arithmetic; offsets as in varlen_attn_fwd. */
sma_status varlen_attn_bwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t head_dim, int32_t total_q, int32_t total_k, int32_t max_q,
                           int32_t max_k, float scale, int32_t is_causal, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, const void* q, const int64_t q_strides[2],
                           const void* k, const int64_t k_strides[2], const void* v,
                           const int64_t v_strides[2], const void* out, const int64_t o_strides[2],
                           const float* lse, const void* dout, const int64_t do_strides[2],
                           void* dq, const int64_t dq_strides[2], void* dk,
                           const int64_t dk_strides[2], void* dv, const int64_t dv_strides[2],
                           void* workspace, size_t workspace_bytes, void* stream);

/* Packed batches with a mask and / or bias (reading R33: PR #197's varlen
 * function sits next to the mask creation it centralises, so a packed batch
 * takes the same mask / bias as the padded call).  They come in the padded
 * per-sequence layout of masked_attn_fwd for the problem [batch, max_q,
 * heads, max_k]: sizes (B|1, H|KVH|1, max_q|1, round_up(max_k, 128)|max_k|1),
 * element (b, h, q, k) for query q and key k of sequence b (both
 * sequence-local), any of mask / bias NULL.  Everything else, including the
 * causal rule, as varlen_attn_fwd / varlen_attn_bwd; dbias (nullable) as in
 * masked_attn_bwd, at the bias's sizes with sequence-local rows and columns.
 * The workspaces also hold the mask's tile codes: query them with the mask's
 * sizes (NULL: none). */
sma_status varlen_masked_attn_fwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                                 int32_t max_q, int32_t max_k, int32_t head_dim,
                                                 const int64_t mask_sizes[4], size_t* bytes);

sma_status varlen_masked_attn_fwd(
    int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads, int32_t head_dim, int32_t total_q,
    int32_t total_k, int32_t max_q, int32_t max_k, float scale, int32_t is_causal,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const void* q,
    const int64_t q_strides[2], const void* k, const int64_t k_strides[2], const void* v,
    const int64_t v_strides[2], const uint8_t* mask, const int64_t mask_sizes[4],
    const int64_t mask_strides[4], const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
    const int64_t bias_strides[4], void* out, const int64_t o_strides[2], float* lse,
    void* workspace, size_t workspace_bytes, void* stream);

sma_status varlen_masked_attn_bwd_workspace_size(int32_t batch, int32_t heads, int32_t kv_heads,
                                                 int32_t total_q, int32_t max_q, int32_t max_k,
                                                 int32_t head_dim, const int64_t mask_sizes[4],
                                                 size_t* bytes);

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
    void* workspace, size_t workspace_bytes, void* stream);

/* pad: padded [batch, max_len, heads, d] (strides[3] = batch, row, head) from
 * packed rows, zero past each sequence's length; unpad: the reverse (rows
 * past a length are not read).  Rows must be 16-byte multiples. */
sma_status varlen_pad(int32_t dtype, int32_t batch, int32_t max_len, int32_t heads,
                      int32_t head_dim, const int32_t* cu_seqlens, const void* packed,
                      const int64_t packed_strides[2], void* padded,
                      const int64_t padded_strides[3], void* stream);

sma_status varlen_unpad(int32_t dtype, int32_t batch, int32_t max_len, int32_t heads,
                        int32_t head_dim, const int32_t* cu_seqlens, const void* padded,
                        const int64_t padded_strides[3], void* packed,
                        const int64_t packed_strides[2], void* stream);

/* ------------------------------------------------------------------------
 * Index-gather attention under a query-broadcast keep mask.
 *
 * Source: flash-sparse-attention PR #197 (Design: the top-k keep mask of a
 * bias row, broadcast over the query dim in its Usage) with the mask/bias
 * contract and causal rule of PR #190.  Computes exactly what
 * masked_attn_fwd computes for the same arguments, but only over the kept
 * keys: per (batch row, head row) of the mask the kept key indices are
 * listed in ascending order, the K/V rows (and bias columns) they name are
 * copied into compacted operands in the workspace, and attention runs over
 * those with the causal bound applied to the original indices.  Work scales
 * with the kept keys, not with k_len.
 *
 * mask      required; the 4D contract above with sizes[2] == 1 (one row for
 *           every query) and sizes[1] in {1, kv_heads} (or heads when heads
 *           == kv_heads): rows shared by the query heads of a KV head.
 *           Other masks return SMA_ERR_UNSUPPORTED (use masked_attn_fwd).
 * bias      NULL or the 4D contract above (any broadcast shape).
 * max_keys  upper bound on the kept keys of any mask row (e.g. the top-k
 *           window_size); <= 0 or > k_len means k_len.  It sizes the
 *           compacted operands.  A row with more kept keys is cut to its
 *           first max_keys and raises SMA_ERR_DEVICE_INPUT in the device
 *           error word (read with sma_device_status).
 * dtype     SMA_BF16 / SMA_FP16 (tensor cores) or SMA_FP32 (FFMA).
 * Other arguments as masked_attn_fwd; all q_len >= 1 run the prefill kernel
 * (with the key-range split over the compacted key tiles when too few units
 * fill the SMs).  A row that keeps no key gives out = 0 and lse = -inf. */
sma_status sparse_attn_fwd_workspace_size(int32_t dtype, int32_t batch, int32_t heads,
                                          int32_t kv_heads, int32_t q_len, int32_t k_len,
                                          int32_t head_dim, const int64_t mask_sizes[4],
                                          int32_t bias_dtype, const int64_t bias_sizes[4],
                                          int32_t max_keys, size_t* bytes);

sma_status sparse_attn_fwd(int32_t dtype, int32_t batch, int32_t heads, int32_t kv_heads,
                           int32_t q_len, int32_t k_len, int32_t head_dim, float scale,
                           int32_t is_causal, const void* q, const int64_t q_strides[3],
                           const void* k, const int64_t k_strides[3], const void* v,
                           const int64_t v_strides[3], const uint8_t* mask,
                           const int64_t mask_sizes[4], const int64_t mask_strides[4],
                           const void* bias, int32_t bias_dtype, const int64_t bias_sizes[4],
                           const int64_t bias_strides[4], int32_t max_keys, void* out,
                           const int64_t o_strides[3], float* lse, void* workspace,
                           size_t workspace_bytes, void* stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* SMA_H_ */
