"""DFlash draft-training keep mask, written out densely (float-free, bool).

Test infrastructure only (see ``oracle/__init__.py``).

Sources
-------
* SpecForge issue #452 "flex_attention BlockMask incorrectly created with
  H=num_heads", Problem paragraph: the visibility pattern is the same for
  every head -- a draft query sees the context that precedes its block and
  the tokens of its own block.  The mask therefore has a head dim of 1.
* SpecForge PR #905 "Fix DFlash attention masking", Motivation list: how
  ``is_causal`` (absent / False / True) decides between bidirectional and
  causal attention inside a block for full- and sliding-attention layers.
* Same page, maintainer reply, item 1 (#934): the in-block sliding window
  keeps only its left bound.

Readings where the pages are silent:
* keys are laid out as ``concat(context[0:Lc], block_0, ..., block_{N-1})``;
* query ``i`` of block ``j`` sits at position ``anchor_j + i``; context key
  ``k`` sits at position ``k``; the window keeps a key iff
  ``pos_q - pos_k < W`` (W positions including the query itself);
* a query of block ``j`` sees context keys ``k < anchor_j`` (strict), the
  wording of the tiny DFlash workload;
* the window applies on sliding-attention layers only.
"""
from __future__ import annotations

import numpy as np

IS_CAUSAL_UNSET = -1
LAYER_FULL = 0
LAYER_SLIDING = 1


def resolve_in_block_causal(is_causal, layer_type: int) -> bool:
    """Causal-inside-the-block decision.

    SpecForge PR #905, Motivation list: ``is_causal`` absent -> bidirectional
    for full-attention layers and causal for sliding-attention layers;
    ``False`` -> bidirectional for both; ``True`` -> causal for both.
    ``None`` and ``-1`` both mean "absent".
    """
    if is_causal is None or int(is_causal) == IS_CAUSAL_UNSET:
        return layer_type == LAYER_SLIDING
    return bool(int(is_causal))


def resolve_window(layer_type: int, sliding_window: int):
    """Left window size W for the layer, or None for full-attention layers."""
    if layer_type == LAYER_SLIDING:
        if sliding_window < 1:
            raise ValueError("sliding layers need sliding_window >= 1")
        return int(sliding_window)
    return None


def dflash_keep_rows(anchors, ctx_len: int, block_size: int, in_block_causal: bool,
                     window, q_start: int, q_stop: int) -> np.ndarray:
    """Rows ``[q_start, q_stop)`` of the dense keep mask, shape ``[B, rows, Lk]``.

    ``anchors`` is ``[B, N]``; ``Lk = ctx_len + N * block_size``.  Query
    ``q = j * block_size + i`` (block ``j``, offset ``i``).

    * context key ``k < ctx_len``: kept iff ``k < anchors[b, j]`` and, with a
      window, ``(anchors[b, j] + i) - k < W``;
    * draft key ``k >= ctx_len`` with ``j' = (k - ctx_len) // block_size`` and
      ``t = (k - ctx_len) % block_size``: kept iff ``j' == j``, ``t <= i`` when
      the block is causal, and ``i - t < W`` with a window (no right bound).
    """
    anchors = np.asarray(anchors, dtype=np.int64)
    n_batch, n_blocks = anchors.shape
    n_q = n_blocks * block_size
    n_k = ctx_len + n_q
    q = np.arange(q_start, q_stop, dtype=np.int64)
    j = q // block_size
    i = q % block_size
    k = np.arange(n_k, dtype=np.int64)

    a = anchors[:, j]                                   # [B, rows]
    kk = k[None, None, :]
    is_ctx = kk < ctx_len
    ctx_keep = is_ctx & (kk < a[:, :, None])
    if window is not None:
        ctx_keep &= (a[:, :, None] + i[None, :, None] - kk) < window

    rel = k - ctx_len
    key_block = np.where(rel >= 0, rel // block_size, -1)
    key_off = np.where(rel >= 0, rel % block_size, -1)
    draft_keep = (rel[None, None, :] >= 0) & (key_block[None, None, :] == j[None, :, None])
    if in_block_causal:
        draft_keep &= key_off[None, None, :] <= i[None, :, None]
    if window is not None:
        draft_keep &= (i[None, :, None] - key_off[None, None, :]) < window
    draft_keep = np.broadcast_to(draft_keep, ctx_keep.shape)
    return ctx_keep | draft_keep


def dflash_keep_mask(anchors, ctx_len: int, block_size: int, in_block_causal: bool,
                     window) -> np.ndarray:
    """Whole dense keep mask ``[B, Nq, Lk]`` (head dim 1 is implied)."""
    anchors = np.asarray(anchors)
    n_q = anchors.shape[1] * block_size
    return dflash_keep_rows(anchors, ctx_len, block_size, in_block_causal, window, 0, n_q)


def dflash_keep_scalar(anchors, ctx_len: int, block_size: int, in_block_causal: bool,
                       window, b: int, q: int, k: int) -> bool:
    """One entry of the keep mask, by walking the positions one at a time.

    Brute-force form used to pin the vectorised construction: it lists the
    positions a query may look back to and asks whether key ``k`` is among
    them, instead of evaluating the closed-form predicate.
    """
    j, i = divmod(q, block_size)
    anchor = int(anchors[b][j])
    q_pos = anchor + i
    visible = set()
    for c in range(ctx_len):              # context keys, position c
        if c >= anchor:
            break
        if window is not None and q_pos - c >= window:
            continue
        visible.add(c)
    block_first = ctx_len + j * block_size
    for t in range(block_size):           # keys of the query's own block
        if in_block_causal and t > i:
            continue
        if window is not None and i - t >= window:
            continue
        visible.add(block_first + t)
    return k in visible


def spec_generate_keep_mask(ctx_lens, ctx_len: int, block_size: int, in_block_causal: bool,
                            window) -> np.ndarray:
    """Keep mask ``[B, block_size, ctx_len + block_size]`` of DFlash inference
    (``spec_generate``): one draft block placed after each row's context.

    SpecForge PR #905 (Motivation list and the maintainer's split note, item
    2/3) moves the mask builders to a module shared by training and inference
    and adds default masks for ``spec_generate``; the plainest reading is the
    training rule above with a single block whose anchor is the row's context
    length ``ctx_lens[b] <= ctx_len`` (keys ``[ctx_lens[b], ctx_len)`` are
    padding and never kept)."""
    anchors = np.asarray(ctx_lens).reshape(-1, 1)
    return dflash_keep_mask(anchors, ctx_len, block_size, in_block_causal, window)
