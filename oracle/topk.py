"""Dynamic top-k keep mask from an attention bias.

Test infrastructure only (see ``oracle/__init__.py``).

Source: flash-sparse-attention PR #197 "Centralize dynamic mask creation for
FDMA".  Design: ``dynamic_mask`` selects the top ``window_size`` entries of
the bias along the key axis after an optional pre-mask has set invalid
positions to a minimum sentinel, and ``create_mask`` first brings a 2D
``(batch, seq_len)`` or 4D pre-mask to the bias shape.  Implementation
Notes: invalid positions are set to the sentinel before the selection so they
are never selected; a 2D mask of length key_len becomes ``(B, 1, 1, K)``, one
of length query_len is padded or cut to key_len.  Changes: the sentinel is
the minimum finite value of the *bias* dtype.

Readings where the pages are silent or loose:
* only columns ``k < Lk`` take part; padded columns are never selected;
* equal values are ordered by lower key index first (the page's selection is
  unsorted, so ties are left open there); ``-0.0 == +0.0``;
* the result is ``selected and pre_mask``, so a masked position is never kept
  even when fewer than ``window_size`` positions are valid;
* ``window_size >= Lk`` selects every column, so the result is the pre-mask;
* a 2D pre-mask of length query_len is padded with False (invalid).
"""
from __future__ import annotations

import numpy as np

# Minimum finite values of the bias dtypes (numpy/torch finfo(...).min).
FINFO_MIN = {
    "bf16": -3.3895313892515355e38,   # -(2 - 2**-7) * 2**127
    "fp16": -65504.0,                 # -(2 - 2**-10) * 2**15
    "fp32": float(np.finfo(np.float32).min),
}


def normalize_pre_mask(pre_mask: np.ndarray, batch: int, n_q: int, n_k: int) -> np.ndarray:
    """``create_mask``'s shape step: return a 4D bool array whose last dim is
    ``n_k`` and whose other dims broadcast against the bias."""
    m = np.asarray(pre_mask, dtype=bool)
    if m.ndim == 2:
        if m.shape[0] != batch:
            raise ValueError("2D pre-mask must be (batch, seq_len)")
        if m.shape[1] == n_k:
            col = m
        elif m.shape[1] == n_q:
            col = np.zeros((batch, n_k), dtype=bool)
            w = min(n_q, n_k)
            col[:, :w] = m[:, :w]
        else:
            raise ValueError("2D pre-mask length must be key_len or query_len")
        return col[:, None, None, :]
    if m.ndim == 4:
        if m.shape[-1] < n_k:
            out = np.zeros(m.shape[:-1] + (n_k,), dtype=bool)
            out[..., : m.shape[-1]] = m
            return out
        return m[..., :n_k]
    raise ValueError("pre-mask must be 2D or 4D")


def dynamic_topk_keep(bias: np.ndarray, n_k: int, pre_mask, window_size: int,
                      sentinel: float) -> np.ndarray:
    """Keep mask of the bias's full shape (last dim = padded K).

    bias: ``[b, h, q, K]`` float array holding the exact bias values
        (``K >= n_k``).
    pre_mask: None or a 4D bool array broadcastable to ``bias[..., :n_k]``.
    sentinel: the bias dtype's minimum finite value.
    """
    bias = np.asarray(bias, dtype=np.float64)
    if bias.ndim != 4:
        raise ValueError("bias must be 4D")
    if window_size < 1:
        raise ValueError("window_size must be >= 1")
    shape = bias.shape
    valid = bias[..., :n_k]
    if pre_mask is None:
        pm = np.ones(valid.shape, dtype=bool)
    else:
        pm = np.broadcast_to(np.asarray(pre_mask, dtype=bool)[..., :n_k], valid.shape)
    vals = np.where(pm, valid, sentinel).reshape(-1, n_k)
    vals = vals + 0.0                     # -0.0 -> +0.0, so signed zeros tie
    n_take = min(window_size, n_k)
    idx = np.broadcast_to(np.arange(n_k), vals.shape)
    order = np.lexsort((idx, -vals), axis=-1)        # value desc, index asc
    taken = np.zeros(vals.shape, dtype=bool)
    np.put_along_axis(taken, order[:, :n_take], True, axis=-1)
    keep_valid = taken.reshape(valid.shape) & pm
    out = np.zeros(shape, dtype=bool)
    out[..., :n_k] = keep_valid
    return out
