"""Dense float64 softmax attention with an explicit keep mask and additive bias.

Test infrastructure only (see ``oracle/__init__.py``).

This is the plain definition that every attention entry point of the library
reaches by a faster route (skipping empty tiles, online softmax):

    s[k]  = scale * <Q[b, q, h], K[b, k, hk]> + bias[b?, h?, q?, k]
    keep  = mask[b?, h?, q?, k]  and  k < Lk  and  (causal -> k <= q + Lk - Lq)
    p     = exp(s - max_kept s) / sum_kept exp(s - max_kept s)
    O     = sum_kept p[k] V[b, k, hk]
    lse   = max + log(sum exp(s - max))          (natural log)

with ``hk = h // (H // KVH)`` (contiguous query-head groups) and a fully
masked row giving ``O = 0`` and ``lse = -inf``.

Sources: flash-sparse-attention PR #190 "Broadcastable 4D mask/bias, ...",
Design section: boolean mask with True = keep, floating bias added to the
scores, aux tensors of shape ({B|1}, {H|KVH|1}, {Lq|1}, round128(Lk)) of which
only the first Lk columns carry meaning.  The causal alignment for Lq != Lk is
bottom-right (the FlashAttention convention that page's ``mha_fwd`` API
follows); the pages say only "causal/non-causal".  A fully masked row is
defined as zero output rather than NaN, following the same page's stated aim
of preventing NaNs.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def causal_keep(n_q: int, n_k: int) -> np.ndarray:
    """Bottom-right aligned causal keep mask ``[n_q, n_k]``: key k visible to
    query q iff ``k <= q + n_k - n_q``."""
    q = np.arange(n_q)[:, None]
    k = np.arange(n_k)[None, :]
    return k <= q + (n_k - n_q)


def aux_view(aux: np.ndarray, n_heads: int, n_kv_heads: int, n_k: int) -> np.ndarray:
    """Turn a 4D mask/bias of the broadcast contract into an array that numpy
    broadcasts against ``[B, H, Lq, Lk]``.

    ``aux`` has shape ``(b', h', q', K)`` with ``K >= n_k`` (the padded
    ``round_up(n_k, 128)`` or ``n_k`` itself), of which only the first ``n_k``
    columns are used, or ``K == 1``: one value for every key, expanded over
    the ``n_k`` keys as the page's interface expands a key dim of 1.  A head
    dim equal to ``n_kv_heads`` (and not to ``n_heads``) is indexed with the
    query head's KV head ``h // (H // KVH)``; size-1 dims broadcast.
    """
    if aux.ndim != 4:
        raise ValueError("mask/bias must be 4D")
    if aux.shape[-1] == 1:
        x = np.broadcast_to(aux, aux.shape[:-1] + (n_k,))
    elif aux.shape[-1] >= n_k:
        x = aux[..., :n_k]
    else:
        raise ValueError("mask/bias key dim must be >= Lk or 1")
    h_aux = x.shape[1]
    if h_aux not in (1, n_heads, n_kv_heads):
        raise ValueError("mask/bias head dim must be 1, H or KVH")
    if h_aux != n_heads and h_aux == n_kv_heads and h_aux != 1:
        x = np.repeat(x, n_heads // n_kv_heads, axis=1)
    return x


def _one_task(q, k, v, b, h, q0, q1, group, scale, keep, keep_rows, bias):
    hk = h // group
    s = (q[b, q0:q1, h, :] @ k[b, :, hk, :].T) * scale
    if bias is not None:
        bb = bias[b if bias.shape[0] > 1 else 0, h if bias.shape[1] > 1 else 0]
        s = s + (bb[q0:q1] if bb.shape[0] > 1 else bb)
    kp = None
    if keep is not None:
        kk = keep[b if keep.shape[0] > 1 else 0, h if keep.shape[1] > 1 else 0]
        kp = kk[q0:q1] if kk.shape[0] > 1 else kk
    if keep_rows is not None:
        kr = keep_rows(b, q0, q1)
        kr = kr[h if kr.shape[0] > 1 else 0]
        kp = kr if kp is None else (kp & kr)
    if kp is not None:
        s = np.where(kp, s, -np.inf)
    m = s.max(axis=1)
    dead = m == -np.inf
    m_safe = np.where(dead, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    l = p.sum(axis=1)
    o = (p @ v[b, :, hk, :]) / np.where(dead, 1.0, l)[:, None]
    o[dead] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(dead, -np.inf, m_safe + np.log(np.where(dead, 1.0, l)))
    return b, h, q0, q1, o, lse


def attention(q, k, v, *, keep=None, keep_rows=None, bias=None, scale=None,
              row_chunk: int = 256, workers: int = 1, rows=None):
    """Dense attention in float64.

    q: ``[B, Lq, H, d]``; k, v: ``[B, Lk, KVH, d]`` (any float dtype, upcast).
    keep: bool array broadcastable to ``[B, H, Lq, Lk]`` (after ``aux_view``)
        or None for "all kept".
    keep_rows: optional callable ``(b, q0, q1) -> bool [H or 1, q1-q0, Lk]``
        producing keep rows on demand (used for masks too large to hold).
    bias: float array broadcastable to ``[B, H, Lq, Lk]`` or None.
    rows: optional iterable of ``(q0, q1)`` row ranges to compute (others are
        left as NaN) -- used to evaluate a sample of a large problem.
    Returns ``out [B, Lq, H, d]`` and ``lse [B, H, Lq]`` as float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_b, n_q, n_h, d = q.shape
    n_kvh = k.shape[2]
    if n_h % n_kvh:
        raise ValueError("H must be a multiple of KVH")
    group = n_h // n_kvh
    if scale is None:
        scale = default_scale(d)
    if keep is not None:
        keep = np.asarray(keep, dtype=bool)
        while keep.ndim < 4:
            keep = keep[None]
    if bias is not None:
        bias = np.asarray(bias, dtype=np.float64)
        while bias.ndim < 4:
            bias = bias[None]
    if rows is None:
        rows = [(r, min(r + row_chunk, n_q)) for r in range(0, n_q, row_chunk)]
    else:
        split = []
        for q0, q1 in rows:
            split += [(r, min(r + row_chunk, q1)) for r in range(q0, q1, row_chunk)]
        rows = split
    out = np.full((n_b, n_q, n_h, d), np.nan)
    lse = np.full((n_b, n_h, n_q), np.nan)
    tasks = [(b, h, q0, q1) for b in range(n_b) for h in range(n_h) for (q0, q1) in rows]

    def run(t):
        return _one_task(q, k, v, *t, group, scale, keep, keep_rows, bias)

    if workers > 1:
        with ThreadPoolExecutor(max_workers=workers) as pool:
            results = list(pool.map(run, tasks))
    else:
        results = [run(t) for t in tasks]
    for b, h, q0, q1, o, l in results:
        out[b, q0:q1, h, :] = o
        lse[b, h, q0:q1] = l
    return out, lse


def varlen_seq_aux(aux, b: int, lq: int, lk: int, n_heads: int, n_kv_heads: int):
    """Sequence b's part of a mask / bias given in the padded per-sequence
    layout ``(b', h', q', K)`` (reading R33 of the packed path): batch row b
    (or the only one), query rows ``[0, lq)`` (or the only one) and key
    columns ``[0, lk)``, as an array broadcasting against ``[1, H, lq, lk]``."""
    a = np.asarray(aux)
    a = a[b:b + 1] if a.shape[0] > 1 else a
    a = a[:, :, :lq] if a.shape[2] > 1 else a
    if a.shape[-1] > 1:
        a = a[..., :lk]
    return aux_view(a, n_heads, n_kv_heads, lk)


def varlen_attention(q, k, v, cu_q, cu_k, causal: bool = False, scale=None, mask=None, bias=None):
    """Packed variable-length sequences: sequence b is rows ``cu_q[b]:cu_q[b+1]``
    of q (``[total_q, H, d]``) and ``cu_k[b]:cu_k[b+1]`` of k / v and attends
    only its own keys, bottom-right causal within the sequence when ``causal``,
    and, when given, the keys its part of ``mask`` keeps, with its part of
    ``bias`` added (both in the padded per-sequence layout, ``varlen_seq_aux``).

    The packed form behind flash-sparse-attention PR #197's varlen function
    and pad / unpad helpers (Changes list); each sequence is the dense
    attention above.  Returns ``out [total_q, H, d]`` and ``lse [H, total_q]``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_heads, n_kv = q.shape[1], k.shape[1]
    out = np.zeros(q.shape)
    lse = np.full((q.shape[1], q.shape[0]), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        lq, lk = q1 - q0, k1 - k0
        keep = causal_keep(lq, lk)[None, None] if causal else None
        if mask is not None:
            m = varlen_seq_aux(mask, b, lq, lk, n_heads, n_kv).astype(bool)
            keep = m if keep is None else (keep & m)
        bb = varlen_seq_aux(bias, b, lq, lk, n_heads, n_kv).astype(np.float64) if bias is not None else None
        o, l = attention(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], keep=keep, bias=bb, scale=scale)
        out[q0:q1] = o[0]
        lse[:, q0:q1] = l[0]
    return out, lse


def host_threads() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
