"""Gradients of dense float64 softmax attention: the backward of
``oracle.attention.attention`` for an upstream gradient ``dO``.

Test infrastructure only (see ``oracle/__init__.py``).

With the forward's definitions (s = scale * <Q, K> + bias on kept keys,
P = softmax over the kept keys of each row, O = P V), the chain rule gives,
per batch b and query head h with KV head hk:

    dP[q, k]  = <dO[q], V[k]>
    D[q]      = <dO[q], O[q]>            (= sum_k P[q, k] dP[q, k])
    dS[q, k]  = P[q, k] * (dP[q, k] - D[q])        (gradient of s)
    dQ[q]     = scale * sum_k dS[q, k] K[k]
    dK[k]    += scale * sum_q dS[q, k] Q[q]        (summed over the heads of hk)
    dV[k]    += sum_q P[q, k] dO[q]                (summed over the heads of hk)
    dbias    += dS                                 (summed over the bias's broadcast dims)

Masked pairs have P = 0 and so contribute nothing; a fully masked row
contributes nothing at all.

Sources: flash-sparse-attention PR #190 "Broadcastable 4D mask/bias, ...",
Changes section (mha_bwd): the backward returns dQ, dK, dV and a dbias that
is reduced over the head groups, the batch and the query dim wherever the
bias broadcasts along them, with its key dim rounded up to 128 and only the
first Lk columns meaningful.  The formulas are the textbook derivative of
softmax attention, written out; no page prints them.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .attention import default_scale


def _probs(q, k, b, h, q0, q1, group, scale, keep, keep_rows, bias):
    """Scores and normalised probabilities of rows q0:q1 (dead rows all 0)."""
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
    p = np.exp(s - np.where(dead, 0.0, m)[:, None])
    p = p / np.where(dead, 1.0, p.sum(axis=1))[:, None]
    p[dead] = 0.0
    return p


def _one_task(q, k, v, do, b, h, q0, q1, group, scale, keep, keep_rows, bias):
    hk = h // group
    p = _probs(q, k, b, h, q0, q1, group, scale, keep, keep_rows, bias)
    vv = v[b, :, hk, :]
    g = do[b, q0:q1, h, :]
    o = p @ vv
    dp = g @ vv.T
    dd = (g * o).sum(axis=1)
    ds = p * (dp - dd[:, None])
    dq = scale * (ds @ k[b, :, hk, :])
    dk = scale * (ds.T @ q[b, q0:q1, h, :])
    dv = p.T @ g
    return b, h, q0, q1, dq, dk, dv, ds


def attention_grad(q, k, v, do, *, keep=None, keep_rows=None, bias=None, scale=None,
                   row_chunk: int = 256, workers: int = 1, dbias_shape=None):
    """Backward of dense attention in float64.

    q, do: ``[B, Lq, H, d]``; k, v: ``[B, Lk, KVH, d]``.  keep / keep_rows /
    bias / scale as in ``attention``.  ``dbias_shape``: the 4D shape of the
    bias as the caller holds it ``(b', h', q', K)`` with ``K >= Lk`` or
    ``K == 1``; dbias is reduced onto that shape (columns >= Lk are 0; a key
    dim of 1, one bias value for every key, sums dS over the keys as well).
    A head dim equal to KVH (when KVH != H) sums the heads of each group.
    Returns ``dq [B, Lq, H, d], dk [B, Lk, KVH, d], dv [B, Lk, KVH, d]`` and
    ``dbias`` (None without ``dbias_shape``).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    n_b, n_q, n_h, d = q.shape
    n_k, n_kvh = k.shape[1], k.shape[2]
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
    rows = [(r, min(r + row_chunk, n_q)) for r in range(0, n_q, row_chunk)]
    tasks = [(b, h, q0, q1) for b in range(n_b) for h in range(n_h) for (q0, q1) in rows]

    def run(t):
        return _one_task(q, k, v, do, *t, group, scale, keep, keep_rows, bias)

    if workers > 1:
        with ThreadPoolExecutor(max_workers=workers) as pool:
            results = list(pool.map(run, tasks))
    else:
        results = [run(t) for t in tasks]

    dq = np.zeros_like(q)
    dk = np.zeros((n_b, n_k, n_kvh, d))
    dv = np.zeros((n_b, n_k, n_kvh, d))
    dbias = None
    if dbias_shape is not None:
        sb, sh, sq, kk = dbias_shape
        if kk < n_k and kk != 1:
            raise ValueError("dbias key dim must be at least Lk, or 1")
        dbias = np.zeros(dbias_shape)
    for b, h, q0, q1, gq, gk, gv, ds in results:
        hk = h // group
        dq[b, q0:q1, h, :] = gq
        dk[b, :, hk, :] += gk
        dv[b, :, hk, :] += gv
        if dbias is not None:
            bi = b if sb > 1 else 0
            if sh == n_h:
                hi = h
            elif sh == n_kvh:
                hi = hk
            else:
                hi = 0
            if kk == 1 and n_k > 1:           # one bias value for every key
                ds = ds.sum(axis=1, keepdims=True)
            if sq > 1:
                dbias[bi, hi, q0:q1, :ds.shape[1]] += ds
            else:
                dbias[bi, hi, 0, :ds.shape[1]] += ds.sum(axis=0)
    return dq, dk, dv, dbias
