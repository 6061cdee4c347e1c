"""Shared helpers of the GPU parity tests (comparison rules, oracle calls)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as at
from oracle import dflash_mask as dm
from oracle import tiles as tl

# Agreement required of attention outputs (the library's stated accuracy;
# the pages fix none): bf16/fp16 inputs max-abs <= 2e-2 and mean-abs <= 2e-3;
# fp32 inputs max-abs <= 1e-4.
TOL = {torch.bfloat16: (2e-2, 2e-3), torch.float16: (2e-2, 2e-3), torch.float32: (1e-4, 1e-4)}
# log-sum-exp is compared with the same absolute bounds scaled by 5 (lse is
# O(log Lk) in magnitude, computed in fp32 from bf16-rounded scores).
LSE_TOL = {torch.bfloat16: 1e-1, torch.float16: 1e-1, torch.float32: 1e-4}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def assert_attention_close(out_gpu, lse_gpu, out_ref, lse_ref, dtype, rows=None, what=""):
    """Element-wise comparison against the oracle; ``rows`` restricts the
    comparison to sampled query rows (a list of (q0, q1))."""
    o = f64(out_gpu)
    if rows is not None:
        sel = np.concatenate([np.arange(a, b) for a, b in rows])
        o = o[:, sel]
        out_ref = out_ref[:, sel]
        if lse_gpu is not None:
            lse_ref = lse_ref[:, :, sel]
    max_abs_tol, mean_abs_tol = TOL[dtype]
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.abs(o - out_ref)
    assert err.max() <= max_abs_tol, f"{what}: max abs err {err.max():.3e} > {max_abs_tol}"
    assert err.mean() <= mean_abs_tol, f"{what}: mean abs err {err.mean():.3e} > {mean_abs_tol}"
    if lse_gpu is not None:
        l = f64(lse_gpu)
        if rows is not None:
            l = l[:, :, sel]
        dead = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(l), dead), f"{what}: -inf lse rows differ"
        if (~dead).any():
            lerr = np.abs(l[~dead] - lse_ref[~dead]).max()
            assert lerr <= LSE_TOL[dtype], f"{what}: lse err {lerr:.3e}"


def masked_oracle(q, k, v, mask, bias, causal, rows=None, workers=8):
    """Dense definition of attention under the 4D mask/bias contract (the
    keep set is mask AND k < Lk AND, if causal, k <= q + Lk - Lq)."""
    b, lq, h, d = q.shape
    lk, kvh = k.shape[1], k.shape[2]
    keep = at.aux_view(mask.cpu().numpy(), h, kvh, lk) if mask is not None else None
    if causal:
        ck = at.causal_keep(lq, lk)[None, None]
        keep = ck if keep is None else (keep & ck)
    bb = at.aux_view(f64(bias), h, kvh, lk) if bias is not None else None
    return at.attention(f64(q), f64(k), f64(v), keep=keep, bias=bb, rows=rows, workers=workers,
                        row_chunk=128)


def dflash_oracle(q, k, v, anchors, ctx_len, block_size, is_causal, layer_type, window, rows=None,
                  workers=8):
    causal = dm.resolve_in_block_causal(is_causal, layer_type)
    w = dm.resolve_window(layer_type, window) if layer_type == dm.LAYER_SLIDING else None
    a = anchors.cpu().numpy()

    def keep_rows(b, q0, q1):
        return dm.dflash_keep_rows(a[b:b + 1], ctx_len, block_size, causal, w, q0, q1)

    return at.attention(f64(q), f64(k), f64(v), keep_rows=keep_rows, rows=rows, workers=workers,
                        row_chunk=128)


def dflash_block_map_oracle(anchors, ctx_len, block_size, is_causal, layer_type, window):
    causal = dm.resolve_in_block_causal(is_causal, layer_type)
    w = dm.resolve_window(layer_type, window) if layer_type == dm.LAYER_SLIDING else None
    a = anchors.cpu().numpy()
    n_q = a.shape[1] * block_size
    n_k = ctx_len + n_q

    def keep_rows(b, q0, q1):
        return dm.dflash_keep_rows(a[b:b + 1], ctx_len, block_size, causal, w, q0, q1)[0]

    return tl.block_map_from_rows(keep_rows, a.shape[0], n_q, n_k)


def sample_tiles(n_q: int, picks=(0, 0.5, 1.0), tile: int = 128):
    """Row ranges of a few query tiles: first, middle, last (ragged tail)."""
    qt = -(-n_q // tile)
    out = []
    for f in picks:
        t = min(qt - 1, int(round(f * (qt - 1))))
        r = (t * tile, min((t + 1) * tile, n_q))
        if r not in out:
            out.append(r)
    return out
