"""GPU: dfa_attn_bwd / masked_attn_bwd (tcgen05 backward) agree with the
float64 oracle's gradients (oracle.attention_grad, pinned by finite
differences) under DFlash and explicit masks, grouped heads, ragged tiles,
and keys that no query attends."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from oracle import attention_grad as ag
from oracle import dflash_mask as dm
from tests._helpers import f64

pytestmark = pytest.mark.gpu

# Gradient agreement (bf16 / fp16 operands, fp32 accumulation): relative to
# the largest reference magnitude m = max(1, max |ref|) of each tensor,
# max-abs <= 2.5e-2 m and mean-abs <= 2.5e-3 m.
GRAD_TOL = (2.5e-2, 2.5e-3)


def _close(name, got, ref):
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= GRAD_TOL[0] * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= GRAD_TOL[1] * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


def _dflash_case(seed, B, H, KVH, D, Lc, N, bs, is_causal, layer, window, dtype="bf16"):
    rng = wl.rng_for(seed)
    nq, lk = N * bs, Lc + N * bs
    q = wl.normal(rng, (B, nq, H, D), dtype)
    k = wl.normal(rng, (B, lk, KVH, D), dtype)
    v = wl.normal(rng, (B, lk, KVH, D), dtype)
    do = wl.normal(rng, (B, nq, H, D), dtype)
    anchors = torch.from_numpy(np.sort(rng.integers(0, Lc + 1, size=(B, N)), axis=1).astype(np.int32))
    return q, k, v, do, anchors


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layer,is_causal,window", [(0, None, 0), (1, None, 40), (0, True, 0)], ids=str)
def test_dflash_backward(D, layer, is_causal, window):
    B, H, KVH, Lc, N, bs = 2, 4, 2, 300, 20, 16   # Nq 320, Lk 620: ragged query and key tiles
    q, k, v, do, anchors = _dflash_case(31, B, H, KVH, D, Lc, N, bs, is_causal, layer, window)
    qc, kc, vc, dc, ac = (t.cuda() for t in (q, k, v, do, anchors))
    out, lse = sma.dfa_attn_fwd(qc, kc, vc, ac, Lc, bs, is_causal, layer, window)
    dq, dk, dv = sma.dfa_attn_bwd(qc, kc, vc, out, lse, dc, ac, Lc, bs, is_causal, layer, window)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    causal = dm.resolve_in_block_causal(is_causal, layer)
    w = dm.resolve_window(layer, window) if layer == dm.LAYER_SLIDING else None
    keep = dm.dflash_keep_mask(anchors.numpy(), Lc, bs, causal, w)[:, None]
    rq, rk, rv, _ = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, workers=8)
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)


B, LQ, LK, H, KVH = 2, 300, 450, 8, 2
KP = sma.round_up_k(LK)


@pytest.mark.parametrize("mshape", [None, (1, 1, LQ, KP), (B, KVH, 1, KP), (B, H, LQ, KP)], ids=str)
@pytest.mark.parametrize("bshape", [None, (B, KVH, 1, KP)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_masked_backward(mshape, bshape, causal):
    rng = wl.rng_for(32)
    q = wl.normal(rng, (B, LQ, H, 128), "bf16")
    k = wl.normal(rng, (B, LK, KVH, 128), "bf16")
    v = wl.normal(rng, (B, LK, KVH, 128), "bf16")
    do = wl.normal(rng, (B, LQ, H, 128), "bf16")
    mask = torch.from_numpy(rng.random(mshape) < 0.7) if mshape else None
    bias = wl.normal(rng, bshape, "bf16") if bshape else None
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, do))
    mc = None if mask is None else mask.cuda()
    bc = None if bias is None else bias.cuda()
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, causal)
    dq, dk, dv = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    keep = at.aux_view(mask.numpy(), H, KVH, LK) if mask is not None else None
    if causal:
        ck = at.causal_keep(LQ, LK)[None, None]
        keep = ck if keep is None else (keep & ck)
    bb = at.aux_view(f64(bias), H, KVH, LK) if bias is not None else None
    rq, rk, rv, _ = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, bias=bb, workers=8)
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)


def test_unattended_keys_and_dead_rows():
    """Keys no query keeps get zero dK / dV; rows with no kept key give zero dQ."""
    rng = wl.rng_for(33)
    q = wl.normal(rng, (1, 200, 4, 128), "bf16")
    k = wl.normal(rng, (1, 500, 2, 128), "bf16")
    v = wl.normal(rng, (1, 500, 2, 128), "bf16")
    do = wl.normal(rng, (1, 200, 4, 128), "bf16")
    kp = sma.round_up_k(500)
    mask = torch.from_numpy(rng.random((1, 1, 200, kp)) < 0.5)
    mask[..., 128:300] = False           # a whole key tile and more unattended
    mask[0, 0, 7] = False                # a dead row
    qc, kc, vc, dc, mc = (t.cuda() for t in (q, k, v, do, mask))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, None, False)
    dq, dk, dv = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, None, False)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    assert (dk[:, 128:300] == 0).all() and (dv[:, 128:300] == 0).all()
    assert (dq[0, 7] == 0).all()
    rq, rk, rv, _ = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=mask.numpy()[..., :500], workers=8)
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)


def test_fp16_and_rejections():
    rng = wl.rng_for(34)
    q = wl.normal(rng, (1, 130, 2, 64), "fp16")
    k = wl.normal(rng, (1, 260, 1, 64), "fp16")
    v = wl.normal(rng, (1, 260, 1, 64), "fp16")
    do = wl.normal(rng, (1, 130, 2, 64), "fp16")
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, do))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, None, None, True)
    dq, dk, dv = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, None, None, True)
    torch.cuda.synchronize()
    rq, rk, rv, _ = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=at.causal_keep(130, 260)[None, None])
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)


def _close_fp32(name, got, ref):
    """fp32 FFMA gradients: max-abs <= 1e-4 m, mean-abs <= 1e-5 m (m as above)."""
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    err = np.abs(g - ref)
    assert err.max() <= 1e-4 * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= 1e-5 * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_masked_backward_with_bias_and_dbias(d):
    """fp32 inputs take the FFMA backward: explicit mask (PARTIAL tiles), a
    per-query-head bias (per-element dbias) and causal masking."""
    rng = wl.rng_for(37)
    q = wl.normal(rng, (B, LQ, H, d), "fp32")
    k = wl.normal(rng, (B, LK, KVH, d), "fp32")
    v = wl.normal(rng, (B, LK, KVH, d), "fp32")
    do = wl.normal(rng, (B, LQ, H, d), "fp32")
    mask = torch.from_numpy(rng.random((1, 1, LQ, KP)) < 0.7)
    bias = wl.normal(rng, (1, H, 1, KP), "fp32")
    qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, mask, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, True)
    dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, True, return_dbias=True)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    keep = at.aux_view(mask.numpy(), H, KVH, LK) & at.causal_keep(LQ, LK)[None, None]
    bb = at.aux_view(f64(bias), H, KVH, LK)
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, bias=bb,
                                        dbias_shape=tuple(bias.shape), workers=8)
    _close_fp32("dq", dq, rq)
    _close_fp32("dk", dk, rk)
    _close_fp32("dv", dv, rv)
    _close_fp32("dbias", db, rdb)


def test_fp32_dflash_backward():
    """fp32 inputs, DFlash sliding layer (in-block causal, window 40)."""
    Lc, bs = 200, 16
    q, k, v, do, anchors = _dflash_case(38, 2, 4, 2, 64, Lc, 12, bs, None, 1, 40, "fp32")
    causal = dm.resolve_in_block_causal(None, 1)
    w = dm.resolve_window(1, 40)
    qc, kc, vc, dc, ac = (t.cuda() for t in (q, k, v, do, anchors))
    out, lse = sma.dfa_attn_fwd(qc, kc, vc, ac, Lc, bs, None, 1, 40)
    dq, dk, dv = sma.dfa_attn_bwd(qc, kc, vc, out, lse, dc, ac, Lc, bs, None, 1, 40)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    keep = dm.dflash_keep_mask(anchors.numpy(), Lc, bs, causal, w)[:, None]
    rq, rk, rv, _ = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, workers=8)
    _close_fp32("dq", dq, rq)
    _close_fp32("dk", dk, rk)
    _close_fp32("dv", dv, rv)


DB_SHAPES = [(B, H, LQ, KP), (B, KVH, LQ, KP), (1, 1, LQ, KP), (B, H, 1, KP), (1, KVH, 1, KP),
             (1, 1, 1, KP)]


@pytest.mark.parametrize("bshape", DB_SHAPES, ids=str)
@pytest.mark.parametrize("D", [64, 128])
def test_masked_backward_dbias(bshape, D):
    """The bias gradient dS summed over every dim the bias broadcasts along
    (batch, the heads of a group or all heads, the queries), against the
    oracle's reduction onto the bias shape; padded key columns stay 0."""
    rng = wl.rng_for(35)
    q = wl.normal(rng, (B, LQ, H, D), "bf16")
    k = wl.normal(rng, (B, LK, KVH, D), "bf16")
    v = wl.normal(rng, (B, LK, KVH, D), "bf16")
    do = wl.normal(rng, (B, LQ, H, D), "bf16")
    mask = torch.from_numpy(rng.random((B, KVH, 1, KP)) < 0.8)
    bias = wl.normal(rng, bshape, "bf16")
    qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, mask, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, True)
    dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, True, return_dbias=True)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    assert db.shape == bias.shape and db.dtype == torch.float32
    keep = at.aux_view(mask.numpy(), H, KVH, LK) & at.causal_keep(LQ, LK)[None, None]
    bb = at.aux_view(f64(bias), H, KVH, LK)
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, bias=bb,
                                        dbias_shape=bshape, workers=8)
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)
    _close("dbias", db, rdb)
    assert (db[..., LK:] == 0).all()


def test_dbias_fp16_per_query_bias_and_rejection():
    rng = wl.rng_for(36)
    q = wl.normal(rng, (1, 130, 4, 128), "fp16")
    k = wl.normal(rng, (1, 260, 2, 128), "fp16")
    v = wl.normal(rng, (1, 260, 2, 128), "fp16")
    do = wl.normal(rng, (1, 130, 4, 128), "fp16")
    kp = sma.round_up_k(260)
    bias = wl.normal(rng, (1, 4, 130, kp), "fp32")
    qc, kc, vc, dc, bc = (t.cuda() for t in (q, k, v, do, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, None, bc, False)
    dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, None, bc, False, return_dbias=True)
    torch.cuda.synchronize()
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), bias=f64(bias)[..., :260],
                                        dbias_shape=tuple(bias.shape))
    _close("dbias", db, rdb)
    _close("dq", dq, rq)
    with pytest.raises(ValueError, match="needs a bias"):
        sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, None, None, False, return_dbias=True)
