"""GPU: the backward kernels on launches where every persistent CTA runs at
least two work units, against the float64 oracle's gradients.

A backward work unit is one (batch, KV head, 128-key tile); the launch
starts min(units, SM count) CTAs and each CTA walks units
``blockIdx.x, blockIdx.x + gridDim.x, ...``.  With at least twice as many
units as SMs (B200: 148), every CTA carries its mbarrier phases, its TMEM
accumulators and its outstanding dQ bulk reductions from one unit into the
next, which small cases never exercise.  The cases are the training DFlash
workload itself (B=2, H=32, KVH=8, d=128, 4096 + 4096 keys: 1024 units), an
explicit mask + query-broadcast bias with dbias, packed sequences, and head
dim 64.

Full-size gradients are checked exactly where the oracle can afford them:
dK and dV of whole KV heads (every key of the head, summed over every query
of its head group) and dQ of every query of those groups' heads.  The DFlash
mask is the same for every head, so one KV head's group is a self-contained
problem for the oracle.

Source: flash-sparse-attention PR #190, Changes (mha_bwd: dQ, dK, dV and a
dbias reduced over the broadcast dims).
"""
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

# Gradient agreement (bf16 operands, fp32 accumulation), as for the small
# backward cases: relative to m = max(1, max |ref|) of each tensor,
# max-abs <= 2.5e-2 m and mean-abs <= 2.5e-3 m.
GRAD_TOL = (2.5e-2, 2.5e-3)
MIN_UNITS_PER_CTA = 2


def _close(name, got, ref):
    g = f64(got) if isinstance(got, torch.Tensor) else got
    m = max(1.0, float(np.abs(ref).max()))
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= GRAD_TOL[0] * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= GRAD_TOL[1] * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


def _sms() -> int:
    return torch.cuda.get_device_properties(0).multi_processor_count


def _assert_multi_unit(n_units: int):
    assert n_units >= MIN_UNITS_PER_CTA * _sms(), f"{n_units} units do not give every CTA two"


def _group(t, b, hk, group):
    """[1, L, group, d] slice of the query heads of KV head hk in batch b."""
    return t[b:b + 1, :, hk * group:(hk + 1) * group]


@pytest.mark.parametrize("w", [wl.DFLASH_TRAIN_FULL, wl.DFLASH_TRAIN_SLIDING], ids=lambda w: w.name)
def test_dflash_training_backward_full_size(w):
    q, k, v, anchors = wl.dflash_inputs(w)
    do = wl.normal(wl.rng_for(w.seed + 500), tuple(q.shape), w.dtype)
    _assert_multi_unit(w.batch * w.kv_heads * -(-w.n_k // 128))
    qc, kc, vc, dc, ac = (t.cuda() for t in (q, k, v, do, anchors))
    args = (ac, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window)
    out, lse = sma.dfa_attn_fwd(qc, kc, vc, *args)
    dq, dk, dv = sma.dfa_attn_bwd(qc, kc, vc, out, lse, dc, *args)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    causal = dm.resolve_in_block_causal(w.is_causal, w.layer_type)
    win = dm.resolve_window(w.layer_type, w.sliding_window) if w.layer_type == dm.LAYER_SLIDING else None
    a = anchors.numpy()
    group = w.heads // w.kv_heads
    for b, hk in [(0, 3), (1, 0), (1, w.kv_heads - 1)]:
        def keep_rows(_b, q0, q1, b=b):
            return dm.dflash_keep_rows(a[b:b + 1], w.ctx_len, w.block_size, causal, win, q0, q1)

        rq, rk, rv, _ = ag.attention_grad(f64(_group(q, b, hk, group)), f64(k[b:b + 1, :, hk:hk + 1]),
                                          f64(v[b:b + 1, :, hk:hk + 1]), f64(_group(do, b, hk, group)),
                                          keep_rows=keep_rows, workers=at.host_threads())
        tag = f"b{b} kvh{hk}"
        _close(f"dk {tag}", dk[b:b + 1, :, hk:hk + 1], rk)
        _close(f"dv {tag}", dv[b:b + 1, :, hk:hk + 1], rv)
        _close(f"dq {tag}", _group(dq, b, hk, group), rq)


@pytest.mark.parametrize("D", [64, 128])
def test_explicit_backward_with_dbias_many_units(D):
    """B=4, H=16, KVH=8, Lq=1000, Lk=1300 (11 key tiles: 352 units); a
    per-(batch, query) random mask, bottom-right causal, and a bias
    broadcast over the queries, shape (B, KVH, 1, K), whose dbias sums dS
    over each group's heads and every query."""
    B, H, KVH, LQ, LK = 4, 16, 8, 1000, 1300
    KP = sma.round_up_k(LK)
    _assert_multi_unit(B * KVH * -(-LK // 128))
    rng = wl.rng_for(70 + D)
    q = wl.normal(rng, (B, LQ, H, D), "bf16")
    k = wl.normal(rng, (B, LK, KVH, D), "bf16")
    v = wl.normal(rng, (B, LK, KVH, D), "bf16")
    do = wl.normal(rng, (B, LQ, H, D), "bf16")
    mask = torch.from_numpy(rng.random((B, 1, LQ, KP)) < 0.85)
    bias = wl.normal(rng, (B, KVH, 1, KP), "bf16")
    qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, mask, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, True)
    dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, True, return_dbias=True)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    keep = at.aux_view(mask.numpy(), H, KVH, LK) & at.causal_keep(LQ, LK)[None, None]
    bb = at.aux_view(f64(bias), H, KVH, LK)
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, bias=bb,
                                        dbias_shape=tuple(bias.shape), workers=at.host_threads())
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)
    _close("dbias", db, rdb)
    assert (db[..., LK:] == 0).all()


def test_dflash_backward_head_dim_64_many_units():
    """Head dim 64 (its own backward kernel): B=2, H=16, KVH=8, 2048 context
    keys and 128 blocks of 16 (32 key tiles: 512 units), sliding layer with
    in-block causality and a window of 700."""
    B, H, KVH, D, Lc, N, bs, W = 2, 16, 8, 64, 2048, 128, 16, 700
    rng = wl.rng_for(80)
    nq, lk = N * bs, Lc + N * bs
    _assert_multi_unit(B * KVH * -(-lk // 128))
    q = wl.normal(rng, (B, nq, H, D), "bf16")
    k = wl.normal(rng, (B, lk, KVH, D), "bf16")
    v = wl.normal(rng, (B, lk, KVH, D), "bf16")
    do = wl.normal(rng, (B, nq, H, D), "bf16")
    anchors = wl.sorted_anchors(rng, B, N, Lc)
    qc, kc, vc, dc, ac = (t.cuda() for t in (q, k, v, do, anchors))
    out, lse = sma.dfa_attn_fwd(qc, kc, vc, ac, Lc, bs, None, 1, W)
    dq, dk, dv = sma.dfa_attn_bwd(qc, kc, vc, out, lse, dc, ac, Lc, bs, None, 1, W)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    causal = dm.resolve_in_block_causal(None, 1)
    win = dm.resolve_window(1, W)
    a = anchors.numpy()
    group = H // KVH
    for b, hk in [(0, 0), (1, 5)]:
        def keep_rows(_b, q0, q1, b=b):
            return dm.dflash_keep_rows(a[b:b + 1], Lc, bs, causal, win, q0, q1)

        rq, rk, rv, _ = ag.attention_grad(f64(_group(q, b, hk, group)), f64(k[b:b + 1, :, hk:hk + 1]),
                                          f64(v[b:b + 1, :, hk:hk + 1]), f64(_group(do, b, hk, group)),
                                          keep_rows=keep_rows, workers=at.host_threads())
        _close(f"dk b{b} kvh{hk}", dk[b:b + 1, :, hk:hk + 1], rk)
        _close(f"dv b{b} kvh{hk}", dv[b:b + 1, :, hk:hk + 1], rv)
        _close(f"dq b{b} kvh{hk}", _group(dq, b, hk, group), rq)


@pytest.mark.parametrize("D,causal", [(128, True), (64, False)])
def test_varlen_backward_many_units(D, causal):
    """Eight packed sequences of 333..2100 tokens (71 key tiles over 8 KV
    heads: 568 units), each against the float64 gradients of the sequence
    on its own."""
    H, KVH = 16, 8
    lens = [1500, 900, 2100, 640, 1300, 333, 777, 1024]
    n_units = KVH * sum(-(-n // 128) for n in lens)
    _assert_multi_unit(n_units)
    rng = wl.rng_for(90 + D)
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    total = int(cu[-1])
    q = wl.normal(rng, (total, H, D), "bf16")
    k = wl.normal(rng, (total, KVH, D), "bf16")
    v = wl.normal(rng, (total, KVH, D), "bf16")
    do = wl.normal(rng, (total, H, D), "bf16")
    cuc = torch.from_numpy(cu).cuda()
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = sma.varlen_attn_fwd(qc, kc, vc, cuc, cuc, max(lens), max(lens), causal)
    dq, dk, dv = sma.varlen_attn_bwd(qc, kc, vc, out, lse, dc, cuc, cuc, max(lens), max(lens), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    rq = np.zeros(tuple(q.shape))
    rk = np.zeros(tuple(k.shape))
    rv = np.zeros(tuple(k.shape))
    for i in range(len(lens)):
        a0, a1 = int(cu[i]), int(cu[i + 1])
        keep = at.causal_keep(a1 - a0, a1 - a0)[None, None] if causal else None
        gq, gk, gv, _ = ag.attention_grad(f64(q[a0:a1])[None], f64(k[a0:a1])[None], f64(v[a0:a1])[None],
                                          f64(do[a0:a1])[None], keep=keep, workers=at.host_threads())
        rq[a0:a1], rk[a0:a1], rv[a0:a1] = gq[0], gk[0], gv[0]
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)
