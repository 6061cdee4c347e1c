"""GPU: packed sequences with a mask and / or bias in the padded
per-sequence layout (varlen_masked_attn_fwd / _bwd) agree with the float64
oracle: broadcast over sequences, heads (H or KVH) and queries, key dims
padded, exact or 1, causal per sequence; gradients dQ, dK, dV and dbias."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from oracle import attention_grad as ag
from tests._helpers import TOL, LSE_TOL, f64

pytestmark = pytest.mark.gpu

H, KVH = 8, 2
LQ = [200, 1, 130, 0, 77]
LK = [260, 40, 130, 5, 304]  # the longest a multiple of 8: rows of 16-byte multiples
MQ, MK = max(LQ), max(LK)
KP = sma.round_up_k(MK)
NB = len(LQ)


def _case(rng, D, dtype):
    cu_q = np.cumsum([0] + LQ).astype(np.int32)
    cu_k = np.cumsum([0] + LK).astype(np.int32)
    q = wl.normal(rng, (int(cu_q[-1]), H, D), dtype)
    k = wl.normal(rng, (int(cu_k[-1]), KVH, D), dtype)
    v = wl.normal(rng, (int(cu_k[-1]), KVH, D), dtype)
    return cu_q, cu_k, q, k, v


def _check_fwd(out, lse, ref_o, ref_l, dtype, what):
    tmax, tmean = TOL[dtype]
    err = np.abs(f64(out) - ref_o)
    assert err.max() <= tmax and err.mean() <= tmean, f"{what}: {err.max():.3e} {err.mean():.3e}"
    l = f64(lse)
    dead = np.isneginf(ref_l)
    assert np.array_equal(np.isneginf(l), dead), what
    if (~dead).any():
        assert np.abs(l[~dead] - ref_l[~dead]).max() <= LSE_TOL[dtype], what


CASES = [((NB, 1, 1, KP), None), ((1, H, MQ, KP), (NB, KVH, 1, KP)), (None, (1, 1, MQ, MK)),
         ((NB, KVH, MQ, MK), (NB, H, MQ, 1)), (None, (NB, KVH, 1, KP))]


@pytest.mark.parametrize("mshape,bshape", CASES, ids=str)
@pytest.mark.parametrize("D,dtype,causal", [(128, "bf16", True), (64, "bf16", False), (128, "fp16", False),
                                            (64, "fp32", True)])
def test_varlen_masked_forward(mshape, bshape, D, dtype, causal):
    rng = wl.rng_for(81)
    cu_q, cu_k, q, k, v = _case(rng, D, dtype)
    mask = torch.from_numpy(rng.random(mshape) < 0.75) if mshape else None
    bias = wl.normal(rng, bshape, dtype) if bshape else None
    out, lse = sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                   torch.from_numpy(cu_k).cuda(), MQ, MK, causal,
                                   mask=mask.cuda() if mask is not None else None,
                                   bias=bias.cuda() if bias is not None else None)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    ref_o, ref_l = at.varlen_attention(f64(q), f64(k), f64(v), cu_q, cu_k, causal,
                                       mask=mask.numpy() if mask is not None else None,
                                       bias=f64(bias) if bias is not None else None)
    _check_fwd(out, lse, ref_o, ref_l, q.dtype, f"{mshape} {bshape} D={D} {dtype}")


def _close_grad(name, got, ref, dtype):
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    tmax, tmean = (1e-4, 1e-5) if dtype == "fp32" else (2.5e-2, 2.5e-3)
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= tmax * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= tmean * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


@pytest.mark.parametrize("mshape,bshape", CASES[1:], ids=str)
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "bf16"), (64, "fp32")])
def test_varlen_masked_backward(mshape, bshape, D, dtype):
    rng = wl.rng_for(82)
    cu_q, cu_k, q, k, v = _case(rng, D, dtype)
    do = wl.normal(rng, tuple(q.shape), dtype)
    mask = torch.from_numpy(rng.random(mshape) < 0.75) if mshape else None
    bias = wl.normal(rng, bshape, dtype)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
    mc = mask.cuda() if mask is not None else None
    bc = bias.cuda()
    out, lse = sma.varlen_attn_fwd(qc, kc, vc, cq, ck, MQ, MK, True, mask=mc, bias=bc)
    dq, dk, dv, db = sma.varlen_attn_bwd(qc, kc, vc, out, lse, dc, cq, ck, MQ, MK, True, mask=mc, bias=bc,
                                         return_dbias=True)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    rq = np.zeros(tuple(q.shape))
    rk = np.zeros(tuple(k.shape))
    rv = np.zeros(tuple(k.shape))
    rdb = np.zeros(tuple(bias.shape))
    mn = mask.numpy() if mask is not None else None
    bn = f64(bias)
    for b in range(NB):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        lq, lk = q1 - q0, k1 - k0
        if lq == 0 or lk == 0:
            continue
        keep = at.causal_keep(lq, lk)[None, None]
        if mn is not None:
            keep = keep & at.varlen_seq_aux(mn, b, lq, lk, H, KVH).astype(bool)
        bseq = at.varlen_seq_aux(bn, b, lq, lk, H, KVH)
        dshape = (1, bias.shape[1], lq if bias.shape[2] > 1 else 1, lk if bias.shape[3] > 1 else 1)
        gq, gk, gv, gdb = ag.attention_grad(f64(q[q0:q1])[None], f64(k[k0:k1])[None], f64(v[k0:k1])[None],
                                            f64(do[q0:q1])[None], keep=keep, bias=bseq, dbias_shape=dshape)
        rq[q0:q1], rk[k0:k1], rv[k0:k1] = gq[0], gk[0], gv[0]
        bi = b if bias.shape[0] > 1 else 0
        rdb[bi, :, :dshape[2], :dshape[3]] += gdb[0]
    _close_grad("dq", dq, rq, dtype)
    _close_grad("dk", dk, rk, dtype)
    _close_grad("dv", dv, rv, dtype)
    _close_grad("dbias", db, rdb, dtype)
