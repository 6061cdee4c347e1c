"""GPU: varlen_attn_fwd / varlen_attn_bwd (packed variable-length sequences:
bf16 / fp16 on the tensor-core kernels, fp32 on the FFMA kernels) agree with
the float64 oracle; pad / unpad are exact inverses;
malformed offsets are reported without writing outside the tensors."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from tests._helpers import TOL, LSE_TOL, f64

pytestmark = pytest.mark.gpu


def _case(rng, lq, lk, H, KVH, D, dtype="bf16"):
    cu_q = np.cumsum([0] + lq).astype(np.int32)
    cu_k = np.cumsum([0] + lk).astype(np.int32)
    q = wl.normal(rng, (int(cu_q[-1]), H, D), dtype)
    k = wl.normal(rng, (int(cu_k[-1]), KVH, D), dtype)
    v = wl.normal(rng, (int(cu_k[-1]), KVH, D), dtype)
    return cu_q, cu_k, q, k, v


def _check(out, lse, ref_o, ref_l, dtype, what):
    o = f64(out)
    tmax, tmean = TOL[dtype]
    err = np.abs(o - ref_o)
    assert err.max() <= tmax and err.mean() <= tmean, f"{what}: {err.max():.3e} {err.mean():.3e}"
    l = f64(lse)
    dead = np.isneginf(ref_l)
    assert np.array_equal(np.isneginf(l), dead), what
    if (~dead).any():
        assert np.abs(l[~dead] - ref_l[~dead]).max() <= LSE_TOL[dtype], what


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_varlen_ragged(causal, D):
    """Lengths spanning several tiles, a ragged tail, a single-token and an
    empty sequence, and (causal) query-longer-than-key rows with no key."""
    rng = wl.rng_for(51)
    lq = [300, 1, 0, 129, 77, 400]
    lk = [300, 5, 7, 260, 40, 128]
    cu_q, cu_k, q, k, v = _case(rng, lq, lk, 8, 2, D)
    out, lse = sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                   torch.from_numpy(cu_k).cuda(), max(lq), max(lk), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    ref_o, ref_l = at.varlen_attention(f64(q), f64(k), f64(v), cu_q, cu_k, causal)
    _check(out, lse, ref_o, ref_l, q.dtype, f"varlen causal={causal} D={D}")


def test_varlen_fp16_many_sequences():
    rng = wl.rng_for(52)
    lens = list(rng.integers(1, 700, size=12))
    cu_q, cu_k, q, k, v = _case(rng, lens, lens, 16, 4, 128, "fp16")
    out, lse = sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                   torch.from_numpy(cu_k).cuda(), max(lens), max(lens), True)
    torch.cuda.synchronize()
    ref_o, ref_l = at.varlen_attention(f64(q), f64(k), f64(v), cu_q, cu_k, True)
    _check(out, lse, ref_o, ref_l, q.dtype, "varlen fp16")


def test_pad_unpad_roundtrip_and_padded_attention():
    """pad then unpad is the identity; padding is zero; the padded batch run
    through masked_attn_fwd with per-row key masks equals the varlen result
    on the valid rows."""
    rng = wl.rng_for(53)
    lens = [130, 7, 256, 0, 61]
    cu_q, cu_k, q, k, v = _case(rng, lens, lens, 4, 2, 128)
    cq = torch.from_numpy(cu_q).cuda()
    qp = sma.varlen_pad(q.cuda(), cq, max(lens))
    assert qp.shape == (5, 256, 4, 128)
    for b, L in enumerate(lens):
        assert torch.equal(qp[b, :L].cpu(), q[cu_q[b]:cu_q[b + 1]])
        assert (qp[b, L:] == 0).all()
    back = sma.varlen_unpad(qp, cq, int(cu_q[-1]))
    assert torch.equal(back.cpu(), q)
    out, _ = sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), cq, cq, max(lens), max(lens), False)
    kp = sma.varlen_pad(k.cuda(), cq, max(lens))
    vp = sma.varlen_pad(v.cuda(), cq, max(lens))
    mask = torch.zeros((5, 1, 1, 256), dtype=torch.bool)
    for b, L in enumerate(lens):
        mask[b, 0, 0, :L] = True
    op, _ = sma.masked_attn_fwd(qp, kp, vp, mask.cuda(), None, False)
    got = sma.varlen_unpad(op, cq, int(cu_q[-1]))
    assert (got.float() - out.float()).abs().max() <= 2e-2


def test_malformed_offsets_are_reported():
    rng = wl.rng_for(54)
    cu_q, cu_k, q, k, v = _case(rng, [100, 50], [100, 50], 2, 1, 64)
    bad = torch.tensor([0, 120, 150], dtype=torch.int32)          # sequence 0 longer than max_q = 100
    out = torch.full_like(q, 7.0).cuda()
    sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), bad.cuda(), torch.from_numpy(cu_k).cuda(), 100, 100,
                        False, out=out)
    assert sma.device_status() == 6   # SMA_ERR_DEVICE_INPUT
    assert sma.device_status() == 0
    assert (out[:120] == 7.0).all()   # the malformed sequence's rows are left untouched


# Gradient agreement as for the padded backward: relative to m = max(1,
# max |ref|) of each tensor, max-abs <= 2.5e-2 m and mean-abs <= 2.5e-3 m.
# fp32 inputs (FFMA arithmetic): max-abs <= 1e-4 m and mean-abs <= 1e-5 m.
def _close_grad(name, got, ref):
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    tmax, tmean = (1e-4, 1e-5) if got.dtype == torch.float32 else (2.5e-2, 2.5e-3)
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= tmax * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= tmean * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_varlen_fp32_forward(causal, D):
    """fp32 packed sequences on the FFMA kernel: the fp32 bound (1e-4 max-abs)
    over ragged lengths, an empty sequence and causal rows with no key."""
    rng = wl.rng_for(55)
    lq = [300, 1, 0, 129, 77, 200]
    lk = [300, 5, 7, 260, 40, 128]
    cu_q, cu_k, q, k, v = _case(rng, lq, lk, 4, 2, D, "fp32")
    out, lse = sma.varlen_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                   torch.from_numpy(cu_k).cuda(), max(lq), max(lk), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    ref_o, ref_l = at.varlen_attention(f64(q), f64(k), f64(v), cu_q, cu_k, causal)
    _check(out, lse, ref_o, ref_l, q.dtype, f"varlen fp32 causal={causal} D={D}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "bf16"), (128, "fp16"), (64, "fp32"),
                                     (128, "fp32")])
def test_varlen_backward(causal, D, dtype):
    """dQ, dK, dV of packed sequences against the float64 gradients of each
    sequence on its own: lengths spanning several tiles and ragged tails, one
    query over 40 keys, an empty sequence, different query and key lengths
    (bottom-right causal), and tiles that straddle sequence boundaries."""
    from oracle import attention_grad as ag
    rng = wl.rng_for(61)
    H, KVH = 8, 2
    lq = [130, 1, 257, 0, 100, 64]
    lk = [130, 40, 257, 0, 300, 64]
    cu_q, cu_k, q, k, v = _case(rng, lq, lk, H, KVH, D, dtype)
    do = wl.normal(rng, tuple(q.shape), dtype)
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = sma.varlen_attn_fwd(qc, kc, vc, cq, ck, max(lq), max(lk), causal)
    dq, dk, dv = sma.varlen_attn_bwd(qc, kc, vc, out, lse, dc, cq, ck, max(lq), max(lk), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    rq = np.zeros(tuple(q.shape))
    rk = np.zeros(tuple(k.shape))
    rv = np.zeros(tuple(k.shape))
    for i in range(len(lq)):
        q0, q1, k0, k1 = cu_q[i], cu_q[i + 1], cu_k[i], cu_k[i + 1]
        if q1 == q0 or k1 == k0:
            continue
        keep = at.causal_keep(q1 - q0, k1 - k0)[None, None] if causal else None
        gq, gk, gv, _ = ag.attention_grad(f64(q[q0:q1])[None], f64(k[k0:k1])[None], f64(v[k0:k1])[None],
                                          f64(do[q0:q1])[None], keep=keep)
        rq[q0:q1], rk[k0:k1], rv[k0:k1] = gq[0], gk[0], gv[0]
    _close_grad("dq", dq, rq)
    _close_grad("dk", dk, rk)
    _close_grad("dv", dv, rv)
