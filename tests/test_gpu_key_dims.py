"""GPU: the three key dims of a mask / bias -- round_up(Lk, 128), Lk, and 1
(one value for every key) -- read in place by every entry point that takes
them, against the float64 oracle.

flash-sparse-attention PR #190, Changes (interface) and Design (contract for
aux tensors): the page's interface pads the key dim to a multiple of 128 and
expands a key dim of 1 before its kernels run.  Here no copy is made, so the
padded and the unpadded form must give element-identical results (the
kernels take the same arithmetic path; padded columns are poisoned so that a
kernel reading them as meaningful would be caught), and a key dim of 1 must
match its explicit expansion within the attention tolerance (the row-constant
bias is added to the row's max rather than to each score, which changes
only the rounding).  Two unpadded layouts are used: Lk = 1008, contiguous
(rows of 16-byte multiples), and Lk = 1000 as a slice of a padded tensor
(rows of 1024 columns, a key dim that ends inside a 16-byte block).
"""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from oracle import attention_grad as ag
from oracle import tiles as tl
from oracle import topk as tk
from tests._helpers import TOL, assert_attention_close, f64, masked_oracle

pytestmark = pytest.mark.gpu

B, LQ, H, KVH = 2, 300, 8, 2


def _forms(padded: torch.Tensor, lk: int, poison):
    """(padded with poisoned tail, unpadded) forms of the same aux tensor, on
    the device: Lk = 1008 contiguous, other Lk a strided slice of the padded
    tensor (made on the device: copying a slice to the device would make it
    contiguous)."""
    p = padded.clone()
    p[..., lk:] = poison
    p = p.cuda()
    if lk % 16 == 0:
        u = p[..., :lk].contiguous()
    else:
        u = p[..., :lk]
        assert u.stride(-2) == p.shape[-1] or p.shape[-2] == 1
    return p, u


def _fwd(q, k, v, mask, bias, causal):
    out, lse = sma.masked_attn_fwd(q.cuda(), k.cuda(), v.cuda(), None if mask is None else mask.cuda(),
                                   None if bias is None else bias.cuda(), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    return out, lse


@pytest.mark.parametrize("lk", [1008, 1000])
@pytest.mark.parametrize("bshape", [(B, KVH, 1), (1, H, LQ)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_padded_and_unpadded_key_dims_agree(lk, bshape, causal):
    rng = wl.rng_for(101)
    kp = sma.round_up_k(lk)
    q = wl.normal(rng, (B, LQ, H, 128), "bf16")
    k = wl.normal(rng, (B, lk, KVH, 128), "bf16")
    v = wl.normal(rng, (B, lk, KVH, 128), "bf16")
    mask = torch.from_numpy(rng.random((1, 1, LQ, kp)) < 0.8)
    mask[..., 0] = True
    bias = wl.normal(rng, bshape + (kp,), "bf16")
    mp, mu = _forms(mask, lk, True)
    bp, bu = _forms(bias, lk, float("inf"))
    op, lp = _fwd(q, k, v, mp, bp, causal)
    ou, lu = _fwd(q, k, v, mu, bu, causal)
    assert torch.equal(op, ou) and torch.equal(lp, lu)
    ref_o, ref_l = masked_oracle(q, k, v, mu, bu, causal)
    assert_attention_close(ou, lu, ref_o, ref_l, torch.bfloat16, what=f"Lk {lk}")


@pytest.mark.parametrize("mshape", [(B, 1, LQ), (B, KVH, 1)], ids=str)
def test_key_dim_one_mask_and_bias(mshape):
    """A one-column mask keeps or drops whole rows (or whole heads); a
    one-column bias shifts each row's scores alike (the output is unchanged
    and lse grows by the value)."""
    rng = wl.rng_for(102)
    lk = 1000
    q = wl.normal(rng, (B, LQ, H, 128), "bf16")
    k = wl.normal(rng, (B, lk, KVH, 128), "bf16")
    v = wl.normal(rng, (B, lk, KVH, 128), "bf16")
    flags = torch.from_numpy(rng.random(mshape + (1,)) < 0.6)
    flags.view(-1)[0] = True
    bias = wl.normal(rng, (B, H, LQ, 1), "bf16") * 3.0
    out, lse = _fwd(q, k, v, flags, bias, True)
    ref_o, ref_l = masked_oracle(q, k, v, flags, bias, True)
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, what="key dim 1")
    kp = sma.round_up_k(lk)
    oe, le = _fwd(q, k, v, flags.expand(*mshape, kp).contiguous(), bias.expand(B, H, LQ, kp).contiguous(), True)
    mx, mn = TOL[torch.bfloat16]
    err = (out.double() - oe.double()).abs()
    assert err.max().item() <= mx and err.mean().item() <= mn
    assert torch.equal(torch.isneginf(lse), torch.isneginf(le))


@pytest.mark.parametrize("kd", ["pad", "lk", "one"])
def test_decode_key_dims(kd):
    """The single-query grouped-head path with each key-dim form."""
    rng = wl.rng_for(103)
    lk, h, kvh = 1000, 16, 4
    kp = sma.round_up_k(lk)
    q = wl.normal(rng, (3, 1, h, 128), "bf16")
    k = wl.normal(rng, (3, lk, kvh, 128), "bf16")
    v = wl.normal(rng, (3, lk, kvh, 128), "bf16")
    if kd == "one":
        mask = torch.from_numpy(rng.random((3, kvh, 1, 1)) < 0.7)
        mask.view(-1)[0] = True
        bias = wl.normal(rng, (3, h, 1, 1), "bf16")
    else:
        mask = torch.from_numpy(rng.random((3, kvh, 1, kp)) < 0.9)
        bias = wl.normal(rng, (3, h, 1, kp), "bf16")
        mask, bias = _forms(mask, lk, True)[kd == "lk"], _forms(bias, lk, float("inf"))[kd == "lk"]
    out, lse = _fwd(q, k, v, mask, bias, False)
    ref_o, ref_l = masked_oracle(q, k, v, mask, bias, False)
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, what=f"decode {kd}")


def test_fp32_key_dims():
    """fp32 inputs (the FFMA forward): bias of key dim Lk and mask of key dim 1."""
    rng = wl.rng_for(104)
    lk = 500
    q = wl.normal(rng, (B, 130, H, 64), "fp32")
    k = wl.normal(rng, (B, lk, KVH, 64), "fp32")
    v = wl.normal(rng, (B, lk, KVH, 64), "fp32")
    bias = wl.normal(rng, (B, KVH, 1, lk), "fp32")          # 2000-byte rows
    flags = torch.from_numpy(rng.random((1, 1, 130, 1)) < 0.7)
    out, lse = _fwd(q, k, v, flags, bias, True)
    ref_o, ref_l = masked_oracle(q, k, v, flags, bias, True)
    assert_attention_close(out, lse, ref_o, ref_l, torch.float32, what="fp32")


def _close_grad(name, got, ref, tol=(2.5e-2, 2.5e-3)):
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= tol[0] * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= tol[1] * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("lk", [1008, 1000])
def test_backward_dbias_at_the_bias_key_dim(D, lk):
    """dbias takes the bias's own key dim: the unpadded form's dbias equals
    the padded form's first Lk columns; both match the oracle."""
    rng = wl.rng_for(105)
    kp = sma.round_up_k(lk)
    q = wl.normal(rng, (B, LQ, H, D), "bf16")
    k = wl.normal(rng, (B, lk, KVH, D), "bf16")
    v = wl.normal(rng, (B, lk, KVH, D), "bf16")
    do = wl.normal(rng, (B, LQ, H, D), "bf16")
    mask = torch.from_numpy(rng.random((B, 1, LQ, kp)) < 0.8)
    bias = wl.normal(rng, (B, KVH, 1, kp), "bf16")
    results = []
    for m_, b_ in zip(_forms(mask, lk, True), _forms(bias, lk, float("inf"))):
        qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, m_, b_))
        out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, True)
        results.append(sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, True, return_dbias=True))
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    (dq_p, dk_p, dv_p, db_p), (dq_u, dk_u, dv_u, db_u) = results
    assert db_u.shape == (B, KVH, 1, lk) and (db_p[..., lk:] == 0).all()
    keep = at.aux_view(mask.numpy(), H, KVH, lk) & at.causal_keep(LQ, lk)[None, None]
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep,
                                        bias=at.aux_view(f64(bias), H, KVH, lk),
                                        dbias_shape=(B, KVH, 1, lk), workers=at.host_threads())
    for tag, (dq, dk, dv, db) in (("padded", results[0]), ("unpadded", results[1])):
        _close_grad(f"dq {tag}", dq, rq)
        _close_grad(f"dk {tag}", dk, rk)
        _close_grad(f"dv {tag}", dv, rv)
        _close_grad(f"dbias {tag}", db[..., :lk], rdb)


@pytest.mark.parametrize("D", [64, 128])
def test_backward_key_dim_one(D):
    """A one-column bias has a zero gradient (the call writes zeros) and
    leaves dQ, dK, dV as without it; a one-column mask drops whole rows."""
    rng = wl.rng_for(106)
    lk = 700
    q = wl.normal(rng, (B, LQ, H, D), "bf16")
    k = wl.normal(rng, (B, lk, KVH, D), "bf16")
    v = wl.normal(rng, (B, lk, KVH, D), "bf16")
    do = wl.normal(rng, (B, LQ, H, D), "bf16")
    flags = torch.from_numpy(rng.random((B, 1, LQ, 1)) < 0.7)
    bias = wl.normal(rng, (1, H, LQ, 1), "bf16") * 2.0
    qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, flags, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, False)
    dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, False, return_dbias=True)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    assert db.shape == bias.shape and (db == 0).all()
    keep = at.aux_view(flags.numpy(), H, KVH, lk)
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep,
                                        bias=at.aux_view(f64(bias), H, KVH, lk), dbias_shape=tuple(bias.shape),
                                        workers=at.host_threads())
    assert np.abs(rdb).max() < 1e-9
    _close_grad("dq", dq, rq)
    _close_grad("dk", dk, rk)
    _close_grad("dv", dv, rv)


@pytest.mark.parametrize("kd", ["lk", "one"])
def test_sparse_attn_key_dims(kd):
    """Index-gather attention with a query-broadcast mask of key dim Lk (equal
    to the padded form) or 1 (every key kept or none)."""
    rng = wl.rng_for(107)
    lk, lq, h, kvh = 1000, 260, 8, 2
    kp = sma.round_up_k(lk)
    q = wl.normal(rng, (B, lq, h, 128), "bf16")
    k = wl.normal(rng, (B, lk, kvh, 128), "bf16")
    v = wl.normal(rng, (B, lk, kvh, 128), "bf16")
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    if kd == "lk":
        mask = torch.from_numpy(rng.random((B, kvh, 1, kp)) < 0.15)
        mp, mu = _forms(mask, lk, True)
        op, lp = sma.sparse_attn_fwd(qc, kc, vc, mp.cuda(), None, True, max_keys=256)
        ou, lu = sma.sparse_attn_fwd(qc, kc, vc, mu.cuda(), None, True, max_keys=256)
        torch.cuda.synchronize()
        assert sma.device_status() == 0
        assert torch.equal(op, ou) and torch.equal(lp, lu)
    else:
        mu = torch.tensor([[[[True]], [[False]]], [[[True]], [[True]]]])
        ou, lu = sma.sparse_attn_fwd(qc, kc, vc, mu.cuda(), None, True)
        torch.cuda.synchronize()
        assert sma.device_status() == 0
    ref_o, ref_l = masked_oracle(q, k, v, mu, None, True)
    assert_attention_close(ou, lu, ref_o, ref_l, torch.bfloat16, what=f"sparse {kd}")


SENT = {torch.bfloat16: tk.FINFO_MIN["bf16"], torch.float32: tk.FINFO_MIN["fp32"]}


@pytest.mark.parametrize("dtype,lk,sliced", [(torch.bfloat16, 1000, False), (torch.bfloat16, 16380, True),
                                             (torch.float32, 1001, True)], ids=str)
def test_topk_bias_of_key_dim_lk(dtype, lk, sliced):
    """The top-k mask of a bias whose key dim is Lk has the bias's shape and
    equals the padded bias's mask (first Lk columns), bit for bit, and the
    oracle's."""
    rng = wl.rng_for(108)
    kp = sma.round_up_k(lk)
    padded = wl.normal(rng, (2, 2, 3, kp), "bf16" if dtype == torch.bfloat16 else "fp32").cuda()
    pre = torch.from_numpy(rng.random((2, lk)) < 0.9)
    unp = padded[..., :lk] if sliced else padded[..., :lk].contiguous()
    assert (unp.stride(-2) == kp) == sliced
    got_p = sma.dynamic_topk_mask(padded, lk, 300, pre.cuda())
    got_u = sma.dynamic_topk_mask(unp, lk, 300, pre.cuda())
    torch.cuda.synchronize()
    assert got_u.shape == unp.shape
    assert torch.equal(got_p[..., :lk], got_u)
    pm = tk.normalize_pre_mask(pre.numpy(), 2, 3, lk)
    want = tk.dynamic_topk_keep(f64(unp), lk, pm, 300, SENT[dtype])
    np.testing.assert_array_equal(got_u.cpu().numpy(), want)


@pytest.mark.parametrize("form", ["pad", "lk", "one"])
def test_mask_tile_summary_key_dims(form):
    rng = wl.rng_for(109)
    lk = 1000
    kp = sma.round_up_k(lk)
    if form == "one":
        mask = torch.from_numpy(rng.random((2, 1, 400, 1)) < 0.5)
        mask[0, 0, :128] = True
        mask[1, 0, 128:256] = False
    else:
        mask = torch.from_numpy(rng.random((2, 1, 400, kp)) < 0.97)
        mask[0, 0, :, :256] = True
        mask = _forms(mask, lk, True)[form == "lk"]
    got = sma.mask_tile_summary(mask.cuda(), lk).cpu().numpy()
    np.testing.assert_array_equal(got, tl.mask_tile_summary(mask.cpu().numpy(), lk))
