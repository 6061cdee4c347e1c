"""Pins for the oracle's attention gradients (CPU only).

Pinned to: a hand-worked two-key example; central finite differences of the
forward oracle (every input, with masks, dead rows, grouped heads and
broadcast / per-query biases); closed forms (a row with one kept key has no
query or key gradient and passes dO to that key's value); and float64
autograd through torch's softmax as an independent routine.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as at
from oracle import attention_grad as ag
from tests.conftest import GOLDEN


def _vals(tokens):
    out = []
    for t in tokens:
        if t.endswith("ln3"):
            out.append(float(t[:-3]) * math.log(3.0))
        else:
            out.append(float(t))
    return np.array(out)


def test_worked_two_keys():
    want = {}
    with open(os.path.join(GOLDEN, "attention_grad_worked.txt")) as f:
        for ln in f:
            ln = ln.split("#")[0].strip()
            if ln:
                name, *vals = ln.split()
                want[name] = _vals(vals)
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[0.0, 0.0], [math.log(3.0), 0.0]]).reshape(1, 2, 1, 2)
    v = np.array([[4.0, 0.0], [0.0, 8.0]]).reshape(1, 2, 1, 2)
    do = np.array([1.0, 1.0]).reshape(1, 1, 1, 2)
    bias = np.zeros((1, 1, 1, 2))
    dq, dk, dv, db = ag.attention_grad(q, k, v, do, bias=bias, scale=1.0, dbias_shape=(1, 1, 1, 2))
    np.testing.assert_allclose(dq[0, 0, 0], want["dq"], atol=1e-15)
    np.testing.assert_allclose(dk[0, 0, 0], want["dk0"], atol=1e-15)
    np.testing.assert_allclose(dk[0, 1, 0], want["dk1"], atol=1e-15)
    np.testing.assert_allclose(dv[0, 0, 0], want["dv0"], atol=1e-15)
    np.testing.assert_allclose(dv[0, 1, 0], want["dv1"], atol=1e-15)
    np.testing.assert_allclose(db[0, 0, 0], want["dbias"], atol=1e-15)


def _case(seed, bias_shape):
    rng = np.random.default_rng(seed)
    B, LQ, LK, H, KVH, D = 2, 5, 7, 4, 2, 3
    q = rng.standard_normal((B, LQ, H, D))
    k = rng.standard_normal((B, LK, KVH, D))
    v = rng.standard_normal((B, LK, KVH, D))
    do = rng.standard_normal((B, LQ, H, D))
    keep = rng.random((B, 1, LQ, LK)) < 0.7
    keep[0, 0, 2] = False          # a dead row
    keep[1, 0, 3] = False
    keep[1, 0, 3, 4] = True        # a row with one key
    bias = rng.standard_normal(bias_shape) if bias_shape else None
    return q, k, v, do, keep, bias


def _loss(q, k, v, do, keep, bias, scale):
    o, _ = at.attention(q, k, v, keep=keep,
                        bias=None if bias is None else at.aux_view(bias, q.shape[2], k.shape[2], k.shape[1]),
                        scale=scale)
    return float((o * do).sum())


@pytest.mark.parametrize("bias_shape", [None, (1, 2, 1, 8), (2, 4, 5, 8), (1, 1, 1, 8), (2, 2, 5, 8)], ids=str)
@pytest.mark.parametrize("which", ["q", "k", "v", "bias"])
def test_central_differences(bias_shape, which):
    if which == "bias" and bias_shape is None:
        pytest.skip("no bias")
    q, k, v, do, keep, bias = _case(11, bias_shape)
    scale = 0.7
    bview = None if bias is None else at.aux_view(bias, 4, 2, 7)
    dq, dk, dv, db = ag.attention_grad(q, k, v, do, keep=keep, bias=bview, scale=scale,
                                       dbias_shape=None if bias is None else bias.shape)
    rng = np.random.default_rng(12)
    args = {"q": q, "k": k, "v": v, "bias": bias}
    grads = {"q": dq, "k": dk, "v": dv, "bias": db}
    direction = rng.standard_normal(args[which].shape)
    if which == "bias":
        direction[..., 7:] = 0.0      # columns >= Lk carry no meaning
    eps = 1e-6

    def at_(t):
        a = dict(args)
        a[which] = args[which] + t * direction
        return _loss(a["q"], a["k"], a["v"], do, keep, a["bias"], scale)

    fd = (at_(eps) - at_(-eps)) / (2 * eps)
    an = float((grads[which] * direction).sum())
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


def test_one_kept_key_closed_form():
    q, k, v, do, keep, _ = _case(13, None)
    keep = np.zeros_like(keep)
    keep[..., 4] = True                                  # every row keeps key 4 only
    dq, dk, dv, _ = ag.attention_grad(q, k, v, do, keep=keep)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    want = do.reshape(2, 5, 2, 2, 3).sum(axis=(1, 3))     # sum over rows and the group's heads
    np.testing.assert_allclose(dv[:, 4], want, atol=1e-13)
    assert np.abs(np.delete(dv, 4, axis=1)).max() == 0.0


def test_matches_float64_autograd():
    q, k, v, do, keep, bias = _case(14, (2, 4, 5, 8))
    scale = 0.9
    dq, dk, dv, db = ag.attention_grad(q, k, v, do, keep=keep, bias=at.aux_view(bias, 4, 2, 7), scale=scale,
                                       dbias_shape=bias.shape)
    tq, tk, tv, tb = (torch.tensor(a, requires_grad=True) for a in (q, k, v, bias))
    kk = tk.repeat_interleave(2, dim=2)
    vv = tv.repeat_interleave(2, dim=2)
    s = torch.einsum("bqhd,bkhd->bhqk", tq, kk) * scale + tb[..., :7]
    s = s.masked_fill(~torch.from_numpy(keep), float("-inf"))
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)
    o = torch.einsum("bhqk,bkhd->bqhd", p, vv)
    (o * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(db, tb.grad.numpy(), atol=1e-12)


def test_per_sequence_gradients_equal_block_diagonal_mask():
    """Packed sequences' gradients, computed one sequence at a time (how the
    packed backward's parity test builds its reference), equal the gradients
    of the concatenated batch under the block-diagonal keep mask with
    bottom-right causality inside each block."""
    rng = np.random.default_rng(21)
    lq, lk = [3, 5, 2], [4, 5, 6]
    H, KVH, d = 4, 2, 3
    cq, ck = np.cumsum([0] + lq), np.cumsum([0] + lk)
    q = rng.standard_normal((1, cq[-1], H, d))
    k = rng.standard_normal((1, ck[-1], KVH, d))
    v = rng.standard_normal((1, ck[-1], KVH, d))
    do = rng.standard_normal((1, cq[-1], H, d))
    keep = np.zeros((1, 1, cq[-1], ck[-1]), dtype=bool)
    for i in range(3):
        keep[0, 0, cq[i]:cq[i + 1], ck[i]:ck[i + 1]] = at.causal_keep(lq[i], lk[i])
    dq, dk, dv, _ = ag.attention_grad(q, k, v, do, keep=keep)
    for i in range(3):
        s_q, s_k = slice(cq[i], cq[i + 1]), slice(ck[i], ck[i + 1])
        gq, gk, gv, _ = ag.attention_grad(q[:, s_q], k[:, s_k], v[:, s_k], do[:, s_q],
                                          keep=at.causal_keep(lq[i], lk[i])[None, None])
        np.testing.assert_allclose(dq[:, s_q], gq, atol=1e-13)
        np.testing.assert_allclose(dk[:, s_k], gk, atol=1e-13)
        np.testing.assert_allclose(dv[:, s_k], gv, atol=1e-13)


def test_dbias_key_dim_forms():
    """dbias at the bias's own key dim.  Key dim Lk: the padded dbias's first
    Lk columns.  Key dim 1 (one value for every key of a row): the gradient of
    a shift shared by every score of the row, which is exactly zero
    (sum_k P (dP - D) = D - D), while dQ, dK and dV equal those without the
    bias (softmax ignores the shift); also equal to the full-shape dbias of
    the expanded bias summed over the keys, and to torch autograd."""
    q, k, v, do, keep, bias_pad = _case(15, (2, 2, 5, 8))
    lk = 7
    pad = ag.attention_grad(q, k, v, do, keep=keep, bias=at.aux_view(bias_pad, 4, 2, lk),
                            dbias_shape=bias_pad.shape)
    unp = np.ascontiguousarray(bias_pad[..., :lk])
    got = ag.attention_grad(q, k, v, do, keep=keep, bias=at.aux_view(unp, 4, 2, lk), dbias_shape=unp.shape)
    for a, b in zip(pad[:3], got[:3]):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(pad[3][..., :lk], got[3])

    rng = np.random.default_rng(16)
    c = rng.standard_normal((2, 4, 5, 1)) * 2.0
    dq, dk, dv, db = ag.attention_grad(q, k, v, do, keep=keep, bias=at.aux_view(c, 4, 2, lk),
                                       dbias_shape=c.shape)
    assert db.shape == c.shape and np.abs(db).max() < 1e-12
    nq, nk, nv, _ = ag.attention_grad(q, k, v, do, keep=keep)
    np.testing.assert_allclose(dq, nq, atol=1e-12)
    np.testing.assert_allclose(dk, nk, atol=1e-12)
    np.testing.assert_allclose(dv, nv, atol=1e-12)
    full = np.repeat(c, lk, axis=-1)
    _, _, _, dfull = ag.attention_grad(q, k, v, do, keep=keep, bias=full, dbias_shape=full.shape)
    np.testing.assert_allclose(db[..., 0], dfull.sum(axis=-1), atol=1e-12)
    tq = torch.tensor(q)
    tc = torch.tensor(c, requires_grad=True)
    kk = torch.tensor(k).repeat_interleave(2, dim=2)
    vv = torch.tensor(v).repeat_interleave(2, dim=2)
    s = torch.einsum("bqhd,bkhd->bhqk", tq, kk) / math.sqrt(3) + tc
    s = s.masked_fill(~torch.from_numpy(keep), float("-inf"))
    o = torch.einsum("bhqk,bkhd->bqhd", torch.softmax(s, dim=-1).nan_to_num(0.0), vv)
    (o * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(db, tc.grad.numpy(), atol=1e-12)
