"""Pins for the oracle's dense attention (CPU only).

Pinned to: a hand-worked single-row example; torch's float64
scaled_dot_product_attention (no mask, bool mask, additive float mask, and
its bottom-right causal bias); scipy's logsumexp; and invariants (one kept
key returns that value row, broadcast equals explicit expansion, columns at or
beyond Lk never matter).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp
from torch.nn.attention.bias import causal_lower_right

from oracle import attention as at
from oracle import dflash_mask as dm
from tests.conftest import GOLDEN


def _val(tok):
    tok = tok.strip()
    if tok.startswith("ln"):
        return math.log(float(tok[2:]))
    if tok == "-inf":
        return -math.inf
    return float(tok)


def test_worked_single_row():
    with open(os.path.join(GOLDEN, "attention_worked.txt")) as f:
        rows = [ln.split("#")[0] for ln in f if ln.split("#")[0].strip()]
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[0.0, 0.0], [math.log(3.0), 0.0]]).reshape(1, 2, 1, 2)
    v = np.array([[4.0, 0.0], [0.0, 8.0]]).reshape(1, 2, 1, 2)
    assert len(rows) == 5
    for row in rows:
        keep_s, bias_s, o_s, lse_s = row.split("|")
        keep = np.array([int(x) for x in keep_s.split()], dtype=bool).reshape(1, 1, 1, 2)
        bias = np.array([_val(x) for x in bias_s.split()]).reshape(1, 1, 1, 2)
        out, lse = at.attention(q, k, v, keep=keep, bias=bias, scale=1.0)
        np.testing.assert_allclose(out[0, 0, 0], [_val(x) for x in o_s.split()], rtol=0, atol=1e-12)
        want = _val(lse_s)
        if want == -math.inf:
            assert lse[0, 0, 0] == -math.inf
        else:
            assert abs(lse[0, 0, 0] - want) < 1e-12


def _sdpa(q, k, v, attn_mask=None, scale=None):
    """torch float64 reference with GQA by repeating KV heads."""
    g = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=attn_mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.fixture
def qkv():
    rng = np.random.default_rng(11)
    b, lq, lk, h, kvh, d = 2, 37, 53, 6, 2, 16
    q = rng.standard_normal((b, lq, h, d))
    k = rng.standard_normal((b, lk, kvh, d))
    v = rng.standard_normal((b, lk, kvh, d))
    return q, k, v


def test_all_keep_equals_sdpa(qkv):
    q, k, v = qkv
    out, lse = at.attention(q, k, v, row_chunk=16)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=0, atol=1e-12)


def test_bool_mask_and_bias_equal_sdpa(qkv):
    q, k, v = qkv
    rng = np.random.default_rng(3)
    b, lq, h, _ = q.shape
    lk = k.shape[1]
    mask = rng.random((b, h, lq, lk)) < 0.6
    mask[..., 0] = True                      # no fully masked rows for SDPA
    bias = rng.standard_normal((b, h, lq, lk))
    out, _ = at.attention(q, k, v, keep=mask, bias=bias, scale=0.3)
    float_mask = torch.from_numpy(np.where(mask, bias, -np.inf))
    np.testing.assert_allclose(out, _sdpa(q, k, v, attn_mask=float_mask, scale=0.3), rtol=0, atol=1e-12)
    out_b, _ = at.attention(q, k, v, keep=mask)
    np.testing.assert_allclose(out_b, _sdpa(q, k, v, attn_mask=torch.from_numpy(mask)), rtol=0, atol=1e-12)


def test_bottom_right_causal_equals_torch_bias(qkv):
    q, k, v = qkv
    lq, lk = q.shape[1], k.shape[1]
    keep = at.causal_keep(lq, lk)
    # hand example: 2 queries, 4 keys -> row 0 keeps 0..2, row 1 keeps 0..3
    np.testing.assert_array_equal(at.causal_keep(2, 4), [[1, 1, 1, 0], [1, 1, 1, 1]])
    out, _ = at.attention(q, k, v, keep=keep[None, None])
    ref = _sdpa(q, k, v, attn_mask=causal_lower_right(lq, lk))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_lse_equals_logsumexp(qkv):
    q, k, v = qkv
    rng = np.random.default_rng(5)
    bias = rng.standard_normal((1, 1, q.shape[1], k.shape[1]))
    out, lse = at.attention(q, k, v, bias=bias, scale=0.25)
    g = q.shape[2] // k.shape[2]
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            s = 0.25 * q[b, :, h, :] @ k[b, :, h // g, :].T + bias[0, 0]
            np.testing.assert_allclose(lse[b, h], logsumexp(s, axis=1), rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one(qkv):
    q, k, _ = qkv
    rng = np.random.default_rng(9)
    keep = rng.random((1, 1, q.shape[1], k.shape[1])) < 0.3
    keep[..., 5] = True
    ones = np.ones_like(k)
    out, _ = at.attention(q, k, ones, keep=keep)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_single_kept_key_returns_value_row(qkv):
    q, k, v = qkv
    b, lq, h, _ = q.shape
    lk = k.shape[1]
    rng = np.random.default_rng(1)
    pick = rng.integers(0, lk, size=(b, h, lq))
    keep = np.zeros((b, h, lq, lk), dtype=bool)
    np.put_along_axis(keep, pick[..., None], True, axis=-1)
    out, _ = at.attention(q, k, v, keep=keep)
    g = h // k.shape[2]
    for bi in range(b):
        for hi in range(h):
            np.testing.assert_array_equal(out[bi, :, hi, :], v[bi, pick[bi, hi], hi // g, :])


def test_fully_masked_row_is_zero_and_minus_inf(qkv):
    q, k, v = qkv
    keep = np.ones((1, 1, q.shape[1], k.shape[1]), dtype=bool)
    keep[..., 3, :] = False
    out, lse = at.attention(q, k, v, keep=keep)
    assert np.all(out[:, 3] == 0.0)
    assert np.all(lse[:, :, 3] == -np.inf)
    assert np.isfinite(out).all()


def test_broadcast_views_equal_explicit_expand(qkv):
    q, k, v = qkv
    b, lq, h, _ = q.shape
    kvh, lk = k.shape[2], k.shape[1]
    kpad = 64
    rng = np.random.default_rng(2)
    for bshape in [(1, 1, 1, kpad), (b, kvh, 1, kpad), (1, h, lq, kpad), (b, 1, lq, kpad)]:
        bias = rng.standard_normal(bshape)
        mask = rng.random(bshape) < 0.7
        mask[..., 0] = True
        explicit_b = np.empty((b, h, lq, lk))
        explicit_m = np.empty((b, h, lq, lk), dtype=bool)
        g = h // kvh
        for bi in range(b):
            for hi in range(h):
                hb = hi if bshape[1] == h else (hi // g if bshape[1] == kvh else 0)
                explicit_b[bi, hi] = bias[bi if bshape[0] > 1 else 0, hb, :, :lk]
                explicit_m[bi, hi] = mask[bi if bshape[0] > 1 else 0, hb, :, :lk]
        o1, l1 = at.attention(q, k, v, keep=at.aux_view(mask, h, kvh, lk), bias=at.aux_view(bias, h, kvh, lk))
        o2, l2 = at.attention(q, k, v, keep=explicit_m, bias=explicit_b)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


def test_columns_beyond_lk_never_matter(qkv):
    q, k, v = qkv
    lk = k.shape[1]
    rng = np.random.default_rng(4)
    bias = rng.standard_normal((1, 1, 1, 64))
    mask = rng.random((1, 1, 1, 64)) < 0.8
    mask[..., 0] = True
    poisoned_b = bias.copy()
    poisoned_b[..., lk:] = np.inf
    poisoned_m = mask.copy()
    poisoned_m[..., lk:] = True
    h, kvh = q.shape[2], k.shape[2]
    o1, _ = at.attention(q, k, v, keep=at.aux_view(mask, h, kvh, lk), bias=at.aux_view(bias, h, kvh, lk))
    o2, _ = at.attention(q, k, v, keep=at.aux_view(poisoned_m, h, kvh, lk),
                         bias=at.aux_view(poisoned_b, h, kvh, lk))
    np.testing.assert_array_equal(o1, o2)


@pytest.mark.parametrize("causal", [False, True])
def test_one_block_dflash_equals_sdpa_on_concatenated_keys(causal):
    """With a single draft block the DFlash mask reduces to attention over
    concat(context[:anchor], block keys): no mask when bidirectional, and the
    bottom-right causal bias when causal."""
    rng = np.random.default_rng(8 + causal)
    ctx, bs, anchor, h, kvh, d = 40, 16, 29, 4, 2, 8
    q = rng.standard_normal((1, bs, h, d))
    k = rng.standard_normal((1, ctx + bs, kvh, d))
    v = rng.standard_normal((1, ctx + bs, kvh, d))
    anchors = np.array([[anchor]])
    keep = dm.dflash_keep_mask(anchors, ctx, bs, causal, None)[:, None]
    out, _ = at.attention(q, k, v, keep=keep)
    sel = np.r_[0:anchor, ctx:ctx + bs]
    ks, vs = k[:, sel], v[:, sel]
    mask = causal_lower_right(bs, len(sel)) if causal else None
    np.testing.assert_allclose(out, _sdpa(q, ks, vs, attn_mask=mask), rtol=0, atol=1e-12)


def test_sampled_rows_match_full_run(qkv):
    q, k, v = qkv
    full, lse = at.attention(q, k, v, row_chunk=8)
    part, lse_p = at.attention(q, k, v, rows=[(3, 11), (30, 37)], row_chunk=8)
    np.testing.assert_array_equal(part[:, 3:11], full[:, 3:11])
    np.testing.assert_array_equal(lse_p[:, :, 30:37], lse[:, :, 30:37])
    assert np.isnan(part[:, 12]).all()


def test_threaded_equals_serial(qkv):
    q, k, v = qkv
    o1, l1 = at.attention(q, k, v, row_chunk=8, workers=1)
    o2, l2 = at.attention(q, k, v, row_chunk=8, workers=4)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_block_diagonal_mask(causal):
    """Packed sequences equal one problem over the packed rows with a
    block-diagonal keep mask (causal bottom-right inside each block)."""
    rng = np.random.default_rng(21)
    lq, lk = [3, 0, 5, 1, 4], [4, 2, 5, 0, 2]
    cu_q, cu_k = np.cumsum([0] + lq), np.cumsum([0] + lk)
    H, KVH, D = 4, 2, 3
    q = rng.standard_normal((cu_q[-1], H, D))
    k = rng.standard_normal((cu_k[-1], KVH, D))
    v = rng.standard_normal((cu_k[-1], KVH, D))
    out, lse = at.varlen_attention(q, k, v, cu_q, cu_k, causal)
    keep = np.zeros((cu_q[-1], cu_k[-1]), bool)
    for b in range(len(lq)):
        blk = np.ones((lq[b], lk[b]), bool)
        if causal:
            blk = at.causal_keep(lq[b], lk[b])
        keep[cu_q[b]:cu_q[b + 1], cu_k[b]:cu_k[b + 1]] = blk
    ref, ref_lse = at.attention(q[None], k[None], v[None], keep=keep[None, None])
    np.testing.assert_allclose(out, ref[0], atol=1e-13)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(ref_lse[0]))
    fin = ~np.isneginf(lse)
    np.testing.assert_allclose(lse[fin], ref_lse[0][fin], atol=1e-13)


@pytest.mark.parametrize("mshape,bshape", [((5, 1, 1, 8), (1, 4, 5, 8)), ((1, 2, 5, 8), (5, 2, 1, 1)),
                                           ((5, 4, 5, 8), None), (None, (1, 1, 5, 6))], ids=str)
def test_varlen_mask_bias_equal_the_block_diagonal_problem(mshape, bshape):
    """A packed batch with a mask / bias in the padded per-sequence layout
    equals one problem over the packed rows whose keep mask is block-diagonal
    and, inside block b, sequence b's mask rows / columns [0, len) (bias
    likewise), for batch-, head- (H or KVH) and query-broadcast shapes and a
    key dim that is padded, exact or 1."""
    rng = np.random.default_rng(22)
    lq, lk = [3, 0, 5, 1, 4], [4, 2, 5, 0, 2]
    cu_q, cu_k = np.cumsum([0] + lq), np.cumsum([0] + lk)
    H, KVH, D = 4, 2, 3
    q = rng.standard_normal((cu_q[-1], H, D))
    k = rng.standard_normal((cu_k[-1], KVH, D))
    v = rng.standard_normal((cu_k[-1], KVH, D))
    mask = rng.random(mshape) < 0.7 if mshape else None
    bias = rng.standard_normal(bshape) if bshape else None
    out, lse = at.varlen_attention(q, k, v, cu_q, cu_k, True, mask=mask, bias=bias)
    tq, tk = cu_q[-1], cu_k[-1]
    keep = np.zeros((H, tq, tk), bool)
    dense_bias = np.zeros((H, tq, tk))
    for b in range(len(lq)):
        for h in range(H):
            for i in range(lq[b]):
                for j in range(lk[b]):
                    ok = j <= i + lk[b] - lq[b]          # bottom-right causal
                    if mask is not None:
                        mb = mask[b if mask.shape[0] > 1 else 0]
                        mh = mb[h if mask.shape[1] == H else (h // (H // KVH) if mask.shape[1] > 1 else 0)]
                        mr = mh[i if mask.shape[2] > 1 else 0]
                        ok = ok and bool(mr[j if mask.shape[3] > 1 else 0])
                    keep[h, cu_q[b] + i, cu_k[b] + j] = ok
                    if bias is not None:
                        bb = bias[b if bias.shape[0] > 1 else 0]
                        bh = bb[h if bias.shape[1] == H else (h // (H // KVH) if bias.shape[1] > 1 else 0)]
                        br = bh[i if bias.shape[2] > 1 else 0]
                        dense_bias[h, cu_q[b] + i, cu_k[b] + j] = br[j if bias.shape[3] > 1 else 0]
    ref, ref_lse = at.attention(q[None], k[None], v[None], keep=keep[None], bias=dense_bias[None])
    np.testing.assert_allclose(out, ref[0], atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(ref_lse[0]))
    fin = ~np.isneginf(lse)
    np.testing.assert_allclose(lse[fin], ref_lse[0][fin], atol=1e-12)


def test_key_dim_forms_of_mask_and_bias(qkv):
    """The three key dims of PR #190's interface (padded to a multiple of 128
    there; padded, Lk, or 1 which the interface expands).  A mask/bias of key
    dim Lk equals the padded one's first Lk columns; a key dim of 1 equals its
    explicit expansion over the keys.  A bias that is one value c per row
    shifts every score of the row alike: the output is that of no bias at all
    and lse grows by exactly c (softmax is shift invariant).  A one-column
    mask keeps a row whole or kills it."""
    q, k, v = qkv
    b, lq, h, _ = q.shape
    kvh, lk = k.shape[2], k.shape[1]
    rng = np.random.default_rng(5)
    pad = rng.standard_normal((b, kvh, lq, 64))
    mpad = rng.random((b, kvh, lq, 64)) < 0.7
    mpad[..., 0] = True
    o1, l1 = at.attention(q, k, v, keep=at.aux_view(mpad, h, kvh, lk), bias=at.aux_view(pad, h, kvh, lk))
    o2, l2 = at.attention(q, k, v, keep=at.aux_view(np.ascontiguousarray(mpad[..., :lk]), h, kvh, lk),
                          bias=at.aux_view(np.ascontiguousarray(pad[..., :lk]), h, kvh, lk))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)

    c = rng.standard_normal((b, h, lq, 1)) * 3.0
    o_c, l_c = at.attention(q, k, v, bias=at.aux_view(c, h, kvh, lk))
    o_x, l_x = at.attention(q, k, v, bias=np.repeat(c, lk, axis=-1))
    np.testing.assert_array_equal(o_c, o_x)
    np.testing.assert_array_equal(l_c, l_x)
    o_0, l_0 = at.attention(q, k, v)
    np.testing.assert_allclose(o_c, o_0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_c, l_0 + c[..., 0], rtol=0, atol=1e-12)

    flag = rng.random((1, 1, lq, 1)) < 0.5
    o_f, l_f = at.attention(q, k, v, keep=at.aux_view(flag, h, kvh, lk))
    rows = flag[0, 0, :, 0]
    np.testing.assert_array_equal(o_f[:, rows], o_0[:, rows])
    assert np.all(o_f[:, ~rows] == 0.0) and np.all(l_f[:, :, ~rows] == -np.inf)
