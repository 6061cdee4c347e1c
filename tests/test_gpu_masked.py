"""GPU: masked_attn_fwd (4D broadcast mask/bias contract, causal, decode)
agrees with the float64 oracle; broadcast and padding invariants hold."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from tests._helpers import TOL, assert_attention_close, f64, sample_tiles

pytestmark = pytest.mark.gpu


def _oracle(q, k, v, mask, bias, causal, rows=None):
    b, lq, h, d = q.shape
    lk, kvh = k.shape[1], k.shape[2]
    keep = at.aux_view(mask.cpu().numpy(), h, kvh, lk) if mask is not None else None
    if causal:
        ck = at.causal_keep(lq, lk)[None, None]
        keep = ck if keep is None else (keep & ck)
    bb = at.aux_view(f64(bias), h, kvh, lk) if bias is not None else None
    return at.attention(f64(q), f64(k), f64(v), keep=keep, bias=bb, rows=rows, workers=8, row_chunk=128)


def _run(q, k, v, mask=None, bias=None, causal=False, rows=None, what=""):
    out, lse = sma.masked_attn_fwd(q.cuda(), k.cuda(), v.cuda(),
                                   None if mask is None else mask.cuda(),
                                   None if bias is None else bias.cuda(), causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    ref_o, ref_l = _oracle(q, k, v, mask, bias, causal, rows)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, rows=rows, what=what)
    return out, lse


def _qkv(rng, b, lq, lk, h, kvh, d, dtype="bf16"):
    return (wl.normal(rng, (b, lq, h, d), dtype), wl.normal(rng, (b, lk, kvh, d), dtype),
            wl.normal(rng, (b, lk, kvh, d), dtype))


B, LQ, LK, H, KVH, D = 2, 300, 450, 8, 2, 128
KP = sma.round_up_k(LK)
AUX_SHAPES = [None, (1, 1, LQ, KP), (B, KVH, 1, KP), (B, H, LQ, KP), (1, H, 1, KP), (B, 1, 1, KP)]


@pytest.mark.parametrize("mshape", AUX_SHAPES, ids=str)
@pytest.mark.parametrize("bshape", [None, (B, KVH, 1, KP), (1, H, LQ, KP)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_small_broadcast_combinations(mshape, bshape, causal):
    rng = wl.rng_for(7)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, D)
    mask = torch.from_numpy(rng.random(mshape) < 0.8) if mshape else None
    if mask is not None:
        mask[..., :1] = True
    bias = wl.normal(rng, bshape, "bf16") if bshape else None
    _run(q, k, v, mask, bias, causal, what=f"{mshape} {bshape} {causal}")


@pytest.mark.parametrize("dtype", ["fp16", "fp32"])
def test_other_dtypes(dtype):
    rng = wl.rng_for(8)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, 64 if dtype == "fp32" else D, dtype)
    mask = torch.from_numpy(rng.random((B, 1, LQ, KP)) < 0.7)
    bias = wl.normal(rng, (1, KVH, 1, KP), "fp32")
    _run(q, k, v, mask, bias, True, what=dtype)


def test_padding_columns_never_matter():
    rng = wl.rng_for(9)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, D)
    mask = torch.from_numpy(rng.random((1, 1, LQ, KP)) < 0.8)
    bias = wl.normal(rng, (B, KVH, 1, KP), "bf16")
    o1, l1 = _run(q, k, v, mask, bias, False, what="clean pads")
    mask2, bias2 = mask.clone(), bias.clone()
    mask2[..., LK:] = True
    bias2[..., LK:] = float("inf")
    o2, l2 = sma.masked_attn_fwd(q.cuda(), k.cuda(), v.cuda(), mask2.cuda(), bias2.cuda(), False)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_stride0_equals_explicit_expand():
    """A stride-0 view of a broadcast mask/bias is read exactly as the compact
    tensor (bit-identical results); its contiguous expansion has a bias row
    per query, which the softmax adds itself instead of the tensor cores
    (rounding differs), so it agrees within the attention tolerance, and all
    three match the oracle."""
    rng = wl.rng_for(10)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, D)
    base_m = torch.from_numpy(rng.random((1, 1, LQ, KP)) < 0.8).cuda()
    base_b = wl.normal(rng, (B, 1, 1, KP), "bf16").cuda()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = sma.masked_attn_fwd(qc, kc, vc, base_m.expand(B, H, LQ, KP), base_b.expand(B, H, LQ, KP))
    o2, l2 = sma.masked_attn_fwd(qc, kc, vc, base_m.expand(B, H, LQ, KP).contiguous(),
                                 base_b.expand(B, H, LQ, KP).contiguous())
    o3, l3 = sma.masked_attn_fwd(qc, kc, vc, base_m, base_b)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
    mx, mn = TOL[torch.bfloat16]
    err = (o1.double() - o2.double()).abs()
    assert err.max().item() <= mx and err.mean().item() <= mn
    ref_o, ref_l = _oracle(q, k, v, base_m.cpu(), base_b.cpu(), False)
    for o, l in ((o1, l1), (o2, l2)):
        assert_attention_close(o, l, ref_o, ref_l, torch.bfloat16, what="stride 0")


def test_fully_masked_rows_are_zero():
    rng = wl.rng_for(11)
    q, k, v = _qkv(rng, 1, 200, 300, 4, 2, D)
    kp = sma.round_up_k(300)
    mask = torch.ones((1, 1, 200, kp), dtype=torch.bool)
    mask[0, 0, 5] = False
    mask[0, 0, 130:140] = False
    out, lse = _run(q, k, v, mask, None, False, what="dead rows")
    assert (out[0, 5] == 0).all() and torch.isneginf(lse[0, :, 5]).all()


def test_prefill_workload_sampled():
    w = wl.BROADCAST_PREFILL
    q, k, v, mask, bias = wl.masked_inputs(w)
    rows = sample_tiles(w.n_q, picks=(0, 0.02, 0.5, 1.0))   # tile 0 is fully masked (k <= q - 192)
    _run(q, k, v, mask, bias, w.is_causal, rows=rows, what=w.name)


# ------------------------------------------------------------------ decode


@pytest.mark.parametrize("bshape,mshape", [((3, 8, 1, 1024), None), ((3, 2, 1, 1024), (3, 8, 1, 1024)),
                                          (None, (1, 2, 1, 1024)), ((1, 1, 1, 1024), (3, 1, 1, 1024))],
                         ids=str)
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(bshape, mshape, d):
    rng = wl.rng_for(12)
    q, k, v = _qkv(rng, 3, 1, 1000, 8, 2, d)
    mask = torch.from_numpy(rng.random(mshape) < 0.9) if mshape else None
    bias = wl.normal(rng, bshape, "bf16") if bshape else None
    _run(q, k, v, mask, bias, False, what=f"decode {bshape} {mshape}")


@pytest.mark.parametrize("heads,kv_heads", [(8, 8), (8, 4), (8, 1), (6, 2), (12, 2)], ids=str)
@pytest.mark.parametrize("d", [64, 128])
def test_decode_query_head_groups(heads, kv_heads, d):
    """Groups of 1, 2, 8 query heads per KV head (and 3, 6, which leave rows
    of the CTA's head block empty): each lane of a key sums and keeps the
    softmax of one head of its block, so every block size is checked."""
    rng = wl.rng_for(14)
    q, k, v = _qkv(rng, 2, 1, 1500, heads, kv_heads, d)
    bias = wl.normal(rng, (2, heads, 1, 1536), "bf16")
    mask = torch.from_numpy(rng.random((2, 1, 1, 1536)) < 0.8)
    _run(q, k, v, mask, bias, False, what=f"decode H={heads} KVH={kv_heads} d={d}")


def test_decode_equals_unswapped_rows():
    """The grouped-head decode path gives the same rows as the general path
    run on a 2-row query whose first row is the decode query."""
    rng = wl.rng_for(13)
    q, k, v = _qkv(rng, 3, 2, 1000, 8, 2, D)
    bias = wl.normal(rng, (3, 8, 1, 1024), "bf16").cuda()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o_dec, l_dec = sma.masked_attn_fwd(qc[:, :1].contiguous(), kc, vc, None, bias)
    o_two, l_two = sma.masked_attn_fwd(qc, kc, vc, None, bias)
    assert (o_dec[:, 0].float() - o_two[:, 0].float()).abs().max() <= 2e-2
    assert (l_dec[:, :, 0] - l_two[:, :, 0]).abs().max() <= 1e-2


@pytest.mark.parametrize("w", [wl.BROADCAST_DECODE, wl.BROADCAST_DECODE_MASKED], ids=lambda w: w.name)
def test_decode_workload(w):
    q, k, v, mask, bias = wl.masked_inputs(w)
    _run(q, k, v, mask, bias, False, what=w.name)


# ------------------------------------------------- short queries, long keys


LK_LONG = 5000
KP_LONG = sma.round_up_k(LK_LONG)


@pytest.mark.parametrize("mshape,bshape", [(None, None), ((1, 1, 24, KP_LONG), (1, 8, 1, KP_LONG)),
                                           ((1, 8, 24, KP_LONG), None)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_short_queries_long_keys(mshape, bshape, causal, d):
    """24 queries against 5000 keys give 4 (batch, KV head, head pair, query
    tile) units: each unit's key tiles are cut into segments run on separate
    SMs and merged.  Row 3 keeps no key at all, row 5 none of the first 2500
    keys (its early segments are empty)."""
    rng = wl.rng_for(14)
    q, k, v = _qkv(rng, 1, 24, LK_LONG, 8, 2, d)
    mask = None
    if mshape is not None:
        mask = torch.from_numpy(rng.random(mshape) < 0.7)
        if mshape[2] > 1:
            mask[:, :, 3, :] = False
            mask[:, :, 5, :2500] = False
    bias = wl.normal(rng, bshape, "bf16") if bshape else None
    out, lse = _run(q, k, v, mask, bias, causal, what=f"short {mshape} {bshape} {causal} {d}")
    if mshape is not None and mshape[2] > 1:
        assert (out[0, 3] == 0).all() and torch.isneginf(lse[0, :, 3]).all()


def test_short_queries_fp16():
    rng = wl.rng_for(15)
    q, k, v = _qkv(rng, 2, 40, 3000, 4, 4, D, "fp16")
    mask = torch.from_numpy(rng.random((2, 4, 1, sma.round_up_k(3000))) < 0.5)
    _run(q, k, v, mask, None, True, what="short fp16")


@pytest.mark.parametrize("h,kvh,lq", [(16, 2, 40), (4, 2, 64), (8, 4, 2), (16, 2, 16)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_short_queries_heads_packed_per_tile(h, kvh, lq, causal):
    """Up to 64 queries with 2, 4 or 8 heads per KV head: one 128-row tile
    holds every head of the group for 128 / group queries (group 8 and 40
    queries: three blocks of 16, two tiles in one unit and one alone).  The
    bias differs per query head and per query, the mask per KV head."""
    rng = wl.rng_for(16)
    lk = 3000
    kp = sma.round_up_k(lk)
    q, k, v = _qkv(rng, 2, lq, lk, h, kvh, D)
    mask = torch.from_numpy(rng.random((2, kvh, lq, kp)) < 0.6)
    bias = wl.normal(rng, (1, h, lq, kp), "bf16")
    _run(q, k, v, mask, bias, causal, what=f"packed {h}/{kvh} lq={lq} {causal}")


@pytest.mark.parametrize("bshape", [(2, 2, 1, KP), (1, 1, 1, KP), (2, 1, 1, KP)], ids=str)
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp16", 64)])
def test_query_broadcast_bias_large_values(bshape, dtype, d):
    """A bias shared by every query and query head of a KV head, with values
    of +-30 (peaked rows, where the dominant key's probability is exactly
    representable only if the row max includes the bias), keys at -inf (never
    kept), and, where the bias has a row per (batch, KV head), one row at
    -inf everywhere (its queries keep nothing: O = 0, lse = -inf)."""
    rng = wl.rng_for(17)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, d, dtype)
    mask = torch.from_numpy(rng.random((1, 1, LQ, KP)) < 0.8)
    bias = (wl.normal(rng, bshape, "fp32") * 10.0).clamp(-30, 30)
    bias[..., ::7] = -float("inf")
    dead = bshape[0] == 2 and bshape[1] == 2
    if dead:
        bias[1, 1] = -float("inf")
    bias = bias.to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    out, lse = _run(q, k, v, mask, bias, True, what=f"large bias {bshape} {dtype} {d}")
    if dead:
        heads = slice(1 * (H // KVH), 2 * (H // KVH))
        assert (out[1, :, heads] == 0).all() and torch.isneginf(lse[1, heads]).all()


@pytest.mark.parametrize("h,kvh,lq,bshape", [(4, 4, 300, (2, 4, 1)), (16, 2, 40, (2, 2, 1)),
                                             (8, 2, 300, (1, 1, 1)), (8, 8, 24, (1, 8, 1))], ids=str)
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp16", 64)])
def test_query_broadcast_bias_through_the_tensor_cores(h, kvh, lq, bshape, dtype, d):
    """A bias row shared by every query of S (and by the query heads a tile
    pair holds) is added by one more K step of the Q K^T product: one head
    per KV head with a bias per head, head-packed short queries with a bias
    per KV head (key ranges split over SMs and merged), and a single row."""
    rng = wl.rng_for(18)
    lk = 3000
    kp = sma.round_up_k(lk)
    q, k, v = _qkv(rng, 2, lq, lk, h, kvh, d, dtype)
    mask = torch.from_numpy(rng.random((2, 1, lq, kp)) < 0.7)
    bias = (wl.normal(rng, bshape + (kp,), "fp32") * 4.0).to(q.dtype)
    _run(q, k, v, mask, bias, True, what=f"tc bias {h}/{kvh} lq={lq} {bshape} {dtype}")
