"""GPU: sparse_attn_fwd (index-gather attention over the keys a
query-broadcast keep mask selects) agrees with the float64 oracle of the
dense masked definition, at small sizes spanning several compacted tiles and
a ragged tail, on the top-k workload, and in its edge cases."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from tests._helpers import assert_attention_close, masked_oracle, sample_tiles

pytestmark = pytest.mark.gpu


def _run(q, k, v, mask, bias=None, causal=False, max_keys=None, rows=None, what=""):
    out, lse = sma.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), mask.cuda(),
                                   None if bias is None else bias.cuda(), causal, max_keys=max_keys)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    ref_o, ref_l = masked_oracle(q, k, v, mask, bias, causal, rows)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, rows=rows, what=what)
    return out, lse


def _qkv(rng, b, lq, lk, h, kvh, d, dtype="bf16"):
    return (wl.normal(rng, (b, lq, h, d), dtype), wl.normal(rng, (b, lk, kvh, d), dtype),
            wl.normal(rng, (b, lk, kvh, d), dtype))


# ~40% of 1500 keys kept: about 600 compacted keys, 4 full tiles and a ragged one
B, LQ, LK, H, KVH, D = 2, 300, 1500, 8, 2, 128
KP = sma.round_up_k(LK)


@pytest.mark.parametrize("mshape", [(1, 1, 1, KP), (B, KVH, 1, KP), (B, 1, 1, KP), (1, KVH, 1, KP)],
                         ids=str)
@pytest.mark.parametrize("bshape", [None, (B, KVH, 1, KP), (1, H, LQ, KP), (1, 1, 1, KP)], ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_small_broadcast_combinations(mshape, bshape, causal):
    rng = wl.rng_for(21)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, D)
    mask = torch.from_numpy(rng.random(mshape) < 0.4)
    bias = wl.normal(rng, bshape, "bf16") if bshape else None
    _run(q, k, v, mask, bias, causal, what=f"{mshape} {bshape} {causal}")


@pytest.mark.parametrize("dtype,d", [("fp16", 128), ("bf16", 64), ("fp32", 64), ("fp32", 128)])
def test_dtypes_and_head_dims(dtype, d):
    rng = wl.rng_for(22)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, d, dtype)
    mask = torch.from_numpy(rng.random((B, KVH, 1, KP)) < 0.3)
    bias = wl.normal(rng, (B, H, 1, KP), "fp32")
    _run(q, k, v, mask, bias, True, what=f"{dtype} d={d}")


def test_short_queries_many_keys():
    """16 queries over ~10k kept of 20k keys: 4 units, so the compacted key
    tiles of each are cut into segments on separate SMs and merged."""
    rng = wl.rng_for(26)
    q, k, v = _qkv(rng, 1, 16, 20000, 8, 2, D)
    kp = sma.round_up_k(20000)
    mask = torch.from_numpy(rng.random((1, 2, 1, kp)) < 0.5)
    bias = wl.normal(rng, (1, 8, 16, kp), "bf16")
    _run(q, k, v, mask, bias, True, what="short gather")


def test_mha_mask_per_head():
    """heads == kv_heads: a mask row per head."""
    rng = wl.rng_for(23)
    q, k, v = _qkv(rng, 2, 257, 900, 4, 4, D)
    mask = torch.from_numpy(rng.random((2, 4, 1, sma.round_up_k(900))) < 0.5)
    _run(q, k, v, mask, None, True, what="mha")


def test_max_keys_exact_bound():
    """max_keys equal to the largest kept count sizes the compacted operands
    exactly; both capacities give the oracle's result.  (They need not agree
    bit for bit: the capacity sets how many key-range segments a unit's tiles
    are cut into, and so the order of the fp32 sums.)"""
    rng = wl.rng_for(24)
    q, k, v = _qkv(rng, B, LQ, LK, H, KVH, D)
    mask = torch.from_numpy(rng.random((B, KVH, 1, KP)) < 0.25)
    mask[..., LK:] = False
    top = int(mask.sum(-1).max())
    _run(q, k, v, mask, None, True, max_keys=top, what="exact max_keys")
    _run(q, k, v, mask, None, True, what="default max_keys")


def test_rows_over_max_keys_raise_device_input():
    rng = wl.rng_for(25)
    q, k, v = _qkv(rng, 1, 128, 512, 2, 1, D)
    mask = torch.from_numpy(rng.random((1, 1, 1, 512)) < 0.6)
    sma.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), mask.cuda(), None, False, max_keys=64)
    assert sma.device_status() == 6  # SMA_ERR_DEVICE_INPUT
    assert sma.device_status() == 0  # reading clears it


def test_empty_and_degenerate_rows():
    """A mask row with no key gives out = 0 and lse = -inf; a row with one
    key copies that key's value row; causal bound cutting every key of the
    first queries."""
    rng = wl.rng_for(26)
    q, k, v = _qkv(rng, 2, 200, 700, 4, 2, D)
    kp = sma.round_up_k(700)
    mask = torch.zeros((2, 2, 1, kp), dtype=torch.bool)
    mask[0, 1, 0, 650] = True                 # one key, late: causal cuts it for early rows
    mask[1, 0, 0, ::7] = True
    mask[1, 0, 0, 700:] = True                # pad columns never count
    out, lse = _run(q, k, v, mask, None, True, what="degenerate")
    assert (out[0, :, 0:2] == 0).all() and torch.isneginf(lse[0, 0:2]).all()   # kv head 0 of batch 0
    assert (out[1, :, 2:4] == 0).all() and torch.isneginf(lse[1, 2:4]).all()   # kv head 1 of batch 1
    # rows of batch 0, kv head 1 that see key 650 (q >= 650 - 500) copy v[650]
    seen = out[0, 150:, 2:4].float()
    assert torch.allclose(seen, v[0, 650, 1].float().cuda().expand_as(seen), atol=1e-2)
    assert torch.isneginf(lse[0, 2:4, :150]).all()


def test_equals_masked_path():
    """Same arguments through masked_attn_fwd and sparse_attn_fwd."""
    rng = wl.rng_for(27)
    q, k, v = (t.cuda() for t in _qkv(rng, B, LQ, LK, H, KVH, D))
    mask = torch.from_numpy(rng.random((B, KVH, 1, KP)) < 0.2).cuda()
    bias = wl.normal(rng, (B, KVH, 1, KP), "bf16").cuda()
    o1, l1 = sma.masked_attn_fwd(q, k, v, mask, bias, True)
    o2, l2 = sma.sparse_attn_fwd(q, k, v, mask, bias, True)
    assert (o1.float() - o2.float()).abs().max() <= 2e-2
    dead = torch.isneginf(l1)
    assert torch.equal(dead, torch.isneginf(l2))
    assert (l1[~dead] - l2[~dead]).abs().max() <= 1e-2


def test_unsupported_masks_are_rejected():
    rng = wl.rng_for(28)
    q, k, v = (t.cuda() for t in _qkv(rng, B, LQ, LK, H, KVH, D))
    per_query = torch.ones((1, 1, LQ, KP), dtype=torch.bool, device="cuda")
    with pytest.raises(sma.SmaError, match="broadcast over queries"):
        sma.sparse_attn_fwd(q, k, v, per_query)
    per_qhead = torch.ones((1, H, 1, KP), dtype=torch.bool, device="cuda")
    with pytest.raises(sma.SmaError, match="shared by the query heads"):
        sma.sparse_attn_fwd(q, k, v, per_qhead)


def test_topk_workload_sampled():
    """The top-k workload end to end: keep mask (B, KVH, 1, Lk) from the
    dynamic top-k, 32 query heads, causal; max_keys = window."""
    w = wl.TOPK
    bias, pre = wl.topk_inputs(w)
    keep = sma.dynamic_topk_mask(bias.cuda(), w.n_k, w.window, pre.cuda())
    q, k, v = wl.topk_attention_inputs(w)
    rows = sample_tiles(w.n_q, picks=(0, 0.5, 1.0))
    _run(q, k, v, keep.cpu(), None, True, max_keys=w.window, rows=rows, what="topk sparse")


def test_topk_workload_all_rows_match_masked():
    """All rows at full size, against the dense-walk kernel (itself checked
    against the oracle on sampled rows)."""
    w = wl.TOPK
    bias, pre = wl.topk_inputs(w)
    keep = sma.dynamic_topk_mask(bias.cuda(), w.n_k, w.window, pre.cuda())
    q, k, v = (t.cuda() for t in wl.topk_attention_inputs(w))
    o1, l1 = sma.masked_attn_fwd(q, k, v, keep, None, True)
    o2, l2 = sma.sparse_attn_fwd(q, k, v, keep, None, True, max_keys=w.window)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    err = (o1.float() - o2.float()).abs()
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert torch.equal(torch.isneginf(l1), torch.isneginf(l2))
