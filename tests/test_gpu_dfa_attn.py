"""GPU: dfa_attn_fwd agrees with the float64 dense-mask oracle."""
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from tests._helpers import assert_attention_close, dflash_oracle, sample_tiles

pytestmark = pytest.mark.gpu


def _run(q, k, v, anchors, ctx, bs, is_causal, layer, window, rows=None, what=""):
    out, lse = sma.dfa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), anchors.cuda(), ctx, bs, is_causal, layer,
                                window)
    torch.cuda.synchronize()
    assert sma.device_status() == 0, what
    ref_o, ref_l = dflash_oracle(q, k, v, anchors, ctx, bs, is_causal, layer, window, rows=rows)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, rows=rows, what=what)
    return out, lse


def test_tiny_workload_fp32():
    w = wl.DFLASH_TINY
    q, k, v, anchors = wl.dflash_inputs(w)
    _run(q, k, v, anchors, w.ctx_len, w.block_size, None, 0, 0, what="tiny fp32")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_tiny_workload_half(dtype):
    w = wl.DFLASH_TINY
    q, k, v, anchors = wl.dflash_inputs(w)
    _run(q.to(dtype), k.to(dtype), v.to(dtype), anchors, w.ctx_len, w.block_size, None, 0, 0,
         what=f"tiny {dtype}")


# Several query/key tiles, ragged tails (ctx 300, 40 blocks of 16 -> Nq 640, Lk 940).
MEDIUM = [
    # (B, H, KVH, d, ctx, N, bs, is_causal, layer, window, dtype)
    (2, 8, 2, 128, 300, 40, 16, None, 0, 0, torch.bfloat16),
    (2, 8, 2, 128, 300, 40, 16, None, 1, 100, torch.bfloat16),
    (2, 8, 2, 128, 300, 40, 16, 1, 0, 0, torch.bfloat16),
    (2, 8, 2, 128, 300, 40, 16, 0, 1, 7, torch.bfloat16),
    (1, 6, 2, 128, 300, 40, 16, None, 0, 0, torch.bfloat16),      # odd group (3 heads per KV head)
    (1, 4, 4, 128, 300, 40, 16, 1, 1, 50, torch.bfloat16),        # MHA
    (2, 8, 2, 64, 300, 40, 16, None, 1, 100, torch.bfloat16),      # head_dim 64
    (2, 8, 2, 128, 300, 40, 16, None, 0, 0, torch.float16),
    (1, 4, 2, 128, 1000, 3, 100, 1, 0, 0, torch.bfloat16),        # large blocks
    (2, 4, 2, 128, 0, 24, 16, None, 0, 0, torch.bfloat16),         # no context
    (1, 4, 2, 128, 300, 40, 16, None, 0, 0, torch.float32),
    (1, 4, 2, 64, 300, 40, 16, 1, 1, 33, torch.float32),
]


@pytest.mark.parametrize("case", MEDIUM, ids=lambda c: "-".join(str(x) for x in c))
def test_medium_cases(case):
    b, h, kvh, d, ctx, n, bs, is_causal, layer, window, dtype = case
    rng = wl.rng_for(100 + MEDIUM.index(case))
    q = wl.normal(rng, (b, n * bs, h, d), "fp32").to(dtype)
    k = wl.normal(rng, (b, ctx + n * bs, kvh, d), "fp32").to(dtype)
    v = wl.normal(rng, (b, ctx + n * bs, kvh, d), "fp32").to(dtype)
    anchors = wl.random_anchors(rng, b, n, ctx, sort=True, low=0)
    _run(q, k, v, anchors, ctx, bs, is_causal, layer, window, what=str(case))


def test_strided_views():
    """q/k/v given as views into a packed [B, L, heads, 3, d]-like buffer."""
    rng = wl.rng_for(77)
    b, ctx, n, bs, h, kvh, d = 1, 200, 20, 16, 4, 2, 128
    big = wl.normal(rng, (b, ctx + n * bs, kvh * 2, d), "bf16").cuda()
    k, v = big[:, :, 0::2], big[:, :, 1::2]
    q = wl.normal(rng, (b, n * bs, h * 2, d), "bf16").cuda()[:, :, ::2]
    assert not q.is_contiguous() and k.stride(2) == 2 * d
    anchors = wl.random_anchors(rng, b, n, ctx, sort=True)
    out, lse = sma.dfa_attn_fwd(q, k, v, anchors.cuda(), ctx, bs)
    ref_o, ref_l = dflash_oracle(q, k, v, anchors, ctx, bs, None, 0, 0)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, what="strided")


@pytest.mark.parametrize("w", [wl.DFLASH_TRAIN_FULL, wl.DFLASH_TRAIN_SLIDING], ids=lambda w: w.name)
def test_training_workload_sampled(w):
    q, k, v, anchors = wl.dflash_inputs(w)
    rows = sample_tiles(w.n_q, picks=(0, 0.37, 1.0))
    _run(q, k, v, anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window,
         rows=rows, what=w.name)


@pytest.mark.parametrize("w", [wl.DFLASH_LONG_FULL, wl.DFLASH_LONG_SLIDING], ids=lambda w: w.name)
def test_long_context_sampled(w):
    q, k, v, anchors = wl.dflash_inputs(w)
    rows = sample_tiles(w.n_q, picks=(0.5, 1.0))
    _run(q, k, v, anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window,
         rows=rows, what=w.name)


def test_repeated_calls_are_deterministic():
    w = wl.DFLASH_TINY
    q, k, v, anchors = wl.dflash_inputs(w)
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
    o1, l1 = sma.dfa_attn_fwd(q, k, v, anchors.cuda(), w.ctx_len, w.block_size)
    o2, l2 = sma.dfa_attn_fwd(q, k, v, anchors.cuda(), w.ctx_len, w.block_size)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
