"""GPU: DFlash inference attention (one draft block after a padded context
per row) agrees with the float64 oracle of the inference mask."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from oracle import dflash_mask as dm
from tests._helpers import assert_attention_close, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layer,is_causal,window", [(0, None, 0), (1, None, 300), (0, True, 0), (1, False, 7)],
                         ids=str)
@pytest.mark.parametrize("D", [64, 128])
def test_spec_generate(layer, is_causal, window, D):
    rng = wl.rng_for(41)
    B, H, KVH, Lc, bs = 4, 8, 2, 1000, 16
    q = wl.normal(rng, (B, bs, H, D), "bf16")
    k = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    v = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    ctx_lens = torch.tensor([0, 1, 517, Lc], dtype=torch.int32)
    out, lse = sma.dflash_spec_generate_fwd(q.cuda(), k.cuda(), v.cuda(), ctx_lens.cuda(), Lc, is_causal, layer,
                                            window)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    causal = dm.resolve_in_block_causal(is_causal, layer)
    w = dm.resolve_window(layer, window) if layer == dm.LAYER_SLIDING else None
    keep = dm.spec_generate_keep_mask(ctx_lens.numpy(), Lc, bs, causal, w)[:, None]
    ref_o, ref_l = at.attention(f64(q), f64(k), f64(v), keep=keep)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, what=f"spec {layer} {is_causal} {window} {D}")


def test_spec_generate_long_context_sampled_heads():
    """A 32k-token context (the long-context workload's size) with one block."""
    rng = wl.rng_for(42)
    B, H, KVH, D, Lc, bs = 1, 32, 8, 128, 32768, 16
    q = wl.normal(rng, (B, bs, H, D), "bf16")
    k = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    v = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    ctx_lens = torch.tensor([30001], dtype=torch.int32)
    out, lse = sma.dflash_spec_generate_fwd(q.cuda(), k.cuda(), v.cuda(), ctx_lens.cuda(), Lc, True)
    torch.cuda.synchronize()
    keep = dm.spec_generate_keep_mask(ctx_lens.numpy(), Lc, bs, True, None)[:, None]
    ref_o, ref_l = at.attention(f64(q), f64(k), f64(v), keep=keep, workers=8)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, what="spec long")


@pytest.mark.parametrize("H,KVH", [(8, 2), (16, 2), (4, 2)], ids=str)
@pytest.mark.parametrize("is_causal", [True, False])
def test_spec_generate_segments_of_mixed_lengths(is_causal, H, KVH):
    """An 8k context with one block of 16 queries: the group's heads share a
    128-row tile (4, 8 or 2 heads of 32, 16 or 64 queries) and every unit's
    key tiles are cut into segments.  Row 0's list holds two tiles (most
    segments empty), row 1's about 64."""
    rng = wl.rng_for(43)
    B, D, Lc, bs = 2, 128, 8192, 16
    q = wl.normal(rng, (B, bs, H, D), "bf16")
    k = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    v = wl.normal(rng, (B, Lc + bs, KVH, D), "bf16")
    ctx_lens = torch.tensor([37, 8000], dtype=torch.int32)
    out, lse = sma.dflash_spec_generate_fwd(q.cuda(), k.cuda(), v.cuda(), ctx_lens.cuda(), Lc, is_causal)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    keep = dm.spec_generate_keep_mask(ctx_lens.numpy(), Lc, bs, is_causal, None)[:, None]
    ref_o, ref_l = at.attention(f64(q), f64(k), f64(v), keep=keep, workers=8)
    assert_attention_close(out, lse, ref_o, ref_l, q.dtype, what=f"spec segments {is_causal}")
