"""dfa_attn_fwd_noalloc: the DFlash forward for callers that cannot allocate
device memory (a C host program without its own CUDA memory manager, or a
runtime whose device memory is all pre-reserved by another allocator).  Its
block-map scratch is a fixed 4 MiB array inside the library.

This file is collected last on purpose: the GPU test here runs after every
other test in a run that stops at the first failure.
"""
import ctypes

import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from structured_mask_attention_analytic_b200 import _native as nat
from tests._helpers import TOL, assert_attention_close, dflash_oracle


def _noalloc_via_cabi(q, k, v, anchors, ctx_len, block_size, is_causal, layer_type, window):
    """Calls dfa_attn_fwd_noalloc through the C ABI (ctypes), no workspace."""
    b, nq, h, d = q.shape
    desc = nat.DfaMaskDesc(b, anchors.shape[1], block_size, ctx_len,
                           -1 if is_causal is None else int(is_causal), layer_type, window)
    out = torch.empty_like(q)
    lse = torch.empty((b, h, nq), dtype=torch.float32, device=q.device)
    st = nat.load().dfa_attn_fwd_noalloc(
        ctypes.byref(desc), ctypes.c_void_p(anchors.data_ptr()), nat.SMA_BF16, h, k.shape[2], d,
        ctypes.c_float(0.0),
        ctypes.c_void_p(q.data_ptr()), nat.i64_array(q.stride()[:3]),
        ctypes.c_void_p(k.data_ptr()), nat.i64_array(k.stride()[:3]),
        ctypes.c_void_p(v.data_ptr()), nat.i64_array(v.stride()[:3]),
        ctypes.c_void_p(out.data_ptr()), nat.i64_array(out.stride()[:3]),
        ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    nat.check(st)
    return out, lse


CASES = [
    # (B, H, KVH, d, ctx, N, bs, is_causal, layer, window, seed)
    (2, 8, 2, 128, 300, 40, 16, None, 0, 0, 31),
    (1, 4, 2, 128, 1000, 3, 100, 1, 1, 150, 32),
]


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls_in_a_row():
    """Two calls in a row (the second overwrites the shared scratch the first
    used), each checked element by element against the float64 oracle and
    against dfa_attn_fwd with a caller workspace."""
    max_abs, mean_abs = TOL[torch.bfloat16]
    results = []
    for (b, h, kvh, d, ctx, n, bs, is_causal, layer, window, seed) in CASES:
        rng = wl.rng_for(seed)
        q = wl.normal(rng, (b, n * bs, h, d), "bf16").cuda()
        k = wl.normal(rng, (b, ctx + n * bs, kvh, d), "bf16").cuda()
        v = wl.normal(rng, (b, ctx + n * bs, kvh, d), "bf16").cuda()
        anchors = wl.random_anchors(rng, b, n, ctx, sort=True).cuda()
        got_o, got_l = _noalloc_via_cabi(q, k, v, anchors, ctx, bs, is_causal, layer, window)
        ws_o, ws_l = sma.dfa_attn_fwd(q, k, v, anchors, ctx, bs, is_causal, layer, window)
        results.append((q, k, v, anchors, ctx, bs, is_causal, layer, window, got_o, got_l, ws_o, ws_l))
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    for (q, k, v, anchors, ctx, bs, is_causal, layer, window, got_o, got_l, ws_o, ws_l) in results:
        ref_o, ref_l = dflash_oracle(q, k, v, anchors, ctx, bs, is_causal, layer, window)
        assert_attention_close(got_o, got_l, ref_o, ref_l, torch.bfloat16, what="noalloc vs oracle")
        err = (got_o.double() - ws_o.double()).abs()
        assert err.max().item() <= max_abs and err.mean().item() <= mean_abs
        assert torch.equal(torch.isneginf(got_l), torch.isneginf(ws_l))


def test_noalloc_rejects_a_block_map_above_its_scratch():
    # 8 x 512 query tiles x 1025 key tiles of int32 lists is far above 4 MiB;
    # the size check runs on the host before any CUDA call.  Every device
    # pointer is NULL, so a check that fired first would also reject the call
    # without a launch.
    desc = nat.DfaMaskDesc(8, 4096, 16, 65536, 1, 0, 0)
    z = ctypes.c_void_p(0)
    strides = nat.i64_array([1 << 20, 4096, 128])
    st = nat.load().dfa_attn_fwd_noalloc(ctypes.byref(desc), z, nat.SMA_BF16, 32, 8, 128, ctypes.c_float(0.0),
                                         z, strides, z, strides, z, strides, z, strides, None, None)
    assert st == nat.SMA_ERR_WORKSPACE
    assert "4194304" in nat.load().sma_last_error().decode()
