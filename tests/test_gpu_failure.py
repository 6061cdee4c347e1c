"""GPU: the bounded-wait failure path reports an error and leaves the CUDA
context usable; argument faults are rejected before any launch."""
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from structured_mask_attention_analytic_b200 import _native as nat
from tests._helpers import assert_attention_close, dflash_oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    assert sma.device_status() == 0
    out = torch.zeros(2, dtype=torch.int64, device="cuda")
    sma.selftest_wait_timeout(50_000_000, out)          # 50 ms, nothing ever arrives
    torch.cuda.synchronize()
    assert sma.device_status() == nat.SMA_ERR_DEVICE_TIMEOUT
    gave_up, waited_ns = out.tolist()
    assert gave_up == 1 and 50_000_000 <= waited_ns < 5_000_000_000
    assert sma.device_status() == 0                      # the read cleared the word
    # the context still runs the real kernels correctly
    w = wl.DFLASH_TINY
    q, k, v, anchors = wl.dflash_inputs(w)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    o, lse = sma.dfa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), anchors.cuda(), w.ctx_len, w.block_size)
    ref_o, ref_l = dflash_oracle(q, k, v, anchors, w.ctx_len, w.block_size, None, 0, 0)
    assert_attention_close(o, lse, ref_o, ref_l, torch.bfloat16, what="after timeout")
    assert sma.device_status() == 0


def test_rejected_arguments_launch_nothing():
    q = torch.zeros((1, 64, 2, 96), dtype=torch.bfloat16, device="cuda")     # head_dim 96
    kv = torch.zeros((1, 128, 2, 96), dtype=torch.bfloat16, device="cuda")
    a = torch.tensor([[16, 32, 48, 64]], dtype=torch.int32, device="cuda")
    with pytest.raises(sma.SmaError) as e:
        sma.dfa_attn_fwd(q, kv, kv, a, 64, 16)
    assert e.value.status == nat.SMA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert sma.device_status() == 0
