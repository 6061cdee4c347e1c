"""GPU: dynamic_topk_mask matches the oracle bit for bit; the top-k mask then
drives masked_attn_fwd."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import topk as tk
from tests._helpers import f64, sample_tiles
from tests.test_gpu_masked import _run

pytestmark = pytest.mark.gpu

SENT = {torch.bfloat16: tk.FINFO_MIN["bf16"], torch.float16: tk.FINFO_MIN["fp16"],
        torch.float32: tk.FINFO_MIN["fp32"]}


def _check(bias, k_len, window, pre_mask=None, q_len=None):
    got = sma.dynamic_topk_mask(bias.cuda(), k_len, window,
                                None if pre_mask is None else pre_mask.cuda(), q_len=q_len)
    pm = None
    if pre_mask is not None:
        pm = tk.normalize_pre_mask(pre_mask.numpy(), bias.shape[0],
                                   bias.shape[2] if q_len is None else q_len, k_len)
    want = tk.dynamic_topk_keep(f64(bias), k_len, pm, window, SENT[bias.dtype])
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    return got


def test_topk_workload():
    w = wl.TOPK
    bias, pre = wl.topk_inputs(w)
    got = _check(bias, w.n_k, w.window, pre)
    counts = got.sum(-1).cpu()
    assert (counts == w.window).all()


def test_topk_wide_workload_sampled_rows():
    w = wl.TOPK_WIDE
    bias, pre = wl.topk_inputs(w)
    got = sma.dynamic_topk_mask(bias.cuda(), w.n_k, w.window, pre.cuda()).cpu()
    for (b, h, qr) in [(0, 0, 0), (1, 7, 4095), (1, 3, 1234), (0, 5, 2048)]:
        row = bias[b:b + 1, h:h + 1, qr:qr + 1]
        pm = tk.normalize_pre_mask(pre[b:b + 1].numpy(), 1, w.bias_q, w.n_k)
        want = tk.dynamic_topk_keep(f64(row), w.n_k, pm, w.window, SENT[bias.dtype])
        np.testing.assert_array_equal(got[b, h, qr].numpy(), want[0, 0, 0])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_ties_and_signed_zero(dtype):
    rng = np.random.default_rng(3)
    levels = torch.tensor([-2.0, -0.0, 0.0, 0.5, 1.0, 1.5, 3.0, 7.0])
    idx = torch.from_numpy(rng.integers(0, 8, size=(2, 3, 4, 640)))
    bias = levels[idx].to(dtype)
    bias[0, 0, 0] = 1.0                        # an all-equal row
    bias[0, 0, 1] = -0.0                       # all signed zeros
    bias[0, 0, 2, ::2] = 0.0
    pre = torch.from_numpy(rng.random((2, 1, 4, 600)) < 0.8)
    for window in (1, 7, 100, 333, 599, 600, 1000):
        _check(bias, 600, window, pre)
    _check(bias, 600, 50, None)


def test_window_at_least_lk_is_premask():
    rng = np.random.default_rng(4)
    bias = torch.from_numpy(rng.standard_normal((2, 2, 1, 256), dtype=np.float32)).to(torch.bfloat16)
    pre = torch.from_numpy(rng.random((2, 250)) < 0.5)
    got = _check(bias, 250, 250, pre)
    assert torch.equal(got[:, :, 0, :250].cpu(), pre[:, None, :].expand(2, 2, 250))


def test_premask_of_query_length_pads_invalid():
    rng = np.random.default_rng(5)
    bias = torch.from_numpy(rng.standard_normal((2, 4, 1, 512), dtype=np.float32)).to(torch.bfloat16)
    pre = torch.from_numpy(rng.random((2, 300)) < 0.9)       # q_len 300 < k_len 500
    _check(bias, 500, 320, pre, q_len=300)


def test_few_valid_keys_never_selects_masked():
    bias = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16)
    pre = torch.zeros((1, 128), dtype=torch.bool)
    pre[0, [3, 77]] = True
    got = _check(bias, 128, 16, pre)
    assert got.sum() == 2


def test_topk_then_attention_sampled():
    """End-to-end top-k workload: keep mask (B, KVH, 1, Lk) broadcast over
    queries and over each KV head's query group, causal, 32 heads."""
    w = wl.TOPK
    bias, pre = wl.topk_inputs(w)
    keep = sma.dynamic_topk_mask(bias.cuda(), w.n_k, w.window, pre.cuda())
    q, k, v = wl.topk_attention_inputs(w)
    rows = sample_tiles(w.n_q, picks=(0.25, 1.0))
    _run(q, k, v, keep.cpu(), None, True, rows=rows, what="topk attention")
