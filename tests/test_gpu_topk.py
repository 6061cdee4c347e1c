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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_many_rows_random_full_check(dtype):
    """Enough rows for the many-rows launch shape; N(0,1) values, ragged key
    length, 2D pre-mask; every row checked."""
    rng = np.random.default_rng(6)
    bias = torch.from_numpy(rng.standard_normal((2, 4, 40, 3072), dtype=np.float32)).to(dtype)
    pre = torch.from_numpy(rng.random((2, 3000)) < 0.85)
    for window in (1, 37, 375, 2000, 2999):
        _check(bias, 3000, window, pre)
    _check(bias, 3000, 700, None)


@pytest.mark.parametrize("rows", [(1, 1, 4), (2, 4, 40)], ids=["few", "many"])
def test_heavy_ties_take_the_exact_fallback(rows):
    """Eight distinct values: the sample bracket cannot isolate the threshold
    and the full bisection decides."""
    rng = np.random.default_rng(7)
    levels = torch.tensor([-3.0, -1.0, -0.0, 0.0, 0.25, 1.0, 2.0, 9.0])
    bias = levels[torch.from_numpy(rng.integers(0, 8, size=rows + (2048,)))].to(torch.bfloat16)
    for window in (1, 300, 1024, 2047):
        _check(bias, 2048, window, None)


@pytest.mark.parametrize("rows", [(1, 1, 4), (2, 4, 40)], ids=["few", "many"])
def test_infinities_below_the_sentinel(rows):
    """-inf values rank below the pre-mask sentinel: when the window reaches
    them, pre-masked positions (holding the sentinel) pass the threshold and
    the pre-mask must still clear them."""
    rng = np.random.default_rng(8)
    vals = rng.standard_normal(rows + (1024,), dtype=np.float32)
    vals[rng.random(vals.shape) < 0.3] = -np.inf
    vals[rng.random(vals.shape) < 0.05] = np.inf
    bias = torch.from_numpy(vals).to(torch.bfloat16)
    pre = torch.from_numpy(rng.random((rows[0], 1000)) < 0.7)
    for window in (10, 400, 700, 900):
        _check(bias, 1000, window, pre)


def test_longest_register_row_and_the_next():
    """16384 columns (the register-resident kernel's limit) and 16512 (the
    radix-select kernel) give the oracle's masks."""
    rng = np.random.default_rng(9)
    for k_len in (16384, 16500):
        kp = sma.round_up_k(k_len)
        bias = torch.from_numpy(rng.standard_normal((1, 2, 3, kp), dtype=np.float32)).to(torch.bfloat16)
        pre = torch.from_numpy(rng.random((1, k_len)) < 0.9)
        _check(bias, k_len, 2048, pre)


def test_output_aligned_to_8_bytes_only():
    """An output that is 8- but not 16-byte aligned takes the radix-select
    kernel and gives the same mask."""
    rng = np.random.default_rng(10)
    bias = torch.from_numpy(rng.standard_normal((1, 1, 2, 512), dtype=np.float32)).to(torch.bfloat16).cuda()
    buf = torch.empty(2 * 512 + 8, dtype=torch.bool, device="cuda")
    out = buf[8:].view(1, 1, 2, 512)
    got = sma.dynamic_topk_mask(bias, 500, 64, None, out=out)
    ref = sma.dynamic_topk_mask(bias, 500, 64, None)
    assert torch.equal(got, ref)
