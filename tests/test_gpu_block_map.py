"""GPU: dfa_block_map and mask_tile_summary match the oracle bit for bit."""
import itertools

import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import tiles as tl
from tests._helpers import dflash_block_map_oracle

pytestmark = pytest.mark.gpu


def _check_map(anchors, ctx_len, bs, is_causal, layer, window):
    got = sma.dfa_block_map(anchors.cuda(), ctx_len, bs, is_causal, layer, window)
    want = dflash_block_map_oracle(anchors, ctx_len, bs, is_causal, layer, window)
    for g, w, name in zip(got, want, ("num_full", "full_idx", "num_part", "part_idx")):
        np.testing.assert_array_equal(g.cpu().numpy(), w, err_msg=name)
    assert sma.device_status() == 0


def test_tiny_workload_map():
    w = wl.DFLASH_TINY
    _, _, _, anchors = wl.dflash_inputs(w)
    _check_map(anchors, w.ctx_len, w.block_size, None, 0, 0)


@pytest.mark.parametrize("w", [wl.DFLASH_TRAIN_FULL, wl.DFLASH_TRAIN_SLIDING], ids=lambda w: w.name)
def test_training_workload_maps(w):
    _, _, _, anchors = wl.dflash_inputs(w)
    _check_map(anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window)


@pytest.mark.parametrize("w", [wl.DFLASH_LONG_FULL, wl.DFLASH_LONG_SLIDING], ids=lambda w: w.name)
def test_long_context_maps(w):
    rng = wl.rng_for(w.seed)
    anchors = wl.sorted_anchors(rng, w.batch, w.n_blocks, w.ctx_len)
    _check_map(anchors, w.ctx_len, w.block_size, w.is_causal, w.layer_type, w.sliding_window)


def test_randomised_sweep():
    rng = np.random.default_rng(123)
    cases = 0
    for ctx, n, bs in [(0, 9, 16), (57, 11, 16), (300, 20, 7), (129, 1, 128), (1000, 3, 100),
                       (256, 64, 4)]:
        for is_causal, layer, win in itertools.product((None, 0, 1), (0, 1), (1, 5, 300)):
            if layer == 0 and win != 1:
                continue
            sort = bool(rng.integers(0, 2))
            anchors = wl.random_anchors(rng, 2, n, ctx, sort=sort, low=0)
            anchors[0, 0] = 0
            anchors[1, -1] = ctx
            _check_map(anchors, ctx, bs, is_causal, layer, win)
            cases += 1
    assert cases > 50


def test_out_of_range_anchor_sets_device_error():
    anchors = torch.tensor([[3, 99]], dtype=torch.int32)   # 99 > ctx_len
    sma.dfa_block_map(anchors.cuda(), 16, 4)
    assert sma.device_status() == 6                          # SMA_ERR_DEVICE_INPUT
    assert sma.device_status() == 0                          # read clears it


@pytest.mark.parametrize("shape,k_len", [((1, 1, 300, 256), 200), ((2, 3, 1, 384), 384),
                                         ((2, 1, 129, 512), 500), ((1, 1, 8192, 8064), 8000)])
def test_mask_tile_summary(shape, k_len):
    rng = np.random.default_rng(sum(shape))
    dense = rng.random(shape) < 0.5
    # carve out full and empty tiles
    dense[..., :128, :128] = True
    if shape[2] > 128:
        dense[..., 128:256, :128] = False
    dense[..., :, k_len:] = True                           # padding never counts
    m = torch.from_numpy(dense)
    got = sma.mask_tile_summary(m.cuda(), k_len).cpu().numpy()
    np.testing.assert_array_equal(got, tl.mask_tile_summary(dense, k_len))


def test_mask_tile_summary_broadcast_strides():
    rng = np.random.default_rng(5)
    base = torch.from_numpy(rng.random((1, 1, 260, 256)) < 0.97)
    view = base.expand(3, 2, 260, 256)                    # stride-0 batch/head dims
    got = sma.mask_tile_summary(base.cuda().expand(3, 2, 260, 256), 250)
    want = tl.mask_tile_summary(view.numpy(), 250)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
