"""Pins for the oracle's DFlash keep mask (CPU only).

The fixtures under tests/golden/ are written by hand from the pages' rules;
the brute-force test walks positions one by one instead of evaluating the
closed-form predicate.
"""
import itertools
import os

import numpy as np
import pytest

from oracle import dflash_mask as dm
from tests.conftest import GOLDEN


def _read(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split("#")[0].strip() for ln in f if ln.split("#")[0].strip()]


def _causal_arg(tok):
    return {"unset": None, "false": 0, "true": 1}[tok]


def _layer_arg(tok):
    return {"full": dm.LAYER_FULL, "sliding": dm.LAYER_SLIDING}[tok]


def test_is_causal_table_matches_pr905():
    rows = _read("is_causal_table.txt")
    assert len(rows) == 6
    for row in rows:
        c, layer, mode = row.split()
        got = dm.resolve_in_block_causal(_causal_arg(c), _layer_arg(layer))
        assert got == (mode == "causal"), row
    # -1 is the C-ABI spelling of "absent"
    assert dm.resolve_in_block_causal(-1, dm.LAYER_FULL) is False
    assert dm.resolve_in_block_causal(-1, dm.LAYER_SLIDING) is True


def test_tiny_workload_visibility_by_hand():
    anchors = np.array([[16, 32, 48, 64]])
    keep = dm.dflash_keep_mask(anchors, 64, 16, dm.resolve_in_block_causal(None, dm.LAYER_FULL), None)
    assert keep.shape == (1, 64, 128)
    for row in _read("dflash_tiny_visibility.txt"):
        parts = row.split()
        j = int(parts[0])
        expect = np.zeros(128, dtype=bool)
        for rng in parts[1:]:
            lo, hi = (int(x) for x in rng.split("-"))
            expect[lo:hi + 1] = True
        for i in range(16):
            np.testing.assert_array_equal(keep[0, j * 16 + i], expect, err_msg=f"block {j} row {i}")
    # block 0 row 0 sees exactly keys 0..15 and 64..79
    assert set(np.nonzero(keep[0, 0])[0]) == set(range(16)) | set(range(64, 80))


def test_window_and_causal_cases_by_hand():
    rows = _read("dflash_window_worked.txt")
    anchors = np.array([[2, 6]])
    cases = []
    for row in rows:
        if row.startswith("case"):
            _, c, layer, w = row.split()
            cases.append((c, layer, int(w), {}))
        else:
            q, keys = row.split(":")
            cases[-1][3][int(q)] = [int(x) for x in keys.split()]
    assert len(cases) == 4
    for c, layer, w, expect in cases:
        lt = _layer_arg(layer)
        causal = dm.resolve_in_block_causal(_causal_arg(c), lt)
        window = dm.resolve_window(lt, w) if lt == dm.LAYER_SLIDING else None
        keep = dm.dflash_keep_mask(anchors, 6, 3, causal, window)
        assert keep.shape == (1, 6, 12)
        for q, keys in expect.items():
            assert list(np.nonzero(keep[0, q])[0]) == keys, (c, layer, q)


@pytest.mark.parametrize("ctx_len,n_blocks,block_size", [(0, 2, 4), (5, 3, 1), (7, 2, 4), (16, 3, 4),
                                                        (9, 1, 16)])
def test_vectorised_mask_equals_position_walk(ctx_len, n_blocks, block_size):
    rng = np.random.default_rng(ctx_len * 100 + n_blocks * 10 + block_size)
    anchors = rng.integers(0, ctx_len + 1, size=(2, n_blocks))
    anchors[0, 0] = 0
    anchors[1, -1] = ctx_len
    n_q = n_blocks * block_size
    n_k = ctx_len + n_q
    for is_causal, layer, w in itertools.product((None, 0, 1), (0, 1), (1, 3, 16)):
        causal = dm.resolve_in_block_causal(is_causal, layer)
        window = w if layer == dm.LAYER_SLIDING else None
        if layer == dm.LAYER_FULL and w != 1:
            continue
        keep = dm.dflash_keep_mask(anchors, ctx_len, block_size, causal, window)
        for b in range(2):
            for q in range(n_q):
                for k in range(n_k):
                    want = dm.dflash_keep_scalar(anchors, ctx_len, block_size, causal, window, b, q, k)
                    assert keep[b, q, k] == want, (is_causal, layer, w, b, q, k)


def test_row_slices_compose():
    rng = np.random.default_rng(7)
    anchors = np.sort(rng.integers(1, 65, size=(2, 8)), axis=1)
    full = dm.dflash_keep_mask(anchors, 64, 8, True, 5)
    parts = [dm.dflash_keep_rows(anchors, 64, 8, True, 5, a, min(a + 24, 64)) for a in range(0, 64, 24)]
    np.testing.assert_array_equal(np.concatenate(parts, axis=1), full)


def test_sliding_window_requires_positive_size():
    with pytest.raises(ValueError):
        dm.resolve_window(dm.LAYER_SLIDING, 0)
    assert dm.resolve_window(dm.LAYER_FULL, 0) is None


@pytest.mark.parametrize("causal,window", [(False, None), (True, None), (True, 5), (False, 3)])
def test_spec_generate_mask_equals_position_walk(causal, window):
    """Inference mask (one block after a padded context) against the scalar
    position walk, plus its plain reading: every context key below the row's
    length, nothing of the padding, the block by the in-block rule."""
    ctx_lens = np.array([0, 7, 20, 13])
    Lc, bs = 20, 6
    m = dm.spec_generate_keep_mask(ctx_lens, Lc, bs, causal, window)
    assert m.shape == (4, bs, Lc + bs)
    for b in range(4):
        for i in range(bs):
            for k in range(Lc + bs):
                want = dm.dflash_keep_scalar(ctx_lens.reshape(-1, 1), Lc, bs, causal, window, b, i, k)
                assert m[b, i, k] == want
            assert not m[b, i, ctx_lens[b]:Lc].any()          # padding never kept
            if window is None:
                assert m[b, i, :ctx_lens[b]].all()            # the whole context
            t = np.arange(bs)
            block = (t <= i) if causal else np.ones(bs, bool)
            if window is not None:
                block &= i - t < window
            assert (m[b, i, Lc:] == block).all()
