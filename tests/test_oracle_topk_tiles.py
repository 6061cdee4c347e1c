"""Pins for the oracle's top-k keep mask and tile classification (CPU only)."""
import os

import numpy as np
import pytest
import torch

from oracle import dflash_mask as dm
from oracle import tiles as tl
from oracle import topk as tk
from tests.conftest import GOLDEN


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split("#")[0] for ln in f if ln.split("#")[0].strip()]


# ---------------------------------------------------------------- top-k


def test_sentinels_equal_torch_finfo_min():
    assert tk.FINFO_MIN["bf16"] == torch.finfo(torch.bfloat16).min
    assert tk.FINFO_MIN["fp16"] == torch.finfo(torch.float16).min
    assert tk.FINFO_MIN["fp32"] == torch.finfo(torch.float32).min


def test_topk_worked_rows():
    rows = _rows("topk_worked.txt")
    assert len(rows) == 7
    for row in rows:
        head, bias_s, pm_s, want_s = row.split("|")
        n_k, window = (int(x) for x in head.split())
        bias = np.array([float(x) for x in bias_s.split()]).reshape(1, 1, 1, -1)
        pm = np.array([int(x) for x in pm_s.split()], dtype=bool).reshape(1, 1, 1, -1)
        want = np.array([int(x) for x in want_s.split()], dtype=bool)
        got = tk.dynamic_topk_keep(bias, n_k, pm, window, tk.FINFO_MIN["bf16"])
        np.testing.assert_array_equal(got[0, 0, 0], want, err_msg=row)


def test_topk_equals_torch_topk_without_ties():
    rng = np.random.default_rng(0)
    bias = rng.standard_normal((2, 3, 4, 256))             # distinct values
    for w in (1, 7, 64, 200):
        got = tk.dynamic_topk_keep(bias, 256, None, w, tk.FINFO_MIN["fp32"])
        idx = torch.topk(torch.from_numpy(bias), w, dim=-1, largest=True, sorted=False).indices
        ref = torch.zeros(bias.shape, dtype=torch.bool).scatter_(-1, idx, True).numpy()
        np.testing.assert_array_equal(got, ref)


def test_topk_brute_force_with_ties_and_premask():
    rng = np.random.default_rng(1)
    for trial in range(200):
        n_k = int(rng.integers(1, 24))
        kpad = n_k + int(rng.integers(0, 5))
        levels = np.array([-1.5, -0.0, 0.0, 0.25, 2.0])
        row = levels[rng.integers(0, len(levels), size=kpad)]
        pm = rng.random(kpad) < 0.7
        w = int(rng.integers(1, n_k + 3))
        got = tk.dynamic_topk_keep(row.reshape(1, 1, 1, -1), n_k, pm.reshape(1, 1, 1, -1), w,
                                   tk.FINFO_MIN["bf16"])[0, 0, 0]
        # brute force: python's stable sort on (value desc, index asc)
        vals = [(row[c] if pm[c] else tk.FINFO_MIN["bf16"]) for c in range(n_k)]
        order = sorted(range(n_k), key=lambda c: (-(vals[c] + 0.0), c))
        want = np.zeros(kpad, dtype=bool)
        for c in order[:w]:
            want[c] = pm[c]
        np.testing.assert_array_equal(got, want, err_msg=f"trial {trial}")


def test_topk_invariants_on_bf16_like_rows():
    rng = np.random.default_rng(2)
    vals = torch.from_numpy(rng.standard_normal((4, 2048), dtype=np.float32)).to(torch.bfloat16)
    bias = vals.double().numpy().reshape(4, 1, 1, 2048)
    pm = rng.random((4, 1, 1, 2048)) < 0.9
    w = 300
    keep = tk.dynamic_topk_keep(bias, 2048, pm, w, tk.FINFO_MIN["bf16"])
    for r in range(4):
        b, m, k = bias[r, 0, 0], pm[r, 0, 0], keep[r, 0, 0]
        assert k.sum() == w                     # enough valid keys
        assert not (k & ~m).any()
        kept_min = b[k].min()
        unkept_valid = b[~k & m]
        assert (unkept_valid <= kept_min).all()
        ties = np.nonzero((b == kept_min) & m)[0]
        chosen = ties[k[ties]]
        assert list(chosen) == list(ties[: len(chosen)])   # lowest indices win


def test_normalize_pre_mask_shapes():
    m = np.array([[1, 1, 0, 1], [0, 1, 1, 1]], dtype=bool)
    out = tk.normalize_pre_mask(m, 2, 3, 4)              # length == key_len
    assert out.shape == (2, 1, 1, 4)
    np.testing.assert_array_equal(out[:, 0, 0], m)
    out = tk.normalize_pre_mask(m[:, :3], 2, 3, 5)       # length == query_len < key_len: pad False
    np.testing.assert_array_equal(out[:, 0, 0], [[1, 1, 0, 0, 0], [0, 1, 1, 0, 0]])
    out = tk.normalize_pre_mask(m, 2, 4, 2)              # query_len > key_len: cut
    np.testing.assert_array_equal(out[:, 0, 0], [[1, 1], [0, 1]])
    with pytest.raises(ValueError):
        tk.normalize_pre_mask(m, 2, 7, 9)


def test_window_at_least_lk_returns_premask():
    rng = np.random.default_rng(3)
    bias = rng.standard_normal((1, 2, 1, 16))
    pm = rng.random((1, 2, 1, 16)) < 0.5
    got = tk.dynamic_topk_keep(bias, 12, pm, 12, tk.FINFO_MIN["fp32"])
    np.testing.assert_array_equal(got[..., :12], pm[..., :12])
    assert not got[..., 12:].any()


# ---------------------------------------------------------------- tiles


def test_tile_codes_worked_cases():
    code = {"F": tl.FULL, "P": tl.PARTIAL, "E": tl.EMPTY}
    rows = _rows("tile_map_worked.txt")
    assert len(rows) == 6
    for row in rows:
        left, right = row.split("|")
        ctx, bs, anchors = left.split()
        ctx, bs = int(ctx), int(bs)
        anchors = np.array([[int(a) for a in anchors.split(",")]])
        n_q = anchors.shape[1] * bs
        n_k = ctx + n_q
        keep = dm.dflash_keep_mask(anchors, ctx, bs, False, None)[0]
        got = tl.tile_codes(keep, n_k)
        assert got.shape == (1, 3)
        assert list(got[0]) == [code[c] for c in right.split()], row


def test_lists_are_ascending_and_padded():
    codes = np.array([[[2, 0, 1, 2, 1]], [[0, 0, 0, 0, 0]]], dtype=np.uint8)
    nf, fi, npart, pi = tl.lists_from_codes(codes)
    assert nf.tolist() == [[2], [0]] and npart.tolist() == [[2], [0]]
    assert fi[0, 0].tolist() == [0, 3, -1, -1, -1]
    assert pi[0, 0].tolist() == [2, 4, -1, -1, -1]
    assert (fi[1] == -1).all() and (pi[1] == -1).all()


def test_mask_summary_edges():
    # 130 rows (ragged second query tile), 256 padded columns, Lk = 200
    mask = np.ones((1, 1, 130, 256), dtype=bool)
    s = tl.mask_tile_summary(mask, 200)
    assert s.shape == (1, 1, 2, 2)
    assert s[0, 0, :, 0].tolist() == [tl.FULL, tl.FULL]
    assert s[0, 0, :, 1].tolist() == [tl.PARTIAL, tl.PARTIAL]   # reaches past Lk
    mask[0, 0, 128:, :] = False
    mask[0, 0, 5, 7] = False
    s = tl.mask_tile_summary(mask, 200)
    assert s[0, 0, :, 0].tolist() == [tl.PARTIAL, tl.EMPTY]
    mask[:] = False
    mask[0, 0, 0, 210] = True                                 # only a padded column
    assert (tl.mask_tile_summary(mask, 200) == tl.EMPTY).all()


def test_block_map_codes_agree_with_mask_content():
    rng = np.random.default_rng(4)
    anchors = np.sort(rng.integers(0, 301, size=(2, 20)), axis=1)
    keep = dm.dflash_keep_mask(anchors, 300, 16, True, 100)
    n_q, n_k = keep.shape[1], keep.shape[2]
    nf, fi, npart, pi = tl.block_map_from_rows(lambda b, a, z: keep[b, a:z], 2, n_q, n_k)
    for b in range(2):
        for qt in range(nf.shape[1]):
            rows = keep[b, qt * 128:(qt + 1) * 128]
            for kt in range(-(-n_k // 128)):
                blk = rows[:, kt * 128:(kt + 1) * 128]
                is_full = kt in fi[b, qt, : nf[b, qt]]
                is_part = kt in pi[b, qt, : npart[b, qt]]
                assert is_full == (blk.all() and (kt + 1) * 128 <= n_k)
                assert (is_full or is_part) == bool(blk.any())


def test_key_dim_forms_of_summary_and_topk():
    """A mask of key dim 1 is one flag for every key: its summary equals that
    of the explicit expansion.  A top-k bias of key dim Lk gives the padded
    bias's mask, first Lk columns."""
    rng = np.random.default_rng(21)
    flags = rng.random((2, 1, 300, 1)) < 0.5
    flags[0, 0, :128] = True
    flags[1, 0, 128:256] = False
    np.testing.assert_array_equal(tl.mask_tile_summary(flags, 333),
                                  tl.mask_tile_summary(np.repeat(flags, 384, axis=-1), 333))
    sent = float(np.finfo(np.float32).min)
    bias = rng.standard_normal((2, 2, 3, 384)).astype(np.float32)
    pm = rng.random((2, 1, 1, 333)) < 0.9
    a = tk.dynamic_topk_keep(bias, 333, pm, 50, sent)
    b = tk.dynamic_topk_keep(np.ascontiguousarray(bias[..., :333]), 333, pm, 50, sent)
    assert b.shape == (2, 2, 3, 333)
    np.testing.assert_array_equal(a[..., :333], b)
