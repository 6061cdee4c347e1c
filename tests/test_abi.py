"""The C-ABI library loads, exports every symbol include/sma.h declares, and
its host-side validation rejects bad arguments before touching the GPU.
CPU only: no call here reaches a CUDA API (validation runs first)."""
import ctypes
import os
import re

import pytest

from structured_mask_attention_analytic_b200 import _native as nat
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "sma.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text,
                       flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ["dfa_block_map", "dfa_attn_fwd", "masked_attn_fwd", "dynamic_topk_mask",
                 "mask_tile_summary", "sma_last_error", "sma_device_status"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = nat.load()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert lib.sma_abi_version() == 1


def test_block_map_dims_on_host():
    d = nat.DfaMaskDesc(2, 256, 16, 4096, -1, 0, 0)
    qt, kt = ctypes.c_int32(), ctypes.c_int32()
    assert nat.load().dfa_block_map_dims(ctypes.byref(d), ctypes.byref(qt), ctypes.byref(kt)) == 0
    assert (qt.value, kt.value) == (32, 64)
    d = nat.DfaMaskDesc(1, 4, 16, 64, -1, 0, 0)
    assert nat.load().dfa_block_map_dims(ctypes.byref(d), ctypes.byref(qt), ctypes.byref(kt)) == 0
    assert (qt.value, kt.value) == (1, 1)


@pytest.mark.parametrize("fields,msg", [
    ((0, 4, 16, 64, -1, 0, 0), "batch"),
    ((1, 4, 16, 64, 2, 0, 0), "is_causal"),
    ((1, 4, 16, 64, -1, 3, 0), "layer_type"),
    ((1, 4, 16, 64, -1, 1, 0), "sliding_window"),
    ((1, 4, 0, 64, -1, 0, 0), "block_size"),
])
def test_bad_descriptors_are_rejected(fields, msg):
    d = nat.DfaMaskDesc(*fields)
    qt, kt = ctypes.c_int32(), ctypes.c_int32()
    st = nat.load().dfa_block_map_dims(ctypes.byref(d), ctypes.byref(qt), ctypes.byref(kt))
    assert st == nat.SMA_ERR_INVALID_ARG
    assert msg in nat.load().sma_last_error().decode()


def test_workspace_sizes_on_host():
    lib = nat.load()
    d = nat.DfaMaskDesc(1, 2048, 16, 32768, 1, 0, 0)
    n = ctypes.c_size_t()
    assert lib.dfa_attn_fwd_workspace_size(ctypes.byref(d), 32, 8, 128, ctypes.byref(n)) == 0
    # num_full + num_part (256 each) + two 256 x 512 index arrays, 256-byte aligned
    assert n.value >= 2 * 256 * 4 + 2 * 256 * 512 * 4
    assert lib.dfa_attn_fwd_workspace_size(ctypes.byref(d), 32, 8, 96, ctypes.byref(n)) == nat.SMA_ERR_UNSUPPORTED
    assert lib.dfa_attn_fwd_workspace_size(ctypes.byref(d), 30, 8, 128, ctypes.byref(n)) == nat.SMA_ERR_INVALID_ARG
    ms = nat.i64_array([1, 1, 8192, 8064])
    assert lib.masked_attn_fwd_workspace_size(4, 16, 4, 8192, 8000, 128, ms, ctypes.byref(n)) == 0
    assert n.value > 0
    assert lib.masked_attn_fwd_workspace_size(8, 32, 8, 1, 16384, 128, None, ctypes.byref(n)) == 0
    assert n.value > 0


def test_workspace_holds_key_range_segments_for_short_queries():
    """16 queries after an 8k context (4 units on a 148-SM part): the forward
    workspace holds the partial results of 16 key-range segments per unit
    (fp32 O and (max, sum) per segment and row); 64 batch rows fill the SMs
    and need no segments."""
    lib = nat.load()
    n = ctypes.c_size_t()
    short = nat.DfaMaskDesc(1, 1, 16, 8192, 1, 0, 0)
    assert lib.dfa_attn_fwd_workspace_size(ctypes.byref(short), 8, 2, 128, ctypes.byref(n)) == 0
    rows = 1 * 8 * 16
    assert n.value >= 16 * rows * (128 * 4 + 8)
    wide = nat.DfaMaskDesc(64, 1, 16, 8192, 1, 0, 0)
    assert lib.dfa_attn_fwd_workspace_size(ctypes.byref(wide), 8, 2, 128, ctypes.byref(n)) == 0
    assert n.value < 64 * 65 * 4 * 2 + 64 * 4 * 2 + 4096
    ms = nat.i64_array([1, 1, 24, 5120])
    assert lib.masked_attn_fwd_workspace_size(1, 8, 2, 24, 5000, 128, ms, ctypes.byref(n)) == 0
    assert n.value >= 10 * (8 * 24) * (128 * 4 + 8)


def _masked_call(**over):
    """masked_attn_fwd with fake (never dereferenced) aligned pointers."""
    a = dict(dtype=0, batch=2, heads=4, kv_heads=2, q_len=256, k_len=200, head_dim=128,
             q=0x10000, k=0x20000, v=0x30000, out=0x40000,
             qs=[256 * 4 * 128, 4 * 128, 128], ks=[200 * 2 * 128, 2 * 128, 128],
             mask=None, msz=None, mst=None, bias=None, bsz=None, bst=None, ws=0x50000, wsb=1 << 30)
    a.update(over)
    return nat.load().masked_attn_fwd(
        a["dtype"], a["batch"], a["heads"], a["kv_heads"], a["q_len"], a["k_len"], a["head_dim"],
        ctypes.c_float(0.0), 0,
        ctypes.c_void_p(a["q"]), nat.i64_array(a["qs"]), ctypes.c_void_p(a["k"]), nat.i64_array(a["ks"]),
        ctypes.c_void_p(a["v"]), nat.i64_array(a["ks"]),
        ctypes.c_void_p(a["mask"]), a["msz"] and nat.i64_array(a["msz"]), a["mst"] and nat.i64_array(a["mst"]),
        ctypes.c_void_p(a["bias"]), 0, a["bsz"] and nat.i64_array(a["bsz"]), a["bst"] and nat.i64_array(a["bst"]),
        ctypes.c_void_p(a["out"]), nat.i64_array(a["qs"]), None, ctypes.c_void_p(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("over,status,msg", [
    (dict(q=0x10002), nat.SMA_ERR_INVALID_ARG, "aligned"),
    (dict(qs=[256 * 4 * 128, 4 * 128 + 1, 128]), nat.SMA_ERR_INVALID_ARG, "16 bytes"),
    (dict(heads=3), nat.SMA_ERR_INVALID_ARG, "multiple"),
    (dict(head_dim=80), nat.SMA_ERR_UNSUPPORTED, "head_dim"),
    (dict(mask=0x60000, msz=[1, 1, 256, 230], mst=[0, 0, 240, 1]), nat.SMA_ERR_INVALID_ARG, "round_up"),
    (dict(mask=0x60000, msz=[1, 1, 256, 200], mst=[0, 0, 208, 2]), nat.SMA_ERR_INVALID_ARG, "contiguous"),
    (dict(mask=0x60000, msz=[1, 3, 256, 256], mst=[0, 0, 256, 1]), nat.SMA_ERR_INVALID_ARG, "head dim"),
    (dict(mask=0x60000, msz=[2, 1, 7, 256], mst=[256, 0, 256, 1]), nat.SMA_ERR_INVALID_ARG, "query dim"),
    (dict(mask=0x60000, msz=[1, 1, 256, 256], mst=[0, 0, 1, 256]), nat.SMA_ERR_INVALID_ARG, "contiguous"),
    (dict(bias=0x60000, bsz=[3, 1, 1, 256], bst=[256, 0, 0, 1]), nat.SMA_ERR_INVALID_ARG, "batch dim"),
    (dict(wsb=16), nat.SMA_ERR_WORKSPACE, "workspace"),
])
def test_masked_attn_validation(over, status, msg):
    assert _masked_call(**over) == status
    assert msg in nat.load().sma_last_error().decode()


@pytest.mark.parametrize("kd,kst", [(256, 1), (200, 1), (1, 1), (1, 0), (1, 7)], ids=str)
@pytest.mark.parametrize("which", ["mask", "bias"])
def test_masked_attn_accepts_the_three_key_dims(kd, kst, which):
    """Key dim round_up(Lk, 128) = 256, Lk = 200, or 1 (any stride: one value
    for every key).  An accepted call reaches the workspace check, which runs
    after every shape check and before any CUDA call; a 16-byte workspace then
    stops it, so the fake pointers are never used."""
    rows = 208 if kd == 200 else kd    # 16-byte-multiple row strides
    over = {which: 0x60000, which[0] + "sz": [1, 1, 256, kd], which[0] + "st": [0, 0, rows, kst],
            "wsb": 16}
    assert _masked_call(**over) == nat.SMA_ERR_WORKSPACE
    assert "workspace" in nat.load().sma_last_error().decode()


def test_topk_validation():
    lib = nat.load()
    bad_window = lib.dynamic_topk_mask(0, ctypes.c_void_p(0x10000), nat.i64_array([1, 1, 1, 256]),
                                       nat.i64_array([256, 256, 256, 1]), 200, None, None, None, 0,
                                       ctypes.c_void_p(0x20000), None)
    assert bad_window == nat.SMA_ERR_INVALID_ARG
    bad_k = lib.dynamic_topk_mask(0, ctypes.c_void_p(0x10000), nat.i64_array([1, 1, 1, 230]),
                                  nat.i64_array([240, 240, 240, 1]), 200, None, None, None, 8,
                                  ctypes.c_void_p(0x20000), None)
    assert bad_k == nat.SMA_ERR_INVALID_ARG
    assert "round_up" in lib.sma_last_error().decode()
    one = lib.dynamic_topk_mask(0, ctypes.c_void_p(0x10000), nat.i64_array([1, 1, 1, 1]),
                                nat.i64_array([8, 8, 8, 1]), 200, None, None, None, 8,
                                ctypes.c_void_p(0x20000), None)
    assert one == nat.SMA_ERR_INVALID_ARG
    assert "one column per key" in lib.sma_last_error().decode()
    # key dims 256 and 200 pass the shape checks; the misaligned output
    # pointer, checked last before the launch, then stops the call
    for kd in (256, 200):
        st = lib.dynamic_topk_mask(0, ctypes.c_void_p(0x10000), nat.i64_array([1, 1, 2, kd]),
                                   nat.i64_array([512, 512, 256, 1]), 200, None, None, None, 8,
                                   ctypes.c_void_p(0x20001), None)
        assert st == nat.SMA_ERR_INVALID_ARG
        assert "8-byte aligned" in lib.sma_last_error().decode()
    bad_pm = lib.dynamic_topk_mask(0, ctypes.c_void_p(0x10000), nat.i64_array([2, 1, 1, 256]),
                                   nat.i64_array([256, 256, 256, 1]), 200, ctypes.c_void_p(0x30000),
                                   nat.i64_array([3, 1, 1, 200]), nat.i64_array([200, 0, 0, 1]), 8,
                                   ctypes.c_void_p(0x20000), None)
    assert bad_pm == nat.SMA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(nat, "LIB_PATH", str(tmp_path / "libsma.so"))
    monkeypatch.setattr(nat, "_lib", None)
    with pytest.raises(nat.NativeLibraryMissing):
        nat.load()


def test_sparse_workspace_and_validation_on_host():
    lib = nat.load()
    n = ctypes.c_size_t()
    ms = nat.i64_array([2, 8, 1, 16384])
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, ms, 0, None, 2048,
                                              ctypes.byref(n)) == 0
    # compacted K and V: 2 x (batch 2, 2048 keys, 8 kv heads, 128) bf16, plus index and tile lists
    kv = 2 * 2 * 2048 * 8 * 128 * 2
    assert kv < n.value < kv + (1 << 20)
    small = n.value
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, ms, 0, None, 0,
                                              ctypes.byref(n)) == 0
    assert n.value > 7 * small            # unbounded: capacity k_len
    bs = nat.i64_array([1, 32, 4096, 16384])
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, ms, 2, bs, 2048,
                                              ctypes.byref(n)) == 0
    assert n.value >= small + 2 * 32 * 4096 * 2048 * 4     # compacted fp32 bias
    per_query = nat.i64_array([1, 1, 4096, 16384])
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, per_query, 0, None, 0,
                                              ctypes.byref(n)) == nat.SMA_ERR_UNSUPPORTED
    assert "broadcast over queries" in lib.sma_last_error().decode()
    per_qhead = nat.i64_array([1, 32, 1, 16384])
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, per_qhead, 0, None, 0,
                                              ctypes.byref(n)) == nat.SMA_ERR_UNSUPPORTED
    mha = nat.i64_array([1, 8, 1, 16384])
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 8, 8, 4096, 16384, 128, mha, 0, None, 0,
                                              ctypes.byref(n)) == 0
    assert lib.sparse_attn_fwd_workspace_size(0, 2, 32, 8, 4096, 16384, 128, None, 0, None, 0,
                                              ctypes.byref(n)) == nat.SMA_ERR_INVALID_ARG


def test_sparse_attn_needs_a_mask():
    qs = [256 * 4 * 128, 4 * 128, 128]
    ks = [200 * 2 * 128, 2 * 128, 128]
    st = nat.load().sparse_attn_fwd(
        0, 2, 4, 2, 256, 200, 128, ctypes.c_float(0.0), 0,
        ctypes.c_void_p(0x10000), nat.i64_array(qs), ctypes.c_void_p(0x20000), nat.i64_array(ks),
        ctypes.c_void_p(0x30000), nat.i64_array(ks), ctypes.c_void_p(0), None, None,
        ctypes.c_void_p(0), 0, None, None, 0,
        ctypes.c_void_p(0x40000), nat.i64_array(qs), None, ctypes.c_void_p(0x50000), 1 << 30, None)
    assert st == nat.SMA_ERR_INVALID_ARG
    assert "needs a mask" in nat.load().sma_last_error().decode()


def test_backward_workspace_and_validation_on_host():
    lib = nat.load()
    n = ctypes.c_size_t()
    d = nat.DfaMaskDesc(1, 2048, 16, 32768, 1, 0, 0)
    assert lib.dfa_attn_bwd_workspace_size(ctypes.byref(d), 32, 8, 128, ctypes.byref(n)) == 0
    # the fp32 dQ accumulator alone is B * Lq * H * d * 4 bytes
    assert n.value >= 32768 * 32 * 128 * 4
    ms = nat.i64_array([1, 1, 8192, 8064])
    assert lib.masked_attn_bwd_workspace_size(4, 16, 4, 8192, 8000, 128, ms, ctypes.byref(n)) == 0
    assert n.value >= 4 * 8192 * 16 * 128 * 4
    assert lib.masked_attn_bwd_workspace_size(4, 16, 4, 8192, 8000, 96, ms, ctypes.byref(n)) == nat.SMA_ERR_UNSUPPORTED

    qs = [256 * 4 * 128, 4 * 128, 128]
    ks = [200 * 2 * 128, 2 * 128, 128]

    def call(dtype=0, lse=0x70000, dbias=0):
        return lib.masked_attn_bwd(
            dtype, 2, 4, 2, 256, 200, 128, ctypes.c_float(0.0), 0,
            ctypes.c_void_p(0x10000), nat.i64_array(qs), ctypes.c_void_p(0x20000), nat.i64_array(ks),
            ctypes.c_void_p(0x30000), nat.i64_array(ks), ctypes.c_void_p(0), None, None,
            ctypes.c_void_p(0), 0, None, None,
            ctypes.c_void_p(0x40000), nat.i64_array(qs), ctypes.c_void_p(lse),
            ctypes.c_void_p(0x50000), nat.i64_array(qs),
            ctypes.c_void_p(0x60000), nat.i64_array(qs), ctypes.c_void_p(0x80000), nat.i64_array(ks),
            ctypes.c_void_p(0x90000), nat.i64_array(ks), ctypes.c_void_p(dbias),
            ctypes.c_void_p(0xa0000), 1 << 30, None)

    # packed batches: an unknown dtype code is rejected before anything runs
    s2 = nat.i64_array([1024, 128])
    assert lib.varlen_attn_bwd(9, 2, 8, 2, 128, 100, 100, 64, 64, ctypes.c_float(0.0), 0,
                               ctypes.c_void_p(0x10000), ctypes.c_void_p(0x11000),
                               *([ctypes.c_void_p(0x20000), s2] * 4), ctypes.c_void_p(0x70000),
                               *([ctypes.c_void_p(0x20000), s2] * 4), ctypes.c_void_p(0xa0000),
                               1 << 30, None) == nat.SMA_ERR_INVALID_ARG
    assert "unknown dtype" in lib.sma_last_error().decode()
    # fp32 packed gradients are accepted up to the workspace check (too small here)
    assert lib.varlen_attn_bwd(2, 2, 8, 2, 128, 100, 100, 64, 64, ctypes.c_float(0.0), 0,
                               ctypes.c_void_p(0x10000), ctypes.c_void_p(0x11000),
                               *([ctypes.c_void_p(0x20000), s2] * 4), ctypes.c_void_p(0x70000),
                               *([ctypes.c_void_p(0x20000), s2] * 4), ctypes.c_void_p(0xa0000),
                               16, None) == nat.SMA_ERR_WORKSPACE
    assert call(lse=0) == nat.SMA_ERR_INVALID_ARG
    assert "lse" in lib.sma_last_error().decode()
    assert call(dbias=0xb0000) == nat.SMA_ERR_INVALID_ARG  # no bias to take the gradient of
    assert "dbias needs the bias" in lib.sma_last_error().decode()


def test_varlen_validation_on_host():
    lib = nat.load()
    n = ctypes.c_size_t()
    assert lib.varlen_attn_fwd_workspace_size(4, 1000, 2000, ctypes.byref(n)) == 0
    nf = n.value
    assert nf >= 2 * 4 * 8 * 16 * 4          # full and partial index arrays
    # backward: the same lists plus their transpose, rowsum(dO * O) and the
    # fp32 dQ accumulator over the packed rows
    assert lib.varlen_attn_bwd_workspace_size(4, 8, 3000, 1000, 2000, 128, ctypes.byref(n)) == 0
    assert n.value >= nf + 3000 * 8 * 4 + 3000 * 8 * 128 * 4
    assert lib.varlen_attn_bwd_workspace_size(0, 8, 3000, 1000, 2000, 128, ctypes.byref(n)) == nat.SMA_ERR_INVALID_ARG
    st = lib.varlen_attn_fwd(2, 2, 4, 2, 128, 100, 100, 60, 60, ctypes.c_float(0.0), 0,
                             ctypes.c_void_p(0x100), ctypes.c_void_p(0x200),
                             ctypes.c_void_p(0x10000), nat.i64_array([512, 128]),
                             ctypes.c_void_p(0x20000), nat.i64_array([256, 128]),
                             ctypes.c_void_p(0x30000), nat.i64_array([256, 128]),
                             ctypes.c_void_p(0x40000), nat.i64_array([512, 128]), None,
                             ctypes.c_void_p(0x50000), 16, None)
    assert st == nat.SMA_ERR_WORKSPACE   # fp32 is accepted; the 16-byte workspace is not
    st = lib.varlen_attn_fwd(0, 2, 4, 2, 128, 100, 100, 60, 60, ctypes.c_float(0.0), 0,
                             ctypes.c_void_p(0), ctypes.c_void_p(0x200),
                             ctypes.c_void_p(0x10000), nat.i64_array([512, 128]),
                             ctypes.c_void_p(0x20000), nat.i64_array([256, 128]),
                             ctypes.c_void_p(0x30000), nat.i64_array([256, 128]),
                             ctypes.c_void_p(0x40000), nat.i64_array([512, 128]), None,
                             ctypes.c_void_p(0x50000), 1 << 20, None)
    assert st == nat.SMA_ERR_INVALID_ARG and "cu_seqlens" in lib.sma_last_error().decode()


def test_varlen_backward_validation_on_host():
    """varlen_attn_bwd rejects a short workspace, a missing lse and missing
    offsets before anything runs (fake, never dereferenced pointers)."""
    lib = nat.load()
    qs, ks = nat.i64_array([512, 128]), nat.i64_array([256, 128])

    def call(ws_bytes=1 << 30, lse=0x60000, cu=0x100):
        return lib.varlen_attn_bwd(
            0, 2, 4, 2, 128, 100, 100, 60, 60, ctypes.c_float(0.0), 1,
            ctypes.c_void_p(cu), ctypes.c_void_p(0x200),
            ctypes.c_void_p(0x10000), qs, ctypes.c_void_p(0x20000), ks, ctypes.c_void_p(0x30000), ks,
            ctypes.c_void_p(0x40000), qs, ctypes.c_void_p(lse), ctypes.c_void_p(0x50000), qs,
            ctypes.c_void_p(0x70000), qs, ctypes.c_void_p(0x80000), ks, ctypes.c_void_p(0x90000), ks,
            ctypes.c_void_p(0xa0000), ws_bytes, None)

    assert call(ws_bytes=256) == nat.SMA_ERR_WORKSPACE
    assert call(lse=0) == nat.SMA_ERR_INVALID_ARG and "lse" in lib.sma_last_error().decode()
    assert call(cu=0) == nat.SMA_ERR_INVALID_ARG and "cu_seqlens" in lib.sma_last_error().decode()


def test_sparse_workspace_includes_key_range_segments_for_short_queries():
    """16 queries over compacted keys: the group's 4 heads share a tile, so
    2 units on a 148-SM part, and the index-gather workspace also holds the
    key-range split's partial results (32 segments, the cap)."""
    lib = nat.load()
    n_short, n_long = ctypes.c_size_t(), ctypes.c_size_t()
    ms = nat.i64_array([1, 2, 1, 20096])
    assert lib.sparse_attn_fwd_workspace_size(0, 1, 8, 2, 16, 20000, 128, ms, 0, None, 0,
                                              ctypes.byref(n_short)) == 0
    assert lib.sparse_attn_fwd_workspace_size(0, 1, 8, 2, 4096, 20000, 128, ms, 0, None, 0,
                                              ctypes.byref(n_long)) == 0
    segments = 32                       # 148 // 2 = 74 per unit, at most 157 // 4, at most 32
    rows = 1 * 8 * 16
    assert n_short.value >= segments * rows * (128 * 4 + 8)


def test_deterministic_dbias_workspace_query():
    """Partial rows per (batch, head): query groups of 64 (either head dim)
    for a query-broadcast bias, every query for a bias with a query dim or
    fp32 operands; nothing when each dbias element has one writer."""
    lib = nat.load()
    n = ctypes.c_size_t()
    q = lambda dt, hd, shape: lib.masked_attn_bwd_dbias_workspace_size(  # noqa: E731
        dt, 4, 16, 8, 1000, hd, nat.i64_array(shape), ctypes.byref(n))
    assert q(nat.SMA_BF16, 128, [4, 8, 1, 1024]) == 0 and n.value == 4 * 16 * 16 * 1024 * 4
    assert q(nat.SMA_BF16, 64, [1, 1, 1, 1000]) == 0 and n.value == 4 * 16 * 16 * 1000 * 4
    assert q(nat.SMA_FP32, 64, [1, 1, 1, 1000]) == 0 and n.value == 4 * 16 * 1000 * 1000 * 4
    assert q(nat.SMA_BF16, 128, [1, 8, 1000, 1024]) == 0 and n.value == 4 * 16 * 1000 * 1024 * 4
    assert q(nat.SMA_BF16, 128, [4, 16, 1000, 1024]) == 0 and n.value == 0
    assert q(nat.SMA_BF16, 96, [4, 8, 1, 1024]) == nat.SMA_ERR_UNSUPPORTED
    assert lib.masked_attn_bwd_dbias_workspace_size(nat.SMA_BF16, 4, 16, 8, 1000, 128, None,
                                                    ctypes.byref(n)) == nat.SMA_ERR_INVALID_ARG


def _decode_splits(batch, heads, kv_heads, k_len, sms=148):
    """The split-KV cost model restated: waves of CTAs over two per SM times
    the 64-key steps of a split plus two of fixed cost; splits keep at least
    512 keys, at most 64; the first minimum wins."""
    group = heads // kv_heads
    base = batch * kv_heads * ((group + 7) // 8)
    steps = -(-k_len // 64)
    best, best_s = None, 1
    for sp in range(1, min(64, max(1, -(-k_len // 512))) + 1):
        cost = -(-base * sp // (2 * sms)) * (-(-steps // sp) + 2)
        if best is None or cost < best:
            best, best_s = cost, sp
    return best_s


def test_decode_workspace_follows_the_split_cost_model():
    """Single-query calls: the workspace holds fp32 O and (max, sum) for each
    (batch, head, split); the split count fills the CTA slots (9 splits of
    16384 keys for 8 x 8 KV heads: 576 CTAs, two waves of 296; 37 for one
    row of 8 KV heads over 32768 keys).  No GPU is present here, so the
    library assumes a 148-SM part."""
    lib = nat.load()
    n = ctypes.c_size_t()
    a256 = lambda x: -(-x // 256) * 256  # noqa: E731
    for (b, h, kvh, lk, want) in [(8, 32, 8, 16384, 9), (1, 32, 8, 32768, 37), (1, 8, 8, 1000, 2)]:
        sp = _decode_splits(b, h, kvh, lk)
        assert sp == want
        assert lib.masked_attn_fwd_workspace_size(b, h, kvh, 1, lk, 128, None, ctypes.byref(n)) == 0
        part_ml = a256(b * h * sp * 128 * 4)
        assert n.value == a256(part_ml + b * h * sp * 2 * 4)
