"""ctypes loader for libsma.so, the C-ABI library declared in include/sma.h.

The library is built in-tree (``python -m
structured_mask_attention_analytic_b200.csrc.build``).  There is no fallback:
if the shared object is missing, importing the ops raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsma.so")

c_i32 = ctypes.c_int32
c_i64p = ctypes.POINTER(ctypes.c_int64)
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t
c_sizep = ctypes.POINTER(ctypes.c_size_t)
c_i32p = ctypes.POINTER(ctypes.c_int32)

SMA_OK = 0
SMA_ERR_INVALID_ARG = 1
SMA_ERR_UNSUPPORTED = 2
SMA_ERR_CUDA = 3
SMA_ERR_WORKSPACE = 4
SMA_ERR_DEVICE_TIMEOUT = 5
SMA_ERR_DEVICE_INPUT = 6

SMA_BF16, SMA_FP16, SMA_FP32 = 0, 1, 2
SMA_TILE = 128
SMA_TILE_EMPTY, SMA_TILE_PARTIAL, SMA_TILE_FULL = 0, 1, 2


class DfaMaskDesc(ctypes.Structure):
    _fields_ = [("batch", c_i32), ("n_blocks", c_i32), ("block_size", c_i32), ("ctx_len", c_i32),
                ("is_causal", c_i32), ("layer_type", c_i32), ("sliding_window", c_i32)]


class DfaBlockMapPtrs(ctypes.Structure):
    _fields_ = [("num_full", c_vp), ("full_idx", c_vp), ("num_part", c_vp), ("part_idx", c_vp)]


class NativeLibraryMissing(RuntimeError):
    pass


class SmaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libsma status {status}: {message}")
        self.status = status


_SIGNATURES = {
    "sma_last_error": (ctypes.c_char_p, []),
    "sma_abi_version": (c_i32, []),
    "sma_device_status": (c_i32, [c_vp, c_i32p]),
    "sma_selftest_wait_timeout": (c_i32, [ctypes.c_int64, c_vp, c_vp]),
    "dfa_block_map_dims": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_i32p, c_i32p]),
    "dfa_block_map": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "dfa_attn_fwd_workspace_size": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_i32, c_i32, c_i32, c_sizep]),
    "dfa_attn_fwd": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_vp, c_i32, c_i32, c_i32, c_i32, ctypes.c_float,
                             c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp,
                             ctypes.POINTER(DfaBlockMapPtrs), c_vp, c_size, c_vp]),
    "dfa_attn_fwd_noalloc": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_vp, c_i32, c_i32, c_i32, c_i32,
                                     ctypes.c_float, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp,
                                     c_i64p, c_vp, c_vp]),
    "mask_tile_summary": (c_i32, [c_vp, c_i64p, c_i64p, c_i32, c_vp, c_vp]),
    "masked_attn_fwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64p, c_sizep]),
    "masked_attn_fwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float, c_i32,
                                c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_i64p, c_i64p,
                                c_vp, c_i32, c_i64p, c_i64p,
                                c_vp, c_i64p, c_vp, c_vp, c_size, c_vp]),
    "dynamic_topk_mask": (c_i32, [c_i32, c_vp, c_i64p, c_i64p, c_i32, c_vp, c_i64p, c_i64p, c_i32, c_vp,
                                  c_vp]),
    "dfa_attn_bwd_workspace_size": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_i32, c_i32, c_i32, c_sizep]),
    "dfa_attn_bwd": (c_i32, [ctypes.POINTER(DfaMaskDesc), c_vp, c_i32, c_i32, c_i32, c_i32, ctypes.c_float,
                             c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                             c_vp, c_i64p, c_vp, c_vp, c_i64p,
                             c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                             c_vp, c_size, c_vp]),
    "masked_attn_bwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64p, c_sizep]),
    "masked_attn_bwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float, c_i32,
                                c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_i64p, c_i64p,
                                c_vp, c_i32, c_i64p, c_i64p,
                                c_vp, c_i64p, c_vp, c_vp, c_i64p,
                                c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_vp, c_size, c_vp]),
    "masked_attn_bwd_dbias_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64p,
                                                     c_sizep]),
    "masked_attn_bwd_deterministic": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float,
                                              c_i32,
                                              c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                              c_vp, c_i64p, c_i64p,
                                              c_vp, c_i32, c_i64p, c_i64p,
                                              c_vp, c_i64p, c_vp, c_vp, c_i64p,
                                              c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                              c_vp, c_vp, c_size, c_vp, c_size, c_vp]),
    "varlen_attn_fwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_sizep]),
    "varlen_attn_fwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float,
                                c_i32, c_vp, c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_vp, c_size, c_vp]),
    "varlen_attn_bwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_sizep]),
    "varlen_attn_bwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float,
                                c_i32, c_vp, c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_size, c_vp]),
    "varlen_masked_attn_fwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64p,
                                                      c_sizep]),
    "varlen_masked_attn_fwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                       ctypes.c_float, c_i32, c_vp, c_vp, c_vp, c_i64p, c_vp, c_i64p,
                                       c_vp, c_i64p, c_vp, c_i64p, c_i64p, c_vp, c_i32, c_i64p, c_i64p,
                                       c_vp, c_i64p, c_vp, c_vp, c_size, c_vp]),
    "varlen_masked_attn_bwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                                      c_i64p, c_sizep]),
    "varlen_masked_attn_bwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                       ctypes.c_float, c_i32, c_vp, c_vp, c_vp, c_i64p, c_vp, c_i64p,
                                       c_vp, c_i64p, c_vp, c_i64p, c_i64p, c_vp, c_i32, c_i64p, c_i64p,
                                       c_vp, c_i64p, c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                       c_vp, c_i64p, c_vp, c_vp, c_size, c_vp]),
    "varlen_pad": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp]),
    "varlen_unpad": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_i64p, c_vp, c_i64p, c_vp]),
    "sparse_attn_fwd_workspace_size": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i64p,
                                               c_i32, c_i64p, c_i32, c_sizep]),
    "sparse_attn_fwd": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.c_float, c_i32,
                                c_vp, c_i64p, c_vp, c_i64p, c_vp, c_i64p,
                                c_vp, c_i64p, c_i64p,
                                c_vp, c_i32, c_i64p, c_i64p, c_i32,
                                c_vp, c_i64p, c_vp, c_vp, c_size, c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """The loaded library (raises NativeLibraryMissing if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise NativeLibraryMissing(
                f"{LIB_PATH} is missing; build it with "
                "`python -m structured_mask_attention_analytic_b200.csrc.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int) -> None:
    if status != SMA_OK:
        msg = load().sma_last_error()
        raise SmaError(status, msg.decode() if msg else "")


def i64_array(values) -> ctypes.Array:
    return (ctypes.c_int64 * len(values))(*[int(v) for v in values])
