"""Structured-mask attention forward and backward for NVIDIA B200 (sm_100a).

Thin Python binding over libsma (C ABI in include/sma.h): DFlash draft-training
masks computed analytically from block anchors, broadcastable 4D mask/bias
attention with the grouped-head decode path, the dynamic top-k keep mask, and
index-gather attention over the keys such a mask keeps.
"""
from ._native import NativeLibraryMissing, SmaError  # noqa: F401
from .ops import (  # noqa: F401
    LAYER_FULL,
    LAYER_SLIDING,
    device_status,
    dfa_attn_bwd,
    dfa_attn_bwd_workspace_size,
    dfa_attn_fwd,
    dfa_attn_fwd_noalloc,
    dfa_attn_fwd_workspace_size,
    dfa_block_map,
    dfa_block_map_dims,
    dflash_spec_generate_fwd,
    dynamic_topk_mask,
    mask_tile_summary,
    masked_attn_bwd,
    masked_attn_bwd_workspace_size,
    masked_attn_bwd_dbias_workspace_size,
    masked_attn_fwd,
    masked_attn_fwd_workspace_size,
    round_up_k,
    selftest_wait_timeout,
    sparse_attn_fwd,
    sparse_attn_fwd_workspace_size,
    varlen_attn_bwd,
    varlen_attn_fwd,
    varlen_pad,
    varlen_unpad,
)
