"""Python binding of libsma: the same entry points as include/sma.h, taking
torch CUDA tensors.

Only argument marshalling happens here (pointers, strides, the current
stream, workspace buffers from the torch allocator); every step of the
computation runs in the library's CUDA kernels.  Nothing falls back to
PyTorch or the CPU: a missing library or a rejected argument raises.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native as nat

_DTYPE = {torch.bfloat16: nat.SMA_BF16, torch.float16: nat.SMA_FP16, torch.float32: nat.SMA_FP32}

LAYER_FULL = 0
LAYER_SLIDING = 1


def _lib():
    return nat.load()


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libsma ops take CUDA tensors")


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def round_up_k(k_len: int) -> int:
    """Key dim of a mask/bias under the broadcast contract: round_up(k_len, 128)."""
    return (k_len + 127) // 128 * 128


def _is_causal_code(is_causal) -> int:
    if is_causal is None:
        return -1
    return 1 if int(is_causal) == 1 else (0 if int(is_causal) == 0 else -1)


def _desc(batch, n_blocks, block_size, ctx_len, is_causal, layer_type, sliding_window):
    return nat.DfaMaskDesc(int(batch), int(n_blocks), int(block_size), int(ctx_len),
                           _is_causal_code(is_causal), int(layer_type), int(sliding_window))


def dfa_block_map_dims(batch, n_blocks, block_size, ctx_len, is_causal=None, layer_type=LAYER_FULL,
                       sliding_window=0):
    d = _desc(batch, n_blocks, block_size, ctx_len, is_causal, layer_type, sliding_window)
    qt, kt = ctypes.c_int32(), ctypes.c_int32()
    nat.check(_lib().dfa_block_map_dims(ctypes.byref(d), ctypes.byref(qt), ctypes.byref(kt)))
    return qt.value, kt.value


def dfa_block_map(anchors: torch.Tensor, ctx_len: int, block_size: int, is_causal=None,
                  layer_type: int = LAYER_FULL, sliding_window: int = 0):
    """DFlash block map of ``anchors`` (int32 [B, N], CUDA).

    Returns ``(num_full [B,QT], full_idx [B,QT,KT], num_part [B,QT],
    part_idx [B,QT,KT])`` int32 tensors."""
    _require_cuda(anchors)
    if anchors.dtype != torch.int32 or anchors.dim() != 2:
        raise ValueError("anchors must be int32 [batch, n_blocks]")
    anchors = anchors.contiguous()
    b, n = anchors.shape
    d = _desc(b, n, block_size, ctx_len, is_causal, layer_type, sliding_window)
    qt, kt = dfa_block_map_dims(b, n, block_size, ctx_len, is_causal, layer_type, sliding_window)
    dev = anchors.device
    nf = torch.empty((b, qt), dtype=torch.int32, device=dev)
    npart = torch.empty((b, qt), dtype=torch.int32, device=dev)
    fi = torch.empty((b, qt, kt), dtype=torch.int32, device=dev)
    pi = torch.empty((b, qt, kt), dtype=torch.int32, device=dev)
    nat.check(_lib().dfa_block_map(ctypes.byref(d), _ptr(anchors), _ptr(nf), _ptr(fi), _ptr(npart),
                                   _ptr(pi), _stream(anchors)))
    return nf, fi, npart, pi


def dfa_attn_fwd_workspace_size(batch, n_blocks, block_size, ctx_len, heads, kv_heads, head_dim,
                                is_causal=None, layer_type=LAYER_FULL, sliding_window=0) -> int:
    d = _desc(batch, n_blocks, block_size, ctx_len, is_causal, layer_type, sliding_window)
    n = ctypes.c_size_t()
    nat.check(_lib().dfa_attn_fwd_workspace_size(ctypes.byref(d), heads, kv_heads, head_dim,
                                                 ctypes.byref(n)))
    return n.value


def _strides3(t: torch.Tensor):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("q/k/v/out must be 4D [batch, len, heads, head_dim] with head_dim contiguous")
    return nat.i64_array(t.stride()[:3])


def dfa_attn_fwd(q, k, v, anchors, ctx_len: int, block_size: int, is_causal=None,
                 layer_type: int = LAYER_FULL, sliding_window: int = 0, scale=None, out=None,
                 return_lse: bool = True, workspace=None, block_map=None):
    """Attention forward under the DFlash draft-training mask.

    q ``[B, N*block_size, H, d]``, k/v ``[B, ctx_len + N*block_size, KVH, d]``,
    anchors int32 ``[B, N]``.  ``block_map`` optionally passes the 4-tuple
    returned by ``dfa_block_map`` for the same mask (the map is then not
    recomputed).  Returns ``(out, lse)`` (lse None unless requested)."""
    _require_cuda(q, k, v, anchors)
    b, nq, h, dh = q.shape
    kvh = k.shape[2]
    if anchors.dtype != torch.int32 or anchors.dim() != 2 or anchors.shape[0] != b:
        raise ValueError("anchors must be int32 [batch, n_blocks]")
    anchors = anchors.contiguous()
    n = anchors.shape[1]
    if nq != n * block_size or k.shape[1] != ctx_len + nq or v.shape != k.shape:
        raise ValueError("q/k/v lengths do not match ctx_len, n_blocks and block_size")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    d = _desc(b, n, block_size, ctx_len, is_causal, layer_type, sliding_window)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((b, h, nq), dtype=torch.float32, device=q.device) if return_lse else None
    map_ptrs = None
    if block_map is not None:
        nf, fi, npart, pi = block_map
        map_ptrs = ctypes.byref(nat.DfaBlockMapPtrs(nf.data_ptr(), fi.data_ptr(), npart.data_ptr(),
                                                    pi.data_ptr()))
        ws_ptr, ws_len = ctypes.c_void_p(0), 0
    else:
        ws_bytes = dfa_attn_fwd_workspace_size(b, n, block_size, ctx_len, h, kvh, dh, is_causal,
                                               layer_type, sliding_window)
        if workspace is None:
            workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
        ws_ptr, ws_len = _ptr(workspace), workspace.numel()
    nat.check(_lib().dfa_attn_fwd(
        ctypes.byref(d), _ptr(anchors), _dtype_code(q), h, kvh, dh,
        ctypes.c_float(0.0 if scale is None else float(scale)),
        _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v), _ptr(out), _strides3(out),
        _ptr(lse), map_ptrs, ws_ptr, ws_len, _stream(q)))
    return out, lse


def dflash_spec_generate_fwd(q, k, v, ctx_lens, ctx_len: int, is_causal=None, layer_type: int = LAYER_FULL,
                             sliding_window: int = 0, scale=None, out=None, return_lse: bool = True,
                             workspace=None):
    """Attention of DFlash inference (``spec_generate``): one draft block of
    ``q.shape[1]`` queries after each row's context.

    q ``[B, block_size, H, d]``; k/v ``[B, ctx_len + block_size, KVH, d]`` with
    row b's context in keys ``[0, ctx_lens[b])`` (the rest of the first
    ``ctx_len`` keys is padding) and the block's own keys last; ``ctx_lens``
    int32 ``[B]`` on the device.  This is ``dfa_attn_fwd`` with one block
    whose anchor is the row's context length (the same C entry point)."""
    _require_cuda(ctx_lens)
    if ctx_lens.dtype != torch.int32 or ctx_lens.dim() != 1 or ctx_lens.shape[0] != q.shape[0]:
        raise ValueError("ctx_lens must be int32 [batch]")
    anchors = ctx_lens.contiguous().view(-1, 1)
    return dfa_attn_fwd(q, k, v, anchors, ctx_len, q.shape[1], is_causal, layer_type, sliding_window,
                        scale=scale, out=out, return_lse=return_lse, workspace=workspace)


def dfa_attn_bwd_workspace_size(batch, n_blocks, block_size, ctx_len, heads, kv_heads, head_dim,
                                is_causal=None, layer_type=LAYER_FULL, sliding_window=0) -> int:
    d = _desc(batch, n_blocks, block_size, ctx_len, is_causal, layer_type, sliding_window)
    n = ctypes.c_size_t()
    nat.check(_lib().dfa_attn_bwd_workspace_size(ctypes.byref(d), heads, kv_heads, head_dim,
                                                 ctypes.byref(n)))
    return n.value


def _grad_outputs(q, k, dq, dk, dv):
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    return dq, dk, dv


def dfa_attn_bwd(q, k, v, out, lse, dout, anchors, ctx_len: int, block_size: int, is_causal=None,
                 layer_type: int = LAYER_FULL, sliding_window: int = 0, scale=None, dq=None, dk=None,
                 dv=None, workspace=None):
    """Gradients of ``dfa_attn_fwd``: ``out`` and ``lse`` are that call's
    results for the same arguments, ``dout`` the upstream gradient.
    Returns ``(dq, dk, dv)``."""
    _require_cuda(q, k, v, out, lse, dout, anchors)
    b, nq, h, dh = q.shape
    kvh = k.shape[2]
    if anchors.dtype != torch.int32 or anchors.dim() != 2 or anchors.shape[0] != b:
        raise ValueError("anchors must be int32 [batch, n_blocks]")
    anchors = anchors.contiguous()
    n = anchors.shape[1]
    if lse.dtype != torch.float32 or tuple(lse.shape) != (b, h, nq) or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous float32 [batch, heads, q_len]")
    d = _desc(b, n, block_size, ctx_len, is_causal, layer_type, sliding_window)
    dq, dk, dv = _grad_outputs(q, k, dq, dk, dv)
    ws_bytes = dfa_attn_bwd_workspace_size(b, n, block_size, ctx_len, h, kvh, dh, is_causal, layer_type,
                                           sliding_window)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    nat.check(_lib().dfa_attn_bwd(
        ctypes.byref(d), _ptr(anchors), _dtype_code(q), h, kvh, dh,
        ctypes.c_float(0.0 if scale is None else float(scale)),
        _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v),
        _ptr(out), _strides3(out), _ptr(lse), _ptr(dout), _strides3(dout),
        _ptr(dq), _strides3(dq), _ptr(dk), _strides3(dk), _ptr(dv), _strides3(dv),
        _ptr(workspace), workspace.numel(), _stream(q)))
    return dq, dk, dv


def dfa_attn_fwd_noalloc(q, k, v, anchors, ctx_len: int, block_size: int, is_causal=None,
                         layer_type: int = LAYER_FULL, sliding_window: int = 0, scale=None, out=None,
                         return_lse: bool = True):
    """dfa_attn_fwd without a workspace, for callers that cannot allocate
    device scratch: the block map goes to a fixed 4 MiB array inside libsma
    (larger problems raise).  Calls share that array, so calls that may run
    concurrently on the GPU race; keep them on one stream."""
    _require_cuda(q, k, v, anchors)
    b, nq, h, dh = q.shape
    kvh = k.shape[2]
    if anchors.dtype != torch.int32 or anchors.dim() != 2 or anchors.shape[0] != b:
        raise ValueError("anchors must be int32 [batch, n_blocks]")
    anchors = anchors.contiguous()
    d = _desc(b, anchors.shape[1], block_size, ctx_len, is_causal, layer_type, sliding_window)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((b, h, nq), dtype=torch.float32, device=q.device) if return_lse else None
    nat.check(_lib().dfa_attn_fwd_noalloc(
        ctypes.byref(d), _ptr(anchors), _dtype_code(q), h, kvh, dh,
        ctypes.c_float(0.0 if scale is None else float(scale)),
        _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v), _ptr(out), _strides3(out),
        _ptr(lse), _stream(q)))
    return out, lse


def _aux_args(t, k_len):
    if t is None:
        return ctypes.c_void_p(0), None, None
    if t.dim() != 4:
        raise ValueError("mask/bias must be 4D ({B|1}, {H|KVH|1}, {Lq|1}, {round_up(Lk,128)|Lk|1})")
    return _ptr(t), nat.i64_array(t.shape), nat.i64_array(t.stride())


def mask_tile_summary(mask: torch.Tensor, k_len: int) -> torch.Tensor:
    """uint8 codes ``[m0, m1, ceil(m2/128), ceil(k_len/128)]`` of a 4D bool mask."""
    _require_cuda(mask)
    if mask.dtype not in (torch.bool, torch.uint8):
        raise ValueError("mask must be bool")
    m0, m1, m2, _ = mask.shape
    codes = torch.empty((m0, m1, (m2 + 127) // 128, (k_len + 127) // 128), dtype=torch.uint8,
                        device=mask.device)
    p, sz, st = _aux_args(mask, k_len)
    nat.check(_lib().mask_tile_summary(p, sz, st, int(k_len), _ptr(codes), _stream(mask)))
    return codes


def masked_attn_fwd_workspace_size(batch, heads, kv_heads, q_len, k_len, head_dim, mask_shape=None) -> int:
    n = ctypes.c_size_t()
    ms = nat.i64_array(mask_shape) if mask_shape is not None else None
    nat.check(_lib().masked_attn_fwd_workspace_size(batch, heads, kv_heads, q_len, k_len, head_dim, ms,
                                                    ctypes.byref(n)))
    return n.value


def masked_attn_fwd(q, k, v, mask=None, bias=None, is_causal: bool = False, scale=None, out=None,
                    return_lse: bool = True, workspace=None):
    """Attention forward with a broadcastable 4D bool mask and/or additive bias.

    mask / bias follow ``({B|1}, {H|KVH|1}, {Lq|1}, {round_up(Lk, 128)|Lk|1})``
    with a contiguous last dim; broadcast dims may have any stride (they are
    read with stride 0), and a key dim of 1 is one value for every key.  No
    padding or expansion is made: the kernels read each form in place.
    ``q_len == 1`` takes the grouped-head decode path.  Returns ``(out, lse)``."""
    _require_cuda(q, k, v, mask, bias)
    b, lq, h, dh = q.shape
    lk, kvh = k.shape[1], k.shape[2]
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    if mask is not None and mask.dtype not in (torch.bool, torch.uint8):
        raise ValueError("mask must be bool")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((b, h, lq), dtype=torch.float32, device=q.device) if return_lse else None
    ws_bytes = masked_attn_fwd_workspace_size(b, h, kvh, lq, lk, dh,
                                              tuple(mask.shape) if mask is not None else None)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    mp, msz, mst = _aux_args(mask, lk)
    bp, bsz, bst = _aux_args(bias, lk)
    nat.check(_lib().masked_attn_fwd(
        _dtype_code(q), b, h, kvh, lq, lk, dh, ctypes.c_float(0.0 if scale is None else float(scale)),
        1 if is_causal else 0,
        _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v),
        mp, msz, mst,
        bp, _dtype_code(bias) if bias is not None else 0, bsz, bst,
        _ptr(out), _strides3(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(q)))
    return out, lse


def masked_attn_bwd_workspace_size(batch, heads, kv_heads, q_len, k_len, head_dim, mask_shape=None) -> int:
    n = ctypes.c_size_t()
    ms = nat.i64_array(mask_shape) if mask_shape is not None else None
    nat.check(_lib().masked_attn_bwd_workspace_size(batch, heads, kv_heads, q_len, k_len, head_dim, ms,
                                                    ctypes.byref(n)))
    return n.value


def masked_attn_bwd_dbias_workspace_size(dtype, batch, heads, kv_heads, q_len, head_dim, bias_shape) -> int:
    n = ctypes.c_size_t()
    nat.check(_lib().masked_attn_bwd_dbias_workspace_size(
        _DTYPE[dtype], batch, heads, kv_heads, q_len, head_dim, nat.i64_array(bias_shape), ctypes.byref(n)))
    return n.value


def masked_attn_bwd(q, k, v, out, lse, dout, mask=None, bias=None, is_causal: bool = False, scale=None,
                    dq=None, dk=None, dv=None, workspace=None, return_dbias: bool = False, dbias=None,
                    deterministic: bool = False, dbias_workspace=None):
    """Gradients of ``masked_attn_fwd`` (same mask / bias / causal / scale):
    ``out`` and ``lse`` are that call's results, ``dout`` the upstream
    gradient.  Returns ``(dq, dk, dv)``, or ``(dq, dk, dv, dbias)`` with
    ``return_dbias`` (or a ``dbias`` buffer): float32 at the bias's shape,
    reduced over the dims the bias broadcasts along (a key dim of 1 too).
    ``deterministic``: dbias through ``masked_attn_bwd_deterministic`` (the
    same bits on every call), with a partial-sum buffer of
    ``masked_attn_bwd_dbias_workspace_size`` bytes (allocated if not given)."""
    _require_cuda(q, k, v, out, lse, dout, mask, bias)
    b, lq, h, dh = q.shape
    lk, kvh = k.shape[1], k.shape[2]
    if lse.dtype != torch.float32 or tuple(lse.shape) != (b, h, lq) or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous float32 [batch, heads, q_len]")
    dq, dk, dv = _grad_outputs(q, k, dq, dk, dv)
    ws_bytes = masked_attn_bwd_workspace_size(b, h, kvh, lq, lk, dh,
                                              tuple(mask.shape) if mask is not None else None)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    mp, msz, mst = _aux_args(mask, lk)
    bp, bsz, bst = _aux_args(bias, lk)
    want_db = return_dbias or dbias is not None
    if want_db:
        if bias is None:
            raise ValueError("dbias needs a bias")
        if dbias is None:
            dbias = torch.empty(tuple(bias.shape), dtype=torch.float32, device=q.device)
        elif dbias.dtype != torch.float32 or tuple(dbias.shape) != tuple(bias.shape) or not dbias.is_contiguous():
            raise ValueError("dbias must be contiguous float32 with the bias's shape")
    args = (_dtype_code(q), b, h, kvh, lq, lk, dh, ctypes.c_float(0.0 if scale is None else float(scale)),
            1 if is_causal else 0,
            _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v),
            mp, msz, mst,
            bp, _dtype_code(bias) if bias is not None else 0, bsz, bst,
            _ptr(out), _strides3(out), _ptr(lse), _ptr(dout), _strides3(dout),
            _ptr(dq), _strides3(dq), _ptr(dk), _strides3(dk), _ptr(dv), _strides3(dv),
            _ptr(dbias) if want_db else ctypes.c_void_p(0), _ptr(workspace), workspace.numel())
    if deterministic and want_db:
        db_bytes = masked_attn_bwd_dbias_workspace_size(q.dtype, b, h, kvh, lq, dh, list(bias.shape))
        if dbias_workspace is None:
            dbias_workspace = torch.empty(max(db_bytes, 1), dtype=torch.uint8, device=q.device)
        nat.check(_lib().masked_attn_bwd_deterministic(*args, _ptr(dbias_workspace), dbias_workspace.numel(),
                                                       _stream(q)))
    else:
        nat.check(_lib().masked_attn_bwd(*args, _stream(q)))
    return (dq, dk, dv, dbias) if want_db else (dq, dk, dv)


def sparse_attn_fwd_workspace_size(dtype, batch, heads, kv_heads, q_len, k_len, head_dim, mask_shape,
                                   bias_dtype=None, bias_shape=None, max_keys=None) -> int:
    n = ctypes.c_size_t()
    bdt = _DTYPE[bias_dtype] if bias_dtype is not None else 0
    nat.check(_lib().sparse_attn_fwd_workspace_size(
        _DTYPE[dtype], batch, heads, kv_heads, q_len, k_len, head_dim, nat.i64_array(mask_shape), bdt,
        nat.i64_array(bias_shape) if bias_shape is not None else None,
        0 if max_keys is None else int(max_keys), ctypes.byref(n)))
    return n.value


def sparse_attn_fwd(q, k, v, mask, bias=None, is_causal: bool = False, scale=None, max_keys=None,
                    out=None, return_lse: bool = True, workspace=None):
    """Index-gather attention under a keep mask shared by every query.

    ``mask`` follows the 4D contract with a query dim of 1 and a head dim of
    1 or KVH (e.g. a dynamic top-k mask); ``max_keys`` bounds the kept keys of
    any mask row (the top-k window size).  The result equals
    ``masked_attn_fwd`` on the same arguments; only the kept keys are read.
    Returns ``(out, lse)``."""
    _require_cuda(q, k, v, mask, bias)
    b, lq, h, dh = q.shape
    lk, kvh = k.shape[1], k.shape[2]
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    if mask is None or mask.dtype not in (torch.bool, torch.uint8):
        raise ValueError("mask must be a bool tensor")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((b, h, lq), dtype=torch.float32, device=q.device) if return_lse else None
    ws_bytes = sparse_attn_fwd_workspace_size(q.dtype, b, h, kvh, lq, lk, dh, tuple(mask.shape),
                                              bias.dtype if bias is not None else None,
                                              tuple(bias.shape) if bias is not None else None, max_keys)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    mp, msz, mst = _aux_args(mask, lk)
    bp, bsz, bst = _aux_args(bias, lk)
    nat.check(_lib().sparse_attn_fwd(
        _dtype_code(q), b, h, kvh, lq, lk, dh, ctypes.c_float(0.0 if scale is None else float(scale)),
        1 if is_causal else 0,
        _ptr(q), _strides3(q), _ptr(k), _strides3(k), _ptr(v), _strides3(v),
        mp, msz, mst,
        bp, _dtype_code(bias) if bias is not None else 0, bsz, bst,
        0 if max_keys is None else int(max_keys),
        _ptr(out), _strides3(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(q)))
    return out, lse


def _strides2(t: torch.Tensor):
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("packed tensors must be 3D [total, heads, head_dim] with head_dim contiguous")
    return nat.i64_array(t.stride()[:2])


def _cu(t: torch.Tensor, batch=None) -> torch.Tensor:
    if t.dtype != torch.int32 or t.dim() != 1 or (batch is not None and t.shape[0] != batch + 1):
        raise ValueError("cu_seqlens must be int32 [batch + 1]")
    return t.contiguous()


def varlen_attn_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    is_causal: bool = False, scale=None, out=None, return_lse: bool = True, workspace=None,
                    mask=None, bias=None):
    """Attention over packed variable-length sequences.

    q ``[total_q, H, d]``, k/v ``[total_k, KVH, d]``; sequence b is rows
    ``cu_seqlens_q[b]:cu_seqlens_q[b+1]`` of q (keys likewise) and attends
    only its own keys (bottom-right causal per sequence when ``is_causal``).
    ``mask`` / ``bias``: 4D in the padded per-sequence layout of
    ``masked_attn_fwd`` for ``[batch, max_seqlen_q, H, max_seqlen_k]``
    (element ``(b, h, q, k)`` for sequence-local q and k), through
    ``varlen_masked_attn_fwd``.  Returns ``(out, lse)``, lse float32
    ``[H, total_q]``."""
    if mask is not None or bias is not None:
        return _varlen_masked_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, is_causal,
                                  scale, out, return_lse, workspace, mask, bias)
    _require_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k)
    total_q, h, dh = q.shape
    total_k, kvh = k.shape[0], k.shape[1]
    b = cu_seqlens_q.shape[0] - 1
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_k, b)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((h, total_q), dtype=torch.float32, device=q.device) if return_lse else None
    n = ctypes.c_size_t()
    nat.check(_lib().varlen_attn_fwd_workspace_size(b, int(max_seqlen_q), int(max_seqlen_k), ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    nat.check(_lib().varlen_attn_fwd(
        _dtype_code(q), b, h, kvh, dh, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k),
        ctypes.c_float(0.0 if scale is None else float(scale)), 1 if is_causal else 0,
        _ptr(cq), _ptr(ck), _ptr(q), _strides2(q), _ptr(k), _strides2(k), _ptr(v), _strides2(v),
        _ptr(out), _strides2(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(q)))
    return out, lse


def _varlen_masked_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_q, max_k, is_causal, scale, out, return_lse,
                       workspace, mask, bias):
    _require_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k, mask, bias)
    total_q, h, dh = q.shape
    total_k, kvh = k.shape[0], k.shape[1]
    b = cu_seqlens_q.shape[0] - 1
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_k, b)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((h, total_q), dtype=torch.float32, device=q.device) if return_lse else None
    n = ctypes.c_size_t()
    ms = nat.i64_array(mask.shape) if mask is not None else None
    nat.check(_lib().varlen_masked_attn_fwd_workspace_size(b, h, kvh, int(max_q), int(max_k), dh, ms,
                                                           ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    mp, msz, mst = _aux_args(mask, max_k)
    bp, bsz, bst = _aux_args(bias, max_k)
    nat.check(_lib().varlen_masked_attn_fwd(
        _dtype_code(q), b, h, kvh, dh, total_q, total_k, int(max_q), int(max_k),
        ctypes.c_float(0.0 if scale is None else float(scale)), 1 if is_causal else 0,
        _ptr(cq), _ptr(ck), _ptr(q), _strides2(q), _ptr(k), _strides2(k), _ptr(v), _strides2(v),
        mp, msz, mst, bp, _dtype_code(bias) if bias is not None else 0, bsz, bst,
        _ptr(out), _strides2(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(q)))
    return out, lse


def varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, is_causal: bool = False, scale=None, dq=None, dk=None, dv=None,
                    workspace=None, mask=None, bias=None, return_dbias: bool = False, dbias=None):
    """Gradients of ``varlen_attn_fwd`` (same sequences, mask / bias, causal
    flag and scale): ``out`` and ``lse`` are that call's results, ``dout`` the
    upstream gradient ``[total_q, H, d]``.  Returns ``(dq, dk, dv)`` in the
    packed layouts of q and k, or ``(dq, dk, dv, dbias)`` with
    ``return_dbias`` (or a ``dbias`` buffer): float32 at the bias's shape."""
    if mask is not None or bias is not None:
        return _varlen_masked_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                  max_seqlen_k, is_causal, scale, dq, dk, dv, workspace, mask, bias,
                                  return_dbias, dbias)
    if return_dbias or dbias is not None:
        raise ValueError("dbias needs a bias")
    _require_cuda(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k)
    total_q, h, dh = q.shape
    total_k, kvh = k.shape[0], k.shape[1]
    b = cu_seqlens_q.shape[0] - 1
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_k, b)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (h, total_q) or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous float32 [heads, total_q]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    n = ctypes.c_size_t()
    nat.check(_lib().varlen_attn_bwd_workspace_size(b, h, total_q, int(max_seqlen_q), int(max_seqlen_k), dh,
                                                    ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    nat.check(_lib().varlen_attn_bwd(
        _dtype_code(q), b, h, kvh, dh, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k),
        ctypes.c_float(0.0 if scale is None else float(scale)), 1 if is_causal else 0,
        _ptr(cq), _ptr(ck), _ptr(q), _strides2(q), _ptr(k), _strides2(k), _ptr(v), _strides2(v),
        _ptr(out), _strides2(out), _ptr(lse), _ptr(dout), _strides2(dout), _ptr(dq), _strides2(dq),
        _ptr(dk), _strides2(dk), _ptr(dv), _strides2(dv), _ptr(workspace), workspace.numel(), _stream(q)))
    return dq, dk, dv


def _varlen_masked_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_q, max_k, is_causal, scale,
                       dq, dk, dv, workspace, mask, bias, return_dbias, dbias):
    _require_cuda(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, mask, bias)
    total_q, h, dh = q.shape
    total_k, kvh = k.shape[0], k.shape[1]
    b = cu_seqlens_q.shape[0] - 1
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_k, b)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (h, total_q) or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous float32 [heads, total_q]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    want_db = return_dbias or dbias is not None
    if want_db:
        if bias is None:
            raise ValueError("dbias needs a bias")
        if dbias is None:
            dbias = torch.empty(tuple(bias.shape), dtype=torch.float32, device=q.device)
        elif dbias.dtype != torch.float32 or tuple(dbias.shape) != tuple(bias.shape) or not dbias.is_contiguous():
            raise ValueError("dbias must be contiguous float32 with the bias's shape")
    n = ctypes.c_size_t()
    ms = nat.i64_array(mask.shape) if mask is not None else None
    nat.check(_lib().varlen_masked_attn_bwd_workspace_size(b, h, kvh, total_q, int(max_q), int(max_k), dh, ms,
                                                           ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    mp, msz, mst = _aux_args(mask, max_k)
    bp, bsz, bst = _aux_args(bias, max_k)
    nat.check(_lib().varlen_masked_attn_bwd(
        _dtype_code(q), b, h, kvh, dh, total_q, total_k, int(max_q), int(max_k),
        ctypes.c_float(0.0 if scale is None else float(scale)), 1 if is_causal else 0,
        _ptr(cq), _ptr(ck), _ptr(q), _strides2(q), _ptr(k), _strides2(k), _ptr(v), _strides2(v),
        mp, msz, mst, bp, _dtype_code(bias) if bias is not None else 0, bsz, bst,
        _ptr(out), _strides2(out), _ptr(lse), _ptr(dout), _strides2(dout), _ptr(dq), _strides2(dq),
        _ptr(dk), _strides2(dk), _ptr(dv), _strides2(dv), _ptr(dbias) if want_db else ctypes.c_void_p(0),
        _ptr(workspace), workspace.numel(), _stream(q)))
    return (dq, dk, dv, dbias) if want_db else (dq, dk, dv)


def varlen_pad(packed: torch.Tensor, cu_seqlens: torch.Tensor, max_len: int) -> torch.Tensor:
    """``[batch, max_len, H, d]`` from packed ``[total, H, d]`` rows (zeros past each length)."""
    _require_cuda(packed, cu_seqlens)
    cu = _cu(cu_seqlens)
    b = cu.shape[0] - 1
    _, h, dh = packed.shape
    padded = torch.empty((b, int(max_len), h, dh), dtype=packed.dtype, device=packed.device)
    nat.check(_lib().varlen_pad(_dtype_code(packed), b, int(max_len), h, dh, _ptr(cu), _ptr(packed),
                                _strides2(packed), _ptr(padded), _strides3(padded), _stream(packed)))
    return padded


def varlen_unpad(padded: torch.Tensor, cu_seqlens: torch.Tensor, total: int) -> torch.Tensor:
    """Packed ``[total, H, d]`` rows from ``[batch, max_len, H, d]``."""
    _require_cuda(padded, cu_seqlens)
    cu = _cu(cu_seqlens, padded.shape[0])
    b, max_len, h, dh = padded.shape
    packed = torch.empty((int(total), h, dh), dtype=padded.dtype, device=padded.device)
    nat.check(_lib().varlen_unpad(_dtype_code(padded), b, max_len, h, dh, _ptr(cu), _ptr(padded),
                                  _strides3(padded), _ptr(packed), _strides2(packed), _stream(padded)))
    return packed


def _pre_mask_view(pre_mask: torch.Tensor, batch: int, q_len: int, k_len: int):
    """create_mask's shape step as a view: a 2D (batch, L) pre-mask becomes
    sizes (batch, 1, 1, L); columns >= L count as invalid, which equals
    padding with False (L == q_len < k_len) or cutting (L > k_len)."""
    if pre_mask.dim() == 2:
        if pre_mask.shape[0] != batch:
            raise ValueError("2D pre-mask must be (batch, seq_len)")
        if pre_mask.shape[1] not in (k_len, q_len):
            raise ValueError("2D pre-mask length must be key_len or query_len")
        return pre_mask.view(batch, 1, 1, pre_mask.shape[1])
    if pre_mask.dim() == 4:
        return pre_mask
    raise ValueError("pre-mask must be 2D or 4D")


def dynamic_topk_mask(bias: torch.Tensor, k_len: int, window_size: int, pre_mask=None, q_len=None,
                      out=None) -> torch.Tensor:
    """Bool keep mask of ``bias``'s shape: per row the ``window_size`` largest
    entries among the first ``k_len`` columns after the pre-mask, and'ed with
    the pre-mask.  The bias's key dim is ``round_up(k_len, 128)`` or
    ``k_len``."""
    _require_cuda(bias, pre_mask)
    if bias.dim() != 4:
        raise ValueError("bias must be 4D")
    if out is None:
        out = torch.empty(bias.shape, dtype=torch.bool, device=bias.device)
    pp, psz, pst = ctypes.c_void_p(0), None, None
    if pre_mask is not None:
        if pre_mask.dtype not in (torch.bool, torch.uint8):
            raise ValueError("pre-mask must be bool")
        pm = _pre_mask_view(pre_mask, bias.shape[0], bias.shape[2] if q_len is None else q_len, k_len)
        pp, psz, pst = _ptr(pm), nat.i64_array(pm.shape), nat.i64_array(pm.stride())
    nat.check(_lib().dynamic_topk_mask(_dtype_code(bias), _ptr(bias), nat.i64_array(bias.shape),
                                       nat.i64_array(bias.stride()), int(k_len), pp, psz, pst,
                                       int(window_size), _ptr(out), _stream(bias)))
    return out


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = ctypes.c_int32()
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    nat.check(_lib().sma_device_status(s, ctypes.byref(v)))
    return v.value


def selftest_wait_timeout(timeout_ns: int, out: torch.Tensor) -> None:
    """Diagnostic: a kernel waits on a barrier nothing completes, gives up
    after ``timeout_ns`` and reports SMA_ERR_DEVICE_TIMEOUT in the device error
    word (read it with ``device_status``).  ``out`` is int64[2] on the device:
    {1 if the wait gave up, nanoseconds waited}."""
    _require_cuda(out)
    if out.dtype != torch.int64 or out.numel() < 2:
        raise ValueError("out must be a CUDA int64 tensor with 2 elements")
    nat.check(_lib().sma_selftest_wait_timeout(int(timeout_ns), _ptr(out), _stream(out)))
