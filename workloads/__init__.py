"""Seeded synthetic inputs for the structured-mask attention workloads.

This module only draws inputs: random tensors, anchors, masks and biases of
the shapes and structures of the workloads below.  It holds none of the
attention, tile-map or top-k arithmetic, and it is the only code that both
the CUDA path's tests/benchmark and the float64 oracle consume.

Recipe: ``numpy.random.default_rng(seed)``; tensors are drawn as float32
N(0, 1) and cast to the target dtype with round-to-nearest-even (torch's
``.to``); the oracle reads the cast values.  Anchors are sorted draws (with
replacement) from ``[1, ctx_len]``.

Workloads (named by what they are):

* ``dflash_tiny``      B=1, H=KVH=2, d=64, fp32; 64 context keys, 4 draft
  blocks of 16 with anchors 16, 32, 48, 64; full layer, is_causal unset.
* ``dflash_train``     B=2, H=32, KVH=8, d=128, bf16; 4096 context keys,
  256 blocks of 16; is_causal unset; full layer and sliding layer (W=2048).
* ``dflash_long``      B=1, H=32, KVH=8, d=128, bf16; 32768 context keys,
  2048 blocks of 16; is_causal=True; full layer and sliding layer (W=4096).
* ``broadcast_prefill`` B=4, H=16, KVH=4, d=128, bf16; Lq=8192, Lk=8000;
  bias (4, 4, 1, 8064) N(0,1); bool mask (1, 1, 8192, 8064) keeping
  ``k <= q + Lk - Lq``.
* ``broadcast_decode`` B=8, H=32, KVH=8, d=128, bf16; Lq=1, Lk=16384;
  bias (8, 32, 1, 16384) N(0,1); optional mask (8, 8, 1, 16384) Bernoulli(0.9).
* ``topk``             bias (2, 8, 1, 16384) bf16 N(0,1); 2D pre-mask
  (2, 16384) with the last 10% of keys invalid in batch 1; window 2048;
  then attention H=32, KVH=8, d=128, Lq=4096, Lk=16384, causal.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

TORCH_DTYPE = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def round_up(x: int, m: int = 128) -> int:
    return (x + m - 1) // m * m


@dataclass(frozen=True)
class DFlashWorkload:
    name: str
    batch: int
    heads: int
    kv_heads: int
    head_dim: int
    dtype: str
    ctx_len: int
    n_blocks: int
    block_size: int
    is_causal: int          # -1 unset, 0, 1
    layer_type: int         # 0 full, 1 sliding
    sliding_window: int
    seed: int
    anchors: tuple = field(default=())   # fixed anchors; empty -> random sorted

    @property
    def n_q(self) -> int:
        return self.n_blocks * self.block_size

    @property
    def n_k(self) -> int:
        return self.ctx_len + self.n_q


DFLASH_TINY = DFlashWorkload("dflash_tiny", 1, 2, 2, 64, "fp32", 64, 4, 16, -1, 0, 0, 0,
                             anchors=(16, 32, 48, 64))
DFLASH_TRAIN_FULL = DFlashWorkload("dflash_train_full", 2, 32, 8, 128, "bf16", 4096, 256, 16,
                                   -1, 0, 0, 1)
DFLASH_TRAIN_SLIDING = replace(DFLASH_TRAIN_FULL, name="dflash_train_sliding", layer_type=1,
                               sliding_window=2048)
DFLASH_LONG_FULL = DFlashWorkload("dflash_long_full", 1, 32, 8, 128, "bf16", 32768, 2048, 16,
                                  1, 0, 0, 2)
DFLASH_LONG_SLIDING = replace(DFLASH_LONG_FULL, name="dflash_long_sliding", layer_type=1,
                              sliding_window=4096)


def rng_for(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def normal(rng: np.random.Generator, shape, dtype: str) -> torch.Tensor:
    """float32 N(0,1) cast (round-to-nearest-even) to ``dtype``; CPU tensor."""
    x = torch.from_numpy(rng.standard_normal(size=shape, dtype=np.float32))
    return x.to(TORCH_DTYPE[dtype])


def sorted_anchors(rng: np.random.Generator, batch: int, n_blocks: int, ctx_len: int) -> torch.Tensor:
    """Sorted draws with replacement from ``[1, ctx_len]``, int32 ``[B, N]``."""
    a = rng.integers(1, ctx_len + 1, size=(batch, n_blocks))
    a.sort(axis=1)
    return torch.from_numpy(a.astype(np.int32))


def dflash_inputs(w: DFlashWorkload, seed: int | None = None):
    """(q [B,Nq,H,d], k [B,Lk,KVH,d], v [B,Lk,KVH,d], anchors int32 [B,N])."""
    rng = rng_for(w.seed if seed is None else seed)
    q = normal(rng, (w.batch, w.n_q, w.heads, w.head_dim), w.dtype)
    k = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    v = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    if w.anchors:
        anchors = torch.tensor([list(w.anchors)] * w.batch, dtype=torch.int32)
    else:
        anchors = sorted_anchors(rng, w.batch, w.n_blocks, w.ctx_len)
    return q, k, v, anchors


def random_anchors(rng: np.random.Generator, batch: int, n_blocks: int, ctx_len: int,
                   sort: bool = False, low: int = 0) -> torch.Tensor:
    """Anchors drawn from ``[low, ctx_len]`` (duplicates allowed), optionally sorted."""
    a = rng.integers(low, ctx_len + 1, size=(batch, n_blocks))
    if sort:
        a.sort(axis=1)
    return torch.from_numpy(a.astype(np.int32))


@dataclass(frozen=True)
class MaskedWorkload:
    name: str
    batch: int
    heads: int
    kv_heads: int
    head_dim: int
    dtype: str
    n_q: int
    n_k: int
    is_causal: bool
    bias_shape: tuple | None        # (b', h', q', K) with K = round_up(n_k)
    mask_shape: tuple | None
    mask_kind: str                  # "causal_keep" | "bernoulli" | "none"
    seed: int
    keep_prob: float = 0.9

    @property
    def k_pad(self) -> int:
        return round_up(self.n_k)


BROADCAST_PREFILL = MaskedWorkload("broadcast_prefill", 4, 16, 4, 128, "bf16", 8192, 8000, False,
                                   (4, 4, 1, 8064), (1, 1, 8192, 8064), "causal_keep", 3)
BROADCAST_DECODE = MaskedWorkload("broadcast_decode", 8, 32, 8, 128, "bf16", 1, 16384, False,
                                  (8, 32, 1, 16384), None, "none", 3)
BROADCAST_DECODE_MASKED = replace(BROADCAST_DECODE, name="broadcast_decode_masked",
                                  mask_shape=(8, 8, 1, 16384), mask_kind="bernoulli")


def causal_keep_mask_input(mask_shape, n_q: int, n_k: int) -> torch.Tensor:
    """Input mask of ``mask_shape`` whose row q keeps columns
    ``k <= q + n_k - n_q`` (bottom-right); padded columns are set True so a
    kernel that read them would be caught."""
    b_, h_, q_, kp = mask_shape
    q = torch.arange(q_).view(q_, 1) if q_ > 1 else torch.full((1, 1), n_q - 1)
    k = torch.arange(kp).view(1, kp)
    m = (k <= q + (n_k - n_q)) | (k >= n_k)
    return m.view(1, 1, q_, kp).expand(b_, h_, q_, kp).contiguous()


def masked_inputs(w: MaskedWorkload, seed: int | None = None):
    """(q, k, v, mask or None, bias or None) as CPU tensors."""
    rng = rng_for(w.seed if seed is None else seed)
    q = normal(rng, (w.batch, w.n_q, w.heads, w.head_dim), w.dtype)
    k = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    v = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    bias = normal(rng, w.bias_shape, w.dtype) if w.bias_shape is not None else None
    mask = None
    if w.mask_shape is not None:
        if w.mask_kind == "causal_keep":
            mask = causal_keep_mask_input(w.mask_shape, w.n_q, w.n_k)
        elif w.mask_kind == "bernoulli":
            mask = torch.from_numpy(rng.random(size=w.mask_shape) < w.keep_prob)
        else:
            raise ValueError(w.mask_kind)
    return q, k, v, mask, bias


@dataclass(frozen=True)
class TopkWorkload:
    name: str
    batch: int
    kv_heads: int
    bias_q: int              # bias q-dim (1 = broadcast over queries)
    n_k: int
    window: int
    invalid_frac_batch1: float
    dtype: str
    seed: int
    heads: int = 32
    head_dim: int = 128
    n_q: int = 4096


TOPK = TopkWorkload("topk", 2, 8, 1, 16384, 2048, 0.1, "bf16", 4)
TOPK_WIDE = replace(TOPK, name="topk_wide", bias_q=4096)


def topk_inputs(w: TopkWorkload, seed: int | None = None):
    """(bias [B, KVH, bias_q, Kpad], pre_mask 2D bool [B, Lk])."""
    rng = rng_for(w.seed if seed is None else seed)
    bias = normal(rng, (w.batch, w.kv_heads, w.bias_q, round_up(w.n_k)), w.dtype)
    pre = torch.ones((w.batch, w.n_k), dtype=torch.bool)
    if w.batch > 1:
        n_bad = int(np.floor(w.invalid_frac_batch1 * w.n_k))
        pre[1, w.n_k - n_bad:] = False
    return bias, pre


def topk_attention_inputs(w: TopkWorkload, seed: int | None = None):
    """(q [B, Lq, H, d], k, v [B, Lk, KVH, d]) for the attention after top-k."""
    rng = rng_for((w.seed if seed is None else seed) + 1000)
    q = normal(rng, (w.batch, w.n_q, w.heads, w.head_dim), w.dtype)
    k = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    v = normal(rng, (w.batch, w.n_k, w.kv_heads, w.head_dim), w.dtype)
    return q, k, v
