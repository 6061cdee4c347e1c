"""Full / partial / empty classification of 128x128 tiles of a dense keep mask.

Test infrastructure only (see ``oracle/__init__.py``).

Source: SpecForge issue #452 "flex_attention BlockMask incorrectly created
with H=num_heads" -- flex_attention's ``create_block_mask`` turns a dense mask
into per-(batch, head, query block) lists of fully and partially visible key
blocks, and the page asks for that map with a head dim of 1.  flash-sparse-
attention PR #190, Stability fix: the kernels walk key blocks of 128 against
the rounded key length, so columns at or beyond Lk are never visible.

Definition used here, over valid query rows only (``q < n_q``):
* FULL    -- the tile lies wholly inside ``[0, Lk)`` and every entry is kept;
* EMPTY   -- no entry is kept;
* PARTIAL -- otherwise.
Index lists are ascending and padded with -1.
"""
from __future__ import annotations

import numpy as np

TILE = 128
EMPTY, PARTIAL, FULL = 0, 1, 2


def classify_block(keep_tile: np.ndarray, cols_in_range: bool) -> int:
    """Code of one tile given its kept entries (rows = valid query rows,
    columns = keys below Lk) and whether the tile lies inside [0, Lk)."""
    if keep_tile.size == 0 or not keep_tile.any():
        return EMPTY
    if cols_in_range and keep_tile.all():
        return FULL
    return PARTIAL


def tile_codes(keep: np.ndarray, n_k: int, tile: int = TILE) -> np.ndarray:
    """Codes ``[ceil(rows/tile), ceil(n_k/tile)]`` of a 2D keep mask whose
    columns beyond ``n_k`` (if any) are ignored."""
    rows = keep.shape[0]
    qt = -(-rows // tile)
    kt = -(-n_k // tile)
    codes = np.zeros((qt, kt), dtype=np.uint8)
    for a in range(qt):
        r0, r1 = a * tile, min((a + 1) * tile, rows)
        for c in range(kt):
            c0, c1 = c * tile, min((c + 1) * tile, n_k)
            codes[a, c] = classify_block(keep[r0:r1, c0:c1], (c + 1) * tile <= n_k)
    return codes


def lists_from_codes(codes: np.ndarray):
    """Ascending full / partial key-tile lists (padded with -1) from a
    ``[..., KT]`` code array."""
    kt = codes.shape[-1]
    flat = codes.reshape(-1, kt)
    n_full = np.zeros(flat.shape[0], dtype=np.int32)
    n_part = np.zeros(flat.shape[0], dtype=np.int32)
    full_idx = np.full((flat.shape[0], kt), -1, dtype=np.int32)
    part_idx = np.full((flat.shape[0], kt), -1, dtype=np.int32)
    for r in range(flat.shape[0]):
        f = np.nonzero(flat[r] == FULL)[0]
        p = np.nonzero(flat[r] == PARTIAL)[0]
        n_full[r], n_part[r] = len(f), len(p)
        full_idx[r, : len(f)] = f
        part_idx[r, : len(p)] = p
    lead = codes.shape[:-1]
    return (n_full.reshape(lead), full_idx.reshape(lead + (kt,)),
            n_part.reshape(lead), part_idx.reshape(lead + (kt,)))


def block_map_from_rows(keep_rows, n_batch: int, n_q: int, n_k: int, tile: int = TILE):
    """Block map of a mask supplied one query tile at a time.

    ``keep_rows(b, q0, q1)`` returns the dense keep rows ``[q1-q0, n_k]`` of
    batch ``b``.  Returns ``(num_full [B,QT], full_idx [B,QT,KT],
    num_part [B,QT], part_idx [B,QT,KT])``.
    """
    qt = -(-n_q // tile)
    kt = -(-n_k // tile)
    codes = np.zeros((n_batch, qt, kt), dtype=np.uint8)
    for b in range(n_batch):
        for a in range(qt):
            r0, r1 = a * tile, min((a + 1) * tile, n_q)
            codes[b, a] = tile_codes(keep_rows(b, r0, r1), n_k, tile)[0]
    return lists_from_codes(codes)


def mask_tile_summary(mask: np.ndarray, n_k: int, tile: int = TILE) -> np.ndarray:
    """Codes of an explicit 4D bool mask at its own (broadcast) shape:
    ``uint8 [b', h', ceil(q'/tile), ceil(n_k/tile)]``; columns >= n_k count
    as not kept.  A key dim of 1 is one flag for every key (expanded over the
    n_k keys)."""
    mask = np.asarray(mask, dtype=bool)
    if mask.shape[-1] == 1:
        mask = np.broadcast_to(mask, mask.shape[:-1] + (n_k,))
    b_, h_, q_, _ = mask.shape
    out = np.zeros((b_, h_, -(-q_ // tile), -(-n_k // tile)), dtype=np.uint8)
    for i in range(b_):
        for j in range(h_):
            out[i, j] = tile_codes(mask[i, j, :, :n_k], n_k, tile)
    return out
