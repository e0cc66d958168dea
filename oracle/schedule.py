"""Brute-force 128x128 tile classification from the explicit mask.

Test infrastructure (see the package docstring).

The pages describe structured masks kept as compact attention slices so a
kernel can skip masked work ([picx] Training Infrastructure,
"Flex-Flash-Attention"); they give no tile format, so the format is this
reading:

* Query tiles are 128 consecutive queries, the first starting at query 0.
* Key tiles are 128 consecutive keys of ONE key source: the cache (its keys
  0..n_cache-1) or the current segments (their keys 0..n_queries-1). Tiles
  are numbered cache tiles first, then current tiles:
  ``t < ceil(n_cache/128)`` is cache keys [128t, 128t+128); otherwise
  ``u = t - ceil(n_cache/128)`` is current keys [128u, 128u+128).
* A tile pair is FULL when all 128x128 positions exist and are visible,
  EMPTY when no existing position is visible, PARTIAL otherwise.
* The schedule lists, per query tile, its non-EMPTY key tiles in ascending
  tile order with their class (CSR).
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np

from .rule import Layout

TILE = 128
EMPTY, PARTIAL, FULL = 0, 1, 2


def key_tiles(layout: Layout) -> List[Tuple[int, int]]:
    """(first key index in the key sequence, number of existing keys) per tile."""
    out = []
    for base, n in ((0, layout.n_cache), (layout.n_cache, layout.n_queries)):
        for t0 in range(0, n, TILE):
            out.append((base + t0, min(TILE, n - t0)))
    return out


def classify_query_tile(layout: Layout, qt: int) -> np.ndarray:
    """Class (EMPTY/PARTIAL/FULL) of every key tile for query tile ``qt``."""
    rows = np.arange(qt * TILE, min((qt + 1) * TILE, layout.n_queries))
    mask = layout.mask_rows(rows)
    tiles = key_tiles(layout)
    out = np.empty(len(tiles), dtype=np.uint8)
    for i, (k0, nk) in enumerate(tiles):
        block = mask[:, k0:k0 + nk]
        seen = int(block.sum())
        if seen == 0:
            out[i] = EMPTY
        elif len(rows) == TILE and nk == TILE and seen == TILE * TILE:
            out[i] = FULL
        else:
            out[i] = PARTIAL
    return out


def n_query_tiles(layout: Layout) -> int:
    return (layout.n_queries + TILE - 1) // TILE


def schedule(layout: Layout) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """CSR schedule: row_ptr [nQt+1], kv_tile [nnz], flag [nnz] (1 PARTIAL, 2 FULL)."""
    row_ptr = [0]
    tiles, flags = [], []
    for qt in range(n_query_tiles(layout)):
        cls = classify_query_tile(layout, qt)
        nz = np.nonzero(cls != EMPTY)[0]
        tiles.append(nz.astype(np.int32))
        flags.append(cls[nz])
        row_ptr.append(row_ptr[-1] + len(nz))
    cat = (lambda xs, dt: np.concatenate(xs).astype(dt) if xs else np.zeros(0, dt))
    return (np.asarray(row_ptr, dtype=np.int32), cat(tiles, np.int32), cat(flags, np.uint8))
