"""Oracle: Sliding-Tile-Attention tile labels.

Test infrastructure only (see the package docstring).

Source: "Sparse-block compensation", §What mlx-arsenal ships (``tile_labels``: cluster
labels matching Sliding Tile Attention tiles) and §Recipe: STA with both repairs.
"""

import numpy as np


def tile_labels(T, H, W, tile):
    """Label of every token of a T × H × W latent grid (raster order t, h, w).

    Token s = (t·H + h)·W + w belongs to tile (t // tt, h // th, w // tw) and gets
    label ((t // tt)·nH + h // th)·nW + w // tw, with nH = ceil(H / th) and
    nW = ceil(W / tw). Reading: the recipe divides the grid with floor division,
    which loses tokens when a tile does not divide its axis (W = 52, tw = 8); here
    the tile counts round up, so edge tiles are partial.
    Returns (labels (T·H·W,) int64, number of tiles).
    """
    tt, th, tw = tile
    nT, nH, nW = -(-T // tt), -(-H // th), -(-W // tw)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    lab = ((t // tt) * nH + (h // th)) * nW + (w // tw)
    return lab.reshape(-1).astype(np.int64), nT * nH * nW


def _window_axis(n, w):
    """Kept key tiles of every query tile along one axis of n tiles, window w tiles:
    (n, n) bool. Reading of the Sliding Tile Attention window: the window holds the key
    tiles within w // 2 of its centre, and the centre is the query tile moved inward at
    the borders (clamped to [w // 2, n − 1 − w // 2]) so that the window stays inside
    the grid; a window at least as wide as the axis keeps every tile."""
    a = np.arange(n)
    r = w // 2
    if 2 * r + 1 >= n:
        return np.ones((n, n), dtype=bool)
    centre = np.clip(a, r, n - 1 - r)
    return np.abs(a[None, :] - centre[:, None]) <= r


def sliding_tile_block_mask(nT, nH, nW, window):
    """Tile-resolution Sliding Tile Attention mask ("Sparse-block compensation",
    §Recipe: STA with both repairs, where it is evaluated at tile resolution, one cell
    per tile): (C, C) bool over the C = nT·nH·nW tiles in the raster order of
    ``tile_labels``; query tile a keeps key tile c when c lies inside a's window on
    every axis (``_window_axis``). ``window`` = (wt, wh, ww) in tiles."""
    wt, wh, ww = window
    mt, mh, mw = _window_axis(nT, wt), _window_axis(nH, wh), _window_axis(nW, ww)
    m = mt[:, None, None, :, None, None] & mh[None, :, None, None, :, None] \
        & mw[None, None, :, None, None, :]
    C = nT * nH * nW
    return m.reshape(C, C)


def sta_token_mask(T, H, W, tile, window, rows=None):
    """Token-level Sliding Tile Attention mask of a T × H × W grid (raster order t, h,
    w), computed token pair by token pair: query token i attends key token j when, on
    every axis, the tile coordinate of j lies inside the window of i's tile coordinate
    (tile coordinate = coordinate // tile size; windows as in ``_window_axis`` over the
    ceil(X / tile) tiles of the axis). (S, S) bool, or (len(rows), S) for the query
    tokens ``rows``. This is the mask that the tile-resolution mask expanded through
    ``tile_labels`` must reproduce."""
    S = T * H * W
    t, h, w = np.unravel_index(np.arange(S), (T, H, W))
    rows = np.arange(S) if rows is None else np.asarray(rows)
    keep = np.ones((len(rows), S), dtype=bool)
    for coord, size, n_ax, win in ((t, tile[0], -(-T // tile[0]), window[0]),
                                   (h, tile[1], -(-H // tile[1]), window[1]),
                                   (w, tile[2], -(-W // tile[2]), window[2])):
        tc = coord // size
        r = win // 2
        if 2 * r + 1 >= n_ax:
            continue
        centre = np.minimum(np.maximum(tc[rows], r), n_ax - 1 - r)
        keep &= np.abs(tc[None, :] - centre[:, None]) <= r
    return keep
