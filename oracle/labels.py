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
