"""GPU parity: the tile-resolution Sliding Tile Attention mask and the video workload
driven by it ("Sparse-block compensation", §Recipe: STA with both repairs)."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _bsa():
    import block_sparse_attention_tcgen05_b200 as bsa
    return bsa


@pytest.mark.parametrize("tiles,window", [((7, 5, 7), (3, 3, 5)), ((3, 3, 4), (3, 3, 3)),
                                          ((4, 3, 6), (3, 1, 5)), ((5, 1, 9), (7, 3, 2)),
                                          ((1, 1, 1), (1, 1, 1)), ((16, 8, 16), (5, 3, 7))])
def test_sliding_tile_mask_bit_exact(tiles, window):
    bsa = _bsa()
    got = bsa.sliding_tile_block_mask(tiles, window).cpu().numpy().astype(bool)
    np.testing.assert_array_equal(got, oracle.sliding_tile_block_mask(*tiles, window))
    assert bsa.device_status()[0] == 0


def test_sta_recipe_video_static_sampled():
    """The recipe at the video shape: tile_labels 3x6x8 on 21x30x52, the STA mask at tile
    resolution with a (3, 3, 5) tile window (19 % of token pairs), centroid compensation;
    the GPU mask expanded through the GPU labels equals the oracle's token-level STA mask
    on sampled rows, and sampled attention rows of four heads match the oracle."""
    bsa = _bsa()
    grid, tile, window = (21, 30, 52), (3, 6, 8), (3, 3, 5)
    q, k, v, _ = wl.positional_qkv(1, 8, 8, grid, 128, ell=(3.0, 6.0, 8.0), amp=2.0,
                                   dtype="bf16", seed=3)
    lab, C = bsa.tile_labels(*grid, tile)
    mask = bsa.sliding_tile_block_mask((7, 5, 7), window)
    lab_n, mask_n = lab.cpu().numpy(), mask.cpu().numpy().astype(bool)
    rows = np.sort(np.random.default_rng(14).choice(32760, 192, replace=False))
    tok = oracle.sta_token_mask(*grid, tile, window, rows=rows)
    np.testing.assert_array_equal(mask_n[lab_n[rows]][:, lab_n], tok)
    out = bsa.centroid_compensated_attention(q.cuda(), k.cuda(), v.cuda(), lab, lab, mask)
    got = out.cpu().numpy()
    assert bsa.device_status()[0] == 0
    heads = [0, 3, 5, 7]
    qh, kh, vh = (t[:, heads].double().numpy() for t in (q, k, v))
    ref = oracle.centroid_compensated_attention(qh, kh, vh, lab_n, lab_n, mask_n, rows=rows,
                                                Cq=C, Ck=C)
    g = got[:, heads][:, :, rows]
    assert np.abs(g - ref).max() <= 2e-2
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3
