"""Pins of the oracle's tile labels, probe selection, residual repair and mask cache
(no GPU)."""

import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- labels
def test_tile_labels_video_grid_counts():
    """21 × 30 × 52 grid cut into 3 × 6 × 8 tiles: 7 × 5 × 7 = 245 tiles; the last
    tile column holds 52 − 6·8 = 4 columns, so 210 tiles of 144 tokens and 35 of 72."""
    lab, C = oracle.tile_labels(21, 30, 52, (3, 6, 8))
    assert C == 245 and lab.shape == (32760,)
    cnt = np.bincount(lab, minlength=C)
    assert sorted(np.unique(cnt).tolist()) == [72, 144]
    assert (cnt == 144).sum() == 210 and (cnt == 72).sum() == 35


def test_tile_labels_encode_tile_coordinates():
    """Expanding a tile-level relation through the labels reproduces the token-level
    relation ("Sparse-block compensation", §Recipe: the tile-resolution mask expanded
    through tile_labels reproduces the token-level mask). Tokens share a label iff
    they share a tile; the window relation on tiles matches the token relation."""
    T, H, W, tile = 4, 6, 10, (2, 3, 4)
    lab, C = oracle.tile_labels(T, H, W, tile)
    t, h, w = np.unravel_index(np.arange(T * H * W), (T, H, W))
    tc = np.stack([t // 2, h // 3, w // 4], 1)
    same = (tc[:, None, :] == tc[None, :, :]).all(-1)
    np.testing.assert_array_equal(same, lab[:, None] == lab[None, :])
    # one tile-level window mask (Chebyshev radius 1), expanded through labels
    reps = np.zeros((C, 3), dtype=int)
    reps[lab] = tc
    tmask = (np.abs(reps[:, None] - reps[None]) <= 1).all(-1)
    tok = (np.abs(tc[:, None] - tc[None]) <= 1).all(-1)
    np.testing.assert_array_equal(tmask[lab][:, lab], tok)


@pytest.mark.parametrize("grid,tile,window", [
    ((4, 6, 10), (2, 3, 4), (1, 1, 3)),      # partial edge tiles along W (10 = 4 + 4 + 2)
    ((6, 6, 8), (2, 2, 2), (3, 3, 3)),       # 3 x 3 x 4 tiles, windows clamped at the borders
    ((5, 4, 9), (1, 2, 2), (5, 1, 3)),       # window as wide as the T axis keeps all of it
    ((3, 5, 7), (1, 1, 1), (3, 5, 9)),       # token resolution, windows past the grid
])
def test_sliding_tile_mask_expands_to_the_token_level_sta_mask(grid, tile, window):
    """"Sparse-block compensation", §Recipe: the tile-resolution sliding-tile mask,
    expanded through tile_labels, reproduces the token-level STA mask (computed token
    pair by token pair from the tokens' own tile coordinates)."""
    lab, C = oracle.tile_labels(*grid, tile)
    n = [-(-g // t) for g, t in zip(grid, tile)]
    m = oracle.sliding_tile_block_mask(*n, window)
    assert m.shape == (C, C)
    np.testing.assert_array_equal(m[lab][:, lab], oracle.sta_token_mask(*grid, tile, window))


def test_sliding_tile_mask_window_by_explicit_loops():
    """The window written the other way round, by loops: along an axis of n tiles a
    window of w = 2r + 1 tiles starts at min(max(a − r, 0), n − w) (shifted inward at
    the borders) and holds w consecutive tiles; a window of at least n tiles holds
    them all. Every query tile therefore keeps exactly the product of min(w, n) key
    tiles, the diagonal is always kept, (1,1,1) is the identity."""
    nT, nH, nW, window = 4, 3, 6, (3, 1, 5)
    m = oracle.sliding_tile_block_mask(nT, nH, nW, window)

    def axis_keep(a, c, n, w):
        if w >= n:
            return True
        start = min(max(a - w // 2, 0), n - w)
        return start <= c < start + w

    for a in range(nT * nH * nW):
        at, ah, aw = a // (nH * nW), (a // nW) % nH, a % nW
        for c in range(nT * nH * nW):
            ct, ch, cw = c // (nH * nW), (c // nW) % nH, c % nW
            want = (axis_keep(at, ct, nT, 3) and axis_keep(ah, ch, nH, 1)
                    and axis_keep(aw, cw, nW, 5))
            assert m[a, c] == want, (a, c)
    assert (m.sum(1) == 3 * 1 * 5).all() and m.diagonal().all()
    np.testing.assert_array_equal(oracle.sliding_tile_block_mask(3, 4, 5, (1, 1, 1)), np.eye(60))
    assert oracle.sliding_tile_block_mask(3, 4, 5, (3, 5, 5)).all()


# ----------------------------------------------------------------------------- probes
def test_probe_rows_tiny_golden():
    rows = np.loadtxt(os.path.join(GOLDEN, "probe_rows_tiny.txt"), comments="#")
    idx, w = oracle.select_probe_rows(np.arange(1024) // 64, 64)
    np.testing.assert_array_equal(idx, rows[:, 1].astype(int))
    np.testing.assert_allclose(w, rows[:, 2], atol=0)


def test_probe_rows_fewer_probes_than_clusters_and_uneven():
    lab = np.repeat(np.arange(10), [5, 1, 2, 9, 3, 4, 4, 6, 2, 1])
    idx, w = oracle.select_probe_rows(lab, 4)
    assert [lab[i] for i in idx] == [0, 2, 5, 7]          # floor(i*10/4)
    assert np.isclose(w.sum(), 1)
    # M = 14 >= C = 10: round-robin over the query clusters in ascending label order
    # ("Sparse-block compensation", §What mlx-arsenal ships), each pass taking the next
    # preferred member of every cluster that still has one. Cluster rows (offsets):
    #   0: 0-4 (5)  1: 5 (1)  2: 6-7 (2)  3: 8-16 (9)  4: 17-19 (3)
    #   5: 20-23 (4)  6: 24-27 (4)  7: 28-33 (6)  8: 34-35 (2)  9: 36 (1)
    # Middle-out order ranks members by |2r - (n-1)|, ties to the lower rank r:
    #   n=5 -> r 2,1,3,0,4;  n=2 -> r 0,1;  n=9 -> r 4,3,5,..;  n=3 -> r 1,0,2;
    #   n=4 -> r 1,2,0,3;  n=6 -> r 2,3,1,4,..
    # Pass 0 takes one row of every cluster: 2, 5, 6, 12, 18, 21, 25, 30, 34, 36.
    # Pass 1 skips the exhausted clusters 1 and 9 and stops after four more rows, all
    # from the first clusters in label order that still have members: 0 -> 1, 2 -> 7,
    # 3 -> 11, 4 -> 17.
    idx, w = oracle.select_probe_rows(lab, 14)
    np.testing.assert_array_equal(idx, [2, 5, 6, 12, 18, 21, 25, 30, 34, 36, 1, 7, 11, 17])
    owners = lab[idx]
    assert np.bincount(owners, minlength=10).tolist() == [2, 1, 2, 2, 2, 1, 1, 1, 1, 1]
    # weights are |G_a| / m_a normalised: sizes 5,1,2,9,3,4,4,6,2,1 over probe counts
    raw = np.array([5 / 2, 1, 2 / 2, 9 / 2, 3 / 2, 4, 4, 6, 2, 1, 5 / 2, 2 / 2, 9 / 2, 3 / 2])
    np.testing.assert_allclose(w, raw / raw.sum())
    # exhaustion: M = 37 takes every row once (clusters drop out as they empty); a
    # larger M cannot take more rows than exist
    idx, w = oracle.select_probe_rows(lab, 37)
    assert sorted(idx.tolist()) == list(range(37))
    np.testing.assert_allclose(w, np.full(37, 1 / 37))
    # passes 6, 7 and 8 only find members left in the 9-row cluster 3, whose middle-out
    # order is r = 4,3,5,2,6,1,7,0,8: its ranks 6, 7, 8 are rows 8 + {7, 0, 8}
    np.testing.assert_array_equal(idx[-3:], [15, 8, 16])
    idx, _ = oracle.select_probe_rows(lab, 50)
    assert len(idx) == 37


def test_probe_rows_centroid_distance_brute_force():
    g = np.random.default_rng(0)
    q = g.standard_normal((1, 2, 30, 4))
    lab = np.arange(30) // 10
    idx, w = oracle.select_probe_rows_centroid(q, lab, 6)
    for h in range(2):
        for a in range(3):
            rows = np.arange(10 * a, 10 * a + 10)
            c = q[0, h, rows].mean(0)
            d = [np.linalg.norm(q[0, h, r] - c) for r in rows]
            best2 = [rows[j] for j in np.argsort(d)[:2]]
            assert idx[0, h, a] == best2[0] and idx[0, h, 3 + a] == best2[1]
    np.testing.assert_allclose(w, 1 / 6)


def test_probe_dense_attention_per_head_gqa_against_library_sdpa():
    """Per-head probe rows under grouped-query attention ("Partition the Support,
    Reconstruct the Residual": M query rows evaluated exactly against all keys, KV
    heads shared by contiguous groups of query heads). Each (b, h) is checked against
    torch's scaled_dot_product_attention on the rows probe_idx[b, h] of query head h and
    KV head h // (Hq / Hkv). Hq = 6 over Hkv = 2 makes a wrong grouping (h % Hkv) or a
    probe index taken from another head fail."""
    import torch

    g = np.random.default_rng(8)
    B, Hq, Hkv, S, D, M = 2, 6, 2, 40, 8, 5
    q = g.standard_normal((B, Hq, S, D))
    k = g.standard_normal((B, Hkv, S, D))
    v = g.standard_normal((B, Hkv, S, D))
    pidx = g.integers(0, S, (B, Hq, M))
    got = oracle.probe_dense_attention(q, k, v, pidx)
    qt, kt, vt = (torch.from_numpy(x) for x in (q, k, v))
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt[b, h, pidx[b, h]][None], kt[b, kv][None], vt[b, kv][None])[0]
            np.testing.assert_allclose(got[b, h], ref.numpy(), atol=1e-12)
    # shared rows (M,): the same rows in every head
    rows = pidx[0, 0]
    shared = oracle.probe_dense_attention(q, k, v, rows)
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt[b, h, rows][None], kt[b, kv][None], vt[b, kv][None])[0]
            np.testing.assert_allclose(shared[b, h], ref.numpy(), atol=1e-12)


# ----------------------------------------------------------------------------- repair
def _repair_case(seed=0, S=200, D=6, M=40):
    g = np.random.default_rng(seed)
    X = g.standard_normal((1, 1, S, D))
    idx = g.choice(S, M, replace=False)
    w = g.random(M) + 0.5
    w /= w.sum()
    Op = X[:, :, idx] + 0.1 * g.standard_normal((1, 1, M, D))
    return X, Op, idx, w


def test_ridge_equals_lstsq_on_augmented_system():
    """With full rank the projector is the identity, and the fit is the ridge
    solution: least squares on [√W·Z̃; √λ·I′] (a library solve)."""
    X, Op, idx, w = _repair_case()
    D = 6
    out, parts = oracle.probe_residual_correction(X, Op, idx, w, rank=D, lam=0.1,
                                                  return_parts=True)
    x = X[0, 0]
    Z = (x - x.mean(0)) / np.sqrt(x.var(0) + 1e-6)
    Zt = np.concatenate([Z, np.ones((len(x), 1))], 1)[idx]
    R = Op[0, 0] - x[idx]
    Ipen = np.sqrt(0.1) * np.eye(D + 1)[:D]
    Aaug = np.concatenate([np.sqrt(w)[:, None] * Zt, Ipen], 0)
    Yaug = np.concatenate([np.sqrt(w)[:, None] * R, np.zeros((D, D))], 0)
    coef = np.linalg.lstsq(Aaug, Yaug, rcond=None)[0]
    np.testing.assert_allclose(parts["coef"][0, 0], coef, atol=1e-10)
    Zall = np.concatenate([(x - x.mean(0)) / np.sqrt(x.var(0) + 1e-6), np.ones((len(x), 1))], 1)
    np.testing.assert_allclose(out[0, 0], x + Zall @ coef, atol=1e-10)


def test_exact_recovery_of_low_rank_affine_residual():
    """R exactly affine in Z and inside a rank-r subspace, λ → 0, M ≥ D + 1: the
    repair reproduces the dense output on every row, not only at the probes."""
    g = np.random.default_rng(1)
    S, D, r, M = 300, 20, 4, 60
    X = g.standard_normal((1, 1, S, D))
    x = X[0, 0]
    Z = (x - x.mean(0)) / np.sqrt(x.var(0) + 1e-6)
    U = np.linalg.qr(g.standard_normal((D, r)))[0]
    Btrue = g.standard_normal((D + 1, r)) @ U.T
    dense = x + np.concatenate([Z, np.ones((S, 1))], 1) @ Btrue
    idx = g.choice(S, M, replace=False)
    w = np.full(M, 1 / M)
    out = oracle.probe_residual_correction(X, dense[None, None, idx], idx, w, rank=r, lam=1e-12)
    np.testing.assert_allclose(out[0, 0], dense, atol=1e-8)


def test_projector_and_probe_identity():
    X, Op, idx, w = _repair_case(seed=2, D=8, M=50)
    out, parts = oracle.probe_residual_correction(X, Op, idx, w, rank=3, return_parts=True)
    Vr = parts["Vr"][0, 0]
    P = Vr @ Vr.T
    np.testing.assert_allclose(P @ P, P, atol=1e-12)
    np.testing.assert_allclose(P, P.T, atol=1e-12)
    R = Op[0, 0] - X[0, 0, idx]
    G = R.T @ (w[:, None] * R)
    ev = np.linalg.eigvalsh(G)[::-1]
    # the subspace is the top-3 eigenspace of RᵀWR
    np.testing.assert_allclose(np.trace(Vr.T @ G @ Vr), ev[:3].sum(), rtol=1e-10)
    # probe rows after repair differ from their dense rows by minus the fit residual
    np.testing.assert_allclose(out[0, 0, idx] - Op[0, 0], -parts["fit_residual"][0, 0],
                               atol=1e-12)


def test_repair_reduces_error_on_sparse_attention():
    """Hard-drop block-sparse output repaired with 64 dense probe rows gets closer to
    dense ("Partition the Support, Reconstruct the Residual", ablations)."""
    g = np.random.default_rng(3)
    S, D = 512, 16
    q = g.standard_normal((1, 1, S, D))
    k = q + 0.3 * g.standard_normal((1, 1, S, D))
    v = g.standard_normal((1, 1, S, D))
    lab = np.arange(S) // 32
    mask = np.abs(np.arange(16)[:, None] - np.arange(16)[None]) <= 2
    sp = oracle.hard_drop_attention(q, k, v, lab, lab, mask)
    dense = oracle.dense_attention(q, k, v)
    idx, w = oracle.select_probe_rows(lab, 64)
    rep = oracle.probe_residual_correction(sp, oracle.probe_dense_attention(q, k, v, idx), idx, w)
    e0 = np.linalg.norm(sp - dense)
    e1 = np.linalg.norm(rep - dense)
    assert e1 < e0


# ----------------------------------------------------------------------------- cache
def test_cache_decisions_hand_computed():
    """"Dynamic block masks and head-wise mask reuse", §HEART: drift = L1 distance of
    pooled q̄, k̄ to the anchor; refresh above δ; gate under 40 % / above 80 %."""
    c = oracle.HeadMaskCache(delta=1.0, gate_lo=-1)
    q0 = np.zeros((1, 5, 4, 2))
    k0 = np.zeros((1, 5, 4, 2))
    assert c.should_refresh(q0, k0).all()          # first call: all heads
    m0 = np.zeros((1, 5, 2, 2), dtype=bool)
    c.update(m0, np.ones((1, 5), dtype=bool))
    q1 = q0.copy()
    q1[0, 0] += 0.6   # q̄ moves by 0.6 in both coordinates: L1 drift 1.2 > 1
    q1[0, 1, :, 0] += 0.9  # drift 0.9 ≤ 1
    ref = c.should_refresh(q1, k0)
    np.testing.assert_array_equal(ref[0], [True, False, False, False, False])
    np.testing.assert_allclose(c.last_drift[0, :2], [1.2, 0.9])
    m1 = np.ones((1, 5, 2, 2), dtype=bool)
    out = c.update(m1, ref)
    assert out[0, 0].all() and not out[0, 1:].any()
    # the anchor of head 0 moved: the same input no longer drifts
    assert not c.should_refresh(q1, k0)[0, 0]


def test_cache_layer_gate_and_relative_and_reset():
    c = oracle.HeadMaskCache(delta=1.0)        # gate 0.4 / 0.8
    q = np.zeros((1, 10, 3, 2))
    k = np.ones((1, 10, 3, 2))
    c.should_refresh(q, k)
    c.update(np.zeros((1, 10, 1, 1), dtype=bool), np.ones((1, 10), dtype=bool))
    q3 = q.copy()
    q3[0, :3] += 1.0            # 3 of 10 heads drift by 2 > 1: 30 % < 40 % -> none
    assert not c.should_refresh(q3, k).any()
    q9 = q.copy()
    q9[0, :9] += 1.0            # 90 % > 80 % -> all
    assert c.should_refresh(q9, k).all()
    q5 = q.copy()
    q5[0, :5] += 1.0            # 50 % -> per head
    np.testing.assert_array_equal(c.should_refresh(q5, k)[0], [True] * 5 + [False] * 5)
    r = oracle.HeadMaskCache(delta=0.5, relative=True, gate_lo=-1)
    r.should_refresh(q, k)
    r.update(np.zeros((1, 10, 1, 1), dtype=bool), np.ones((1, 10), dtype=bool))
    # anchor L1 norm = |q̄|₁ + |k̄|₁ = 0 + 2; drift 2 -> relative 1.0 > 0.5
    assert r.should_refresh(q5, k)[0, :5].all()
    r.reset()
    assert r.should_refresh(q, k).all()
