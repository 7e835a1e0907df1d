"""Pins of the oracle's SVG-EAR error-aware routing (no GPU).

Sources: "Sparse-block compensation", §SVG-EAR — centroid compensation (an
error-aware router chooses which blocks to compute exactly); the SVG-EAR abstract on
the block-sparse attention topic feed (a probe estimates each block's compensation
error; the blocks with the highest error-to-cost ratio are computed exactly).
"""

import numpy as np
import torch

import oracle


def _case(seed=0, B=1, Hq=2, Hkv=1, S=48, D=8, C=6):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, S, D))
    k = g.standard_normal((B, Hkv, S, D))
    v = g.standard_normal((B, Hkv, S, D))
    ql = g.permutation(np.arange(S) % C)
    kl = g.permutation(np.concatenate([np.arange(C), g.integers(0, C, S - C)]))
    return q, k, v, ql, kl


def test_error_equals_probability_deviation_from_the_centroid_term():
    """An independent route to the same number: with p = softmax(scale · K q̄_a) taken by
    the library and p̄_c = exp(scale · q̄_a · k̄_c − logsumexp), the difference of the
    exact and compensated block contributions is Σ_{j∈c} (p_j − p̄_c) v_j, because
    n_c v̄_c = Σ_{j∈c} v_j."""
    q, k, v, ql, kl = _case(Hq=4, Hkv=2)
    C, D = 6, 8
    err = oracle.compensation_errors(q, k, v, ql, kl, C, C)
    for h in range(4):
        g = h // 2
        K, V = torch.from_numpy(k[0, g]), torch.from_numpy(v[0, g])
        for a in range(C):
            qbar = torch.from_numpy(q[0, h, ql == a].mean(0))
            logits = (K @ qbar) * D ** -0.5
            p = torch.softmax(logits, 0)
            lse = torch.logsumexp(logits, 0)
            for c in range(C):
                sel = torch.from_numpy(kl == c)
                kbar = K[sel].mean(0)
                pbar = torch.exp((qbar @ kbar) * D ** -0.5 - lse)
                want = torch.linalg.vector_norm(((p[sel] - pbar)[:, None] * V[sel]).sum(0))
                np.testing.assert_allclose(err[0, h, a, c], want.item(), rtol=1e-10, atol=1e-14)


def test_error_vanishes_where_compensation_is_exact():
    """One key per cluster, or identical keys inside every cluster: the centroid term
    equals the block's exact contribution ("Sparse-block compensation", §SVG-EAR:
    keys of a cluster share one logit), so every block error is 0."""
    g = np.random.default_rng(1)
    q = g.standard_normal((1, 1, 12, 4))
    k = g.standard_normal((1, 1, 12, 4))
    v = g.standard_normal((1, 1, 12, 4))
    lab = np.arange(12)
    assert np.abs(oracle.compensation_errors(q, k, v, lab % 3, lab, 3, 12)).max() < 1e-15
    kc = np.repeat(g.standard_normal((1, 1, 4, 4)), 3, axis=2)   # 4 clusters of 3 equal keys
    err = oracle.compensation_errors(q, kc, v, lab % 3, lab // 3, 3, 4)
    assert np.abs(err).max() < 1e-14


def test_selection_is_the_budgeted_prefix_of_the_ratio_order():
    """The kept blocks are the longest prefix of the (ratio descending, index ascending)
    order whose token pairs fit the budget: written here with Python's sort and a loop.
    Every kept block's ratio is at least every dropped non-empty block's; density 1 keeps
    every non-empty block and density 0 none."""
    q, k, v, ql, kl = _case(seed=2, Hq=3, Hkv=3, C=5)
    C = 5
    nq, nk = np.bincount(ql, minlength=C), np.bincount(kl, minlength=C)
    for density in (0.0, 0.1, 0.3, 0.55, 1.0):
        mask, err = oracle.error_aware_block_mask(q, k, v, ql, kl, C, C, density)
        budget = int(np.floor(density * 48 * 48))
        for h in range(3):
            items = sorted(((-err[0, h, a, c] / nk[c], a * C + c) for a in range(C)
                            for c in range(C) if nq[a] and nk[c]))
            want = np.zeros((C, C), dtype=bool)
            used = 0
            for _, e in items:
                a, c = divmod(e, C)
                if used + nq[a] * nk[c] > budget:
                    break
                used += nq[a] * nk[c]
                want[a, c] = True
            np.testing.assert_array_equal(mask[0, h], want)
            ratio = err[0, h] / nk[None, :]
            if want.any() and (~want).any():
                assert ratio[want].min() >= ratio[~want].max()
        if density == 1.0:
            assert mask.all()
        if density == 0.0:
            assert not mask.any()


def test_empty_clusters_are_never_kept():
    q, k, v, _, _ = _case(seed=3)
    ql = np.arange(48) % 4          # query cluster 4 of 5 is empty
    kl = np.arange(48) % 3          # key clusters 3, 4 of 5 are empty
    mask, err = oracle.error_aware_block_mask(q, k, v, ql, kl, 5, 5, 1.0)
    assert not mask[:, :, 4].any() and not mask[:, :, :, 3:].any()
    assert mask[:, :, :4, :3].all()
    assert (err[:, :, 4] == 0).all() and (err[:, :, :, 3:] == 0).all()


def test_centroid_mass_is_the_softmax_over_centroid_terms_by_library():
    """The cell mass equals torch's softmax of scale · q̄_a · k̄_c + ln n_c over the
    non-empty key clusters; rows sum to 1."""
    q, k, v, ql, kl = _case(seed=4, Hq=2, Hkv=1, C=5)
    kl = np.where(kl == 2, 0, kl)          # key cluster 2 empty
    mass = oracle.centroid_mass(q, k, ql, kl, 5, 5)
    for h in range(2):
        for a in range(5):
            qbar = torch.from_numpy(q[0, h, ql == a].mean(0))
            logits = []
            for c in (0, 1, 3, 4):
                kb = torch.from_numpy(k[0, 0, kl == c].mean(0))
                logits.append((qbar @ kb) * 8 ** -0.5 + np.log((kl == c).sum()))
            p = torch.softmax(torch.stack(logits), 0).numpy()
            np.testing.assert_allclose(mass[0, h, a, [0, 1, 3, 4]], p, rtol=1e-12)
            assert mass[0, h, a, 2] == 0.0
    np.testing.assert_allclose(mass.sum(-1), 1.0)


def test_probe_budget_reserves_the_probe_cost_first():
    """With M probe rows the routing budget is (density − M/Sq)·Sq·Sk pairs: the kept
    cells plus the M·Sk probe pairs never exceed density·Sq·Sk, and the mask is the
    budgeted prefix of the mass-per-pair order."""
    q, k, v, ql, kl = _case(seed=5, Hq=2, Hkv=2, C=6)
    nq, nk = np.bincount(ql, minlength=6), np.bincount(kl, minlength=6)
    for density, M in ((0.3, 8), (0.5, 12), (0.1, 10)):
        mask, mass = oracle.probe_budget_block_mask(q, k, ql, kl, 6, 6, density, M)
        for h in range(2):
            pairs = (nq[:, None] * nk[None, :])[mask[0, h]].sum()
            assert pairs <= max(0.0, density * 48 * 48 - M * 48) + 1e-9
            if M / 48 >= density:            # the probes alone use the whole budget
                assert pairs == 0
        want = oracle.route_blocks(mass, ql, kl, 6, 6, max(0.0, density - M / 48))
        np.testing.assert_array_equal(mask, want)
