"""Pins of the oracle's SparsePR Response-Coupled Partitioning (no GPU).

Source: "Partition the Support, Reconstruct the Residual" (paper summary): keys are
grouped by their pre-softmax response to sampled queries, key-group centroids define
the query coordinates, queries with a similar response direction share a route.
"""

import numpy as np

import oracle


def test_kmeans_one_round_by_explicit_loops():
    """One Lloyd round written with loops: assignment to the nearest centroid (ties to the
    lower index), centroids moved to their rows' means, a final assignment."""
    g = np.random.default_rng(0)
    x = g.standard_normal((23, 3))
    C = 4
    cent = [x[(2 * c + 1) * 23 // (2 * C)].copy() for c in range(C)]

    def assign(cent):
        lab = []
        for i in range(23):
            best, bc = None, None
            for c in range(C):
                d = sum((x[i, t] - cent[c][t]) ** 2 for t in range(3))
                if best is None or d < best:
                    best, bc = d, c
            lab.append(bc)
        return lab

    lab = assign(cent)
    for c in range(C):
        rows = [i for i in range(23) if lab[i] == c]
        if rows:
            cent[c] = np.mean([x[i] for i in rows], axis=0)
    np.testing.assert_array_equal(oracle.kmeans(x, C, 1), assign(cent))
    np.testing.assert_array_equal(oracle.kmeans(x, C, 0), lab)


def test_kmeans_recovers_planted_separated_clusters():
    """Well-separated blobs, one per evenly spaced starting row: every row ends in its
    blob's cluster (a textbook fixed point)."""
    g = np.random.default_rng(1)
    C, n = 6, 20
    centres = g.standard_normal((C, 5)) * 50
    x = np.concatenate([centres[c] + g.standard_normal((n, 5)) for c in range(C)])
    lab = oracle.kmeans(x, C, 8)
    np.testing.assert_array_equal(lab, np.repeat(np.arange(C), n))


def test_features_by_explicit_arithmetic_and_gqa_sharing():
    """Key features are scale times the logits of the sampled queries (token
    floor((s + 1/2) Sq / rK) of query head g G + s mod G); query coordinates are scale
    times the logits against rQ' evenly spaced key-group centroids, over the G heads of
    the group, normalised to unit length. Labels are one array per KV head."""
    g = np.random.default_rng(2)
    B, Hq, Hkv, S, D, C = 1, 4, 2, 40, 6, 5
    q = g.standard_normal((B, Hq, S, D))
    k = g.standard_normal((B, Hkv, S, D))
    ql, kl, fk, xq = oracle.response_coupled_partition(q, k, C, C, r_k=6, r_q=3, iters=2,
                                                       return_features=True)
    assert ql.shape == (1, 2, S) and kl.shape == (1, 2, S)
    sc = D ** -0.5
    for gi in range(Hkv):
        for j in range(S):
            for s in range(6):
                tok, h = (2 * s + 1) * S // 12, gi * 2 + s % 2
                assert abs(fk[0, gi, j, s] - sc * np.dot(q[0, h, tok], k[0, gi, j])) < 1e-12
        np.testing.assert_array_equal(kl[0, gi], oracle.kmeans(fk[0, gi], C, 2))
        kbar = np.stack([k[0, gi, kl[0, gi] == c].mean(0) if (kl[0, gi] == c).any() else
                         np.zeros(D) for c in range(C)])
        cols = [(2 * t + 1) * C // 6 for t in range(3)]
        for i in range(S):
            raw = [sc * np.dot(q[0, gi * 2 + hh, i], kbar[c]) for hh in range(2) for c in cols]
            want = np.array(raw) / np.linalg.norm(raw)
            np.testing.assert_allclose(xq[0, gi, i], want, atol=1e-12)
        np.testing.assert_array_equal(ql[0, gi], oracle.kmeans(xq[0, gi], C, 2))


def test_keys_with_planted_response_profiles_are_grouped():
    """Keys drawn around Ck well-separated directions give Ck response profiles; the key
    partition recovers the planted groups (up to the group numbering)."""
    g = np.random.default_rng(3)
    Ck, n, D = 4, 16, 16
    dirs = np.linalg.qr(g.standard_normal((D, Ck)))[0].T * 12.0
    k = np.concatenate([dirs[c] + 0.05 * g.standard_normal((n, D)) for c in range(Ck)])[None, None]
    q = g.standard_normal((1, 1, 64, D))
    _, kl = oracle.response_coupled_partition(q, k, 4, Ck, r_k=48, iters=8)
    lab = kl[0, 0].reshape(Ck, n)
    assert all(len(set(row)) == 1 for row in lab) and len(set(lab[:, 0])) == Ck
