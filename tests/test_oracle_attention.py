"""Pins of the oracle's attention functions against what the pages and the
mathematics fix (no GPU). Each pin reaches the value by a route that shares no
code with the oracle: torch's scaled_dot_product_attention, explicit loops, or a
special case with a closed form."""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _inputs(B=1, Hq=2, Hkv=2, S=48, D=8, seed=0):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, Hq, S, D)), g.standard_normal((B, Hkv, S, D)),
            g.standard_normal((B, Hkv, S, D)))


def _sdpa(q, k, v, mask, scale):
    """torch's SDPA in float64 with an additive mask (a library softmax)."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask), scale=scale).numpy()


def _labels(S, C, seed):
    g = np.random.default_rng(seed)
    lab = np.concatenate([np.arange(C), g.integers(0, C, size=S - C)])
    return g.permutation(lab)


def test_dense_matches_library_sdpa():
    q, k, v = _inputs()
    out = oracle.dense_attention(q, k, v)
    ref = _sdpa(q, k, v, np.zeros((48, 48)), 8 ** -0.5)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_all_blocks_kept_equals_dense():
    """Every block kept: nothing is skipped, so compensated = hard drop = dense
    ("Sparse-block compensation", §The problem)."""
    q, k, v = _inputs()
    ql, kl = _labels(48, 5, 1), _labels(48, 6, 2)
    mask = np.ones((5, 6), dtype=bool)
    d = oracle.dense_attention(q, k, v)
    np.testing.assert_allclose(oracle.centroid_compensated_attention(q, k, v, ql, kl, mask), d,
                               atol=1e-12)
    np.testing.assert_allclose(oracle.hard_drop_attention(q, k, v, ql, kl, mask), d, atol=1e-12)


def test_one_key_per_cluster_equals_dense():
    """n_c = 1: the centroid is the key itself and ln 1 = 0, so compensating a
    skipped cluster restores its key exactly ("Sparse-block compensation",
    §SVG-EAR — centroid compensation)."""
    q, k, v = _inputs(S=40)
    ql = _labels(40, 4, 3)
    kl = np.random.default_rng(4).permutation(40)
    mask = np.random.default_rng(5).random((4, 40)) < 0.3
    out = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask)
    np.testing.assert_allclose(out, oracle.dense_attention(q, k, v), atol=1e-12)


def test_identical_keys_in_skipped_clusters_equals_dense():
    """If all keys (and values) of every cluster are equal, replacing a skipped
    cluster by one centroid term with prior ln n_c is exact."""
    g = np.random.default_rng(6)
    C, S, D = 6, 60, 8
    kl = g.permutation(np.repeat(np.arange(C), S // C))
    kc, vc = g.standard_normal((C, D)), g.standard_normal((C, D))
    k = kc[kl][None, None]
    v = vc[kl][None, None]
    q = g.standard_normal((1, 1, S, D))
    ql = _labels(S, 3, 7)
    mask = g.random((3, C)) < 0.4
    out = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask)
    np.testing.assert_allclose(out, oracle.dense_attention(q, k, v), atol=1e-12)


def test_compensation_equals_softmax_over_centroid_replaced_keys():
    """The page's starting point: every skipped key k_j is replaced by its cluster
    centroid k̄_c (and v_j by v̄_c) inside ONE softmax over all Sk keys. Collapsing
    the n_c equal logits gives the ln n_c prior; this checks that collapse, the
    centroid means and the label bookkeeping through torch's SDPA."""
    q, k, v = _inputs(Hq=4, Hkv=2, S=64, D=8, seed=8)
    ql, kl = _labels(64, 5, 9), _labels(64, 7, 10)
    mask = np.random.default_rng(11).random((4, 5, 7)) < 0.35
    out = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask)
    for h in range(4):
        g = h // 2
        kbar = np.stack([k[0, g, kl == c].mean(0) for c in range(7)])
        vbar = np.stack([v[0, g, kl == c].mean(0) for c in range(7)])
        for a in range(5):
            rows = np.nonzero(ql == a)[0]
            keep = mask[h, a, kl]
            kmod = np.where(keep[:, None], k[0, g], kbar[kl])
            vmod = np.where(keep[:, None], v[0, g], vbar[kl])
            ref = _sdpa(q[0, h, rows][None], kmod[None], vmod[None],
                        np.zeros((len(rows), 64)), 8 ** -0.5)[0]
            np.testing.assert_allclose(out[0, h, rows], ref, atol=1e-12)


def test_formulations_a_and_b_agree():
    """§No LSE needed: one softmax over [K; K̄] with the 0/−inf and ln n_c/−inf masks
    equals the per-cluster computation (both modes, GQA, an empty cluster)."""
    q, k, v = _inputs(Hq=4, Hkv=2, S=50, D=8, seed=12)
    ql = _labels(50, 4, 13)
    kl = _labels(50, 6, 14)
    kl[kl == 5] = 4  # cluster 5 becomes empty
    mask = np.random.default_rng(15).random((1, 4, 4, 6)) < 0.5
    for comp in (True, False):
        a = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask, compensate=comp, Ck=6)
        b = oracle.extended_key_attention(q, k, v, ql, kl, mask, compensate=comp, Ck=6)
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_hard_drop_equals_token_masked_sdpa():
    """Hard drop = SDPA with the block mask expanded to tokens ("Dynamic block masks
    and head-wise mask reuse", §Recipe: expand the mask to tokens for attention
    without compensation)."""
    q, k, v = _inputs(S=48, seed=16)
    ql, kl = np.arange(48) // 8, np.arange(48) // 12
    mask = np.random.default_rng(17).random((6, 4)) < 0.5
    mask[:, 0] = True  # every row keeps something, so SDPA has no all −inf row
    tok = np.where(np.repeat(np.repeat(mask, 8, 0), 12, 1), 0.0, -np.inf)
    ref = _sdpa(q, k, v, tok, 8 ** -0.5)
    np.testing.assert_allclose(oracle.hard_drop_attention(q, k, v, ql, kl, mask), ref, atol=1e-12)


def test_brute_force_loops_tiny():
    """Explicit scalar loops over the modified key set on a tiny case."""
    g = np.random.default_rng(18)
    S, D, Cq, Ck = 12, 3, 3, 4
    q = g.standard_normal((1, 1, S, D))
    k = g.standard_normal((1, 1, S, D))
    v = g.standard_normal((1, 1, S, D))
    ql = g.integers(0, Cq, S)
    kl = np.arange(S) % Ck
    mask = g.random((Cq, Ck)) < 0.5
    out = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask, Cq=Cq, Ck=Ck)
    sc = 1 / np.sqrt(D)
    for i in range(S):
        terms = []
        for c in range(Ck):
            members = [j for j in range(S) if kl[j] == c]
            if mask[ql[i], c]:
                for j in members:
                    dot = sum(q[0, 0, i, d] * k[0, 0, j, d] for d in range(D))
                    terms.append((sc * dot, v[0, 0, j]))
            else:
                kb = [sum(k[0, 0, j, d] for j in members) / len(members) for d in range(D)]
                vb = sum(v[0, 0, j] for j in members) / len(members)
                dot = sum(q[0, 0, i, d] * kb[d] for d in range(D))
                terms.append((sc * dot + np.log(len(members)), vb))
        mx = max(t for t, _ in terms)
        w = [np.exp(t - mx) for t, _ in terms]
        ref = sum(wi * val for wi, (_, val) in zip(w, terms)) / sum(w)
        np.testing.assert_allclose(out[0, 0, i], ref, atol=1e-12)


def test_all_skipped_row_hard_drop_is_zero_and_compensated_is_centroid_softmax():
    q, k, v = _inputs(S=16, seed=19)
    ql = np.zeros(16, dtype=int)
    kl = np.arange(16) // 4
    mask = np.zeros((1, 4), dtype=bool)
    np.testing.assert_array_equal(oracle.hard_drop_attention(q, k, v, ql, kl, mask), 0.0)
    out = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask)
    assert np.isfinite(out).all() and np.abs(out).max() > 0


def test_rows_subset_matches_full():
    q, k, v = _inputs(Hq=2, Hkv=1, S=40, seed=20)
    ql, kl = _labels(40, 4, 21), _labels(40, 5, 22)
    mask = np.random.default_rng(23).random((4, 5)) < 0.5
    full = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask)
    rows = np.array([39, 0, 17, 5])
    sub = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask, rows=rows)
    np.testing.assert_allclose(sub, full[:, :, rows], atol=0)


def test_executed_pairs_counts_cells():
    ql = np.array([0, 0, 1, 1, 1])
    kl = np.array([0, 1, 1, 2])
    mask = np.array([[1, 0, 1], [0, 1, 0]], dtype=bool)
    # cells: (0,0) 2*1, (0,2) 2*1, (1,1) 3*2  -> 10 per head; 2 heads; probes 3*4 per head
    assert oracle.executed_pairs(ql, kl, mask, H=2, M=3) == 2 * 10 + 2 * 3 * 4
