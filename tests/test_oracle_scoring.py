"""Pins of the oracle's anti-diagonal scoring and top-p selection (no GPU)."""

import itertools

import numpy as np
import torch

import oracle


def _qk(B=1, H=2, N=32, D=4, seed=0):
    g = np.random.default_rng(seed)
    return g.standard_normal((B, H, N, D)), g.standard_normal((B, H, N, D))


def test_rows_sum_to_one():
    """"Dynamic block masks and head-wise mask reuse", §Deviations: rows normalised
    to 1."""
    q, k = _qk(N=64, D=8)
    sc = oracle.antidiagonal_block_scores(q, k, block=16, stride=4)
    np.testing.assert_allclose(sc.sum(-1), 1.0, atol=1e-12)
    assert (sc >= 0).all()


def test_stride_one_is_exact_block_attention_mass():
    """With stride 1 each sub-block is one logit, so the score is the block sum of
    dense softmax attention probabilities divided by the block size (a textbook
    reduction, computed here with torch's softmax)."""
    q, k = _qk(N=32, D=8, seed=1)
    b = 8
    sc = oracle.antidiagonal_block_scores(q, k, block=b, stride=1)
    P = torch.softmax(torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) * 8 ** -0.5,
                      dim=-1).numpy()
    ref = P.reshape(1, 2, 4, b, 4, b).sum(axis=(3, 5)) / b
    np.testing.assert_allclose(sc, ref, atol=1e-12)


def test_brute_force_loops():
    """Explicit loops: sub-block (I, J) of QKᵀ summed along its anti-diagonal, i.e.
    entries (I·s + t, J·s + s − 1 − t)."""
    q, k = _qk(B=1, H=1, N=32, D=3, seed=2)
    s, b = 4, 8
    sc = oracle.antidiagonal_block_scores(q, k, block=b, stride=s)
    ns = 32 // s
    A = np.zeros((ns, ns))
    for I in range(ns):
        for J in range(ns):
            acc = 0.0
            for t in range(s):
                i, j = I * s + t, J * s + s - 1 - t
                acc += sum(q[0, 0, i, d] * k[0, 0, j, d] for d in range(3))
            A[I, J] = acc / np.sqrt(3)
    P = np.exp(A - A.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    ref = np.zeros((4, 4))
    for I in range(ns):
        for J in range(ns):
            ref[I // 2, J // 2] += P[I, J]
    ref /= b // s
    np.testing.assert_allclose(sc[0, 0], ref, atol=1e-12)


def test_antidiagonal_not_diagonal():
    """A case where only the anti-diagonal orientation gives mass: key rows placed so
    that q_{Is+t} meets k_{Js+s-1-t}."""
    N, D, s = 16, 2, 4
    q = np.zeros((1, 1, N, D))
    k = np.zeros((1, 1, N, D))
    q[0, 0, 0] = [30.0, 0]          # I = 0, t = 0
    k[0, 0, 4 + 3] = [30.0, 0]      # J = 1, s-1-t = 3  -> anti-diagonal hit
    k[0, 0, 8 + 0] = [30.0, 0]      # J = 2, offset 0   -> only a diagonal would hit
    sc = oracle.antidiagonal_block_scores(q, k, block=4, stride=4, logit_scale=1.0)
    assert sc[0, 0, 0].argmax() == 1


def _brute_topp(row, tau):
    """Minimal number of blocks whose total reaches tau (all subsets)."""
    n = len(row)
    for r in range(1, n + 1):
        for sub in itertools.combinations(range(n), r):
            if row[list(sub)].sum() >= tau:
                return r
    return n


def test_top_p_minimal_cardinality_brute_force():
    g = np.random.default_rng(3)
    sc = g.dirichlet(np.ones(8), size=(1, 3, 6))
    for tau in (0.3, 0.6, 0.9):
        mask, _ = oracle.top_p_block_mask(sc, tau)
        for h in range(3):
            for i in range(6):
                row = sc[0, h, i]
                assert mask[0, h, i].sum() == _brute_topp(row, tau)
                assert row[mask[0, h, i]].sum() >= tau - 1e-12
                # the kept set is the heaviest one of that size
                assert row[mask[0, h, i]].min() >= row[~mask[0, h, i]].max(initial=-1)


def test_top_p_tiny_tau_is_argmax_and_scale_invariant():
    g = np.random.default_rng(4)
    sc = g.dirichlet(np.ones(10), size=(2, 2, 5))
    m, _ = oracle.top_p_block_mask(sc, 1e-9)
    assert (m.sum(-1) == 1).all()
    np.testing.assert_array_equal(m.argmax(-1), sc.argmax(-1))
    # relative to the row total (§Deviations): raw tile sums with tau scaled agree
    m1, _ = oracle.top_p_block_mask(sc, 0.7)
    m2, _ = oracle.top_p_block_mask(sc * 3.0, 2.1)
    np.testing.assert_array_equal(m1, m2)


def test_top_p_per_head_tau_and_ties():
    sc = np.array([[[[0.5, 0.25, 0.25, 0.0]], [[0.5, 0.25, 0.25, 0.0]]]])
    m, tie = oracle.top_p_block_mask(sc, np.array([0.5, 0.9]))
    np.testing.assert_array_equal(m[0, 0, 0], [True, False, False, False])
    np.testing.assert_array_equal(m[0, 1, 0], [True, True, True, False])
    assert tie[0, 0, 0]  # cum 0.5 sits exactly on tau
    assert not tie[0, 1, 0]  # cut between 0.25 (kept) and 0.0 (dropped): no tie
    m2, tie2 = oracle.top_p_block_mask(np.array([[[[0.4, 0.3, 0.3]]]]), 0.6)
    np.testing.assert_array_equal(m2[0, 0, 0], [True, True, False])  # lower index first
    assert tie2[0, 0, 0]     # equal scores on both sides of the cut


def test_top_p_float32_mode_runs_in_float32():
    g = np.random.default_rng(5)
    sc = g.dirichlet(np.ones(16), size=(1, 1, 4)).astype(np.float32)
    m32, _ = oracle.top_p_block_mask(sc, 0.9, dtype=np.float32)
    for i in range(4):
        row = sc[0, 0, i]
        order = np.argsort(-row, kind="stable")
        acc = np.float32(0)
        keep = []
        for j in order:
            keep.append(j)
            acc = np.float32(acc + row[j])
            if acc >= np.float32(0.9):
                break
        exp = np.zeros(16, dtype=bool)
        exp[keep] = True
        np.testing.assert_array_equal(m32[0, 0, i], exp)
