"""GPU parity: HEART per-head mask cache against the oracle's HeadMaskCache, and the
multi-step mask-reuse recipe."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _bsa():
    import block_sparse_attention_tcgen05_b200 as bsa
    return bsa


def _run_steps(delta, gate, relative, steps=6, H=8, S=2048, D=64, boost=10.0, sigma=0.05):
    bsa = _bsa()
    q0, k0, _ = wl.gaussian_qkv(1, H, H, S, D, "bf16", seed=11)
    Cq = Ck = 4
    gpu = bsa.MaskCache(1, H, Cq, Ck, D, delta, relative, gate[0], gate[1])
    ref = oracle.HeadMaskCache(delta, relative, gate[0], gate[1])
    g = np.random.default_rng(12)
    for t, (q, k) in enumerate(wl.drift_steps(q0, k0, steps, sigma, range(4), boost, seed=13)):
        new = g.random((1, H, Cq, Ck)) < 0.5
        r_gpu, n = gpu.should_refresh(q.cuda(), k.cuda())
        r_ref = ref.should_refresh(q.double().numpy(), k.double().numpy())
        d_gpu = gpu.drift.cpu().numpy()
        near = np.abs(ref.last_drift - delta) <= 1e-4 * max(delta, 1.0)
        if not near.any():
            np.testing.assert_array_equal(r_gpu.cpu().numpy().astype(bool), r_ref)
            assert n == int(r_ref.sum())
        fin = np.isfinite(ref.last_drift)
        np.testing.assert_allclose(d_gpu[fin], ref.last_drift[fin], rtol=1e-4)
        m_gpu = gpu.update(torch.from_numpy(new.astype(np.uint8)).cuda() if n else None)
        m_ref = ref.update(new, r_ref)
        np.testing.assert_array_equal(m_gpu.cpu().numpy().astype(bool), m_ref)
    assert bsa.device_status()[0] == 0


@pytest.mark.parametrize("delta,gate,relative", [
    (0.5, (-1.0, 0.8), False),   # gate off, per-head decisions (boosted heads refresh)
    (0.5, (0.4, 0.8), False),    # gate on: 4 of 8 heads drift -> per-head band
    (2.0, (0.4, 0.8), False),    # nothing drifts past delta
    (0.02, (-1.0, 0.8), True),   # relative drift
    (1e-6, (0.4, 0.8), False),   # every head drifts: gate refreshes all
])
def test_cache_matches_oracle(delta, gate, relative):
    _run_steps(delta, gate, relative)


def test_cache_reset():
    bsa = _bsa()
    q, k, _ = wl.gaussian_qkv(1, 4, 4, 512, 64, "bf16", seed=1)
    c = bsa.MaskCache(1, 4, 2, 2, 64, delta=100.0)
    r, n = c.should_refresh(q.cuda(), k.cuda())
    assert n == 4
    c.update(torch.ones(1, 4, 2, 2, dtype=torch.uint8).cuda())
    r, n = c.should_refresh(q.cuda(), k.cuda())
    assert n == 0
    c.reset()
    r, n = c.should_refresh(q.cuda(), k.cuda())
    assert n == 4


def test_reuse_recipe_reduced():
    """The mask-reuse recipe (pages' §Recipe) over 6 steps on a reduced video grid:
    per-head tau from (0.85, 0.90, 0.95), first 2 steps dense; masks and attention
    outputs checked against the oracle chain each step (masks outside tie rows)."""
    bsa = _bsa()
    grid = (4, 16, 32)   # S = 2048
    H, D, S = 6, 128, 2048
    q0, k0, v, _ = wl.positional_qkv(1, H, H, grid, D, ell=(3.0, 6.0, 8.0), amp=2.0,
                                     dtype="bf16", seed=5)
    tau = np.array([(0.85, 0.90, 0.95)[h % 3] for h in range(H)], dtype=np.float32)
    lab = np.arange(S) // 128
    lt = torch.as_tensor(lab, dtype=torch.int32).cuda()
    cache = bsa.MaskCache(1, H, 16, 16, D, delta=0.5, gate_lo=-1.0)
    ref = oracle.HeadMaskCache(0.5, gate_lo=-1.0)
    vc = v.cuda()
    for t, (q, k) in enumerate(wl.drift_steps(q0, k0, 6, 0.05, range(2), 10.0, seed=6)):
        if t < 2:
            continue  # dense warm-up steps leave the cache untouched
        qc, kc = q.cuda(), k.cuda()
        r, n = cache.should_refresh(qc, kc)
        r_ref = ref.should_refresh(q.double().numpy(), k.double().numpy())
        np.testing.assert_array_equal(r.cpu().numpy().astype(bool), r_ref)
        new = None
        new_ref = None
        if n:
            sc = bsa.antidiagonal_block_scores(qc, kc, 128, 16)
            new = bsa.top_p_block_mask(sc, torch.from_numpy(tau))
            sc_ref = oracle.antidiagonal_block_scores(q.double().numpy(), k.double().numpy(), 128, 16)
            new_ref, tie = oracle.top_p_block_mask(sc_ref, tau)
            bad = (new.cpu().numpy().astype(bool) != new_ref).any(-1) & ~tie
            assert not bad.any()
        m = cache.update(new)
        m_ref = ref.update(new_ref if new_ref is not None else ref.mask, r_ref)
        mg = m.cpu().numpy().astype(bool)
        out = bsa.centroid_compensated_attention(qc, kc, vc, lt, lt, m)
        rows = np.random.default_rng(t).choice(S, 128, replace=False)
        o_ref = oracle.centroid_compensated_attention(q.double().numpy(), k.double().numpy(),
                                                      v.double().numpy(), lab, lab, mg, rows=rows)
        got = out.cpu().numpy()[:, :, rows]
        assert np.abs(got - o_ref).max() <= 2e-2
        assert np.linalg.norm(got - o_ref) / np.linalg.norm(o_ref) <= 5e-3
    assert bsa.device_status()[0] == 0
