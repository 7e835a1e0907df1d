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


def _host_means(x):
    """Float64 token means per head of a (1, H, S, D) device tensor, shaped (1, H, 1, D)
    (the oracle's pooling then reduces a singleton axis); computed head by head."""
    return np.stack([x[0, h].double().mean(0).cpu().numpy() for h in range(x.shape[1])])[None, :, None]


def test_reuse_recipe_video_full_size():
    """The mask-reuse workload at full size: B=1, H=40, S=32760 (21x30x52), D=128,
    20 steps of cumulative N(0, 0.05^2) drift (10x on heads 0-3), first 2 steps dense,
    delta=8, gate 0.4/0.8, tau per head from (0.85, 0.90, 0.95), block 128, stride 16
    (scoring on S padded to 32768), centroid-compensated attention every step.
    Refresh decisions, counts and drifts for every head are checked against the oracle
    cache each step; for sampled heads the oracle computes its own scores, top-p masks
    (equal outside tie rows) and attention rows with its own masks."""
    bsa = _bsa()
    dev = torch.device("cuda", 0)
    grid, H, D, S, Sp, C = (21, 30, 52), 40, 128, 32760, 32768, 256
    heads = [0, 1, 2, 3, 17, 38]
    q0, k0, v = wl.positional_qkv_device(1, H, H, grid, D, ell=(3.0, 6.0, 8.0), amp=2.0,
                                         seed=5, device=dev)
    tau = np.array([(0.85, 0.90, 0.95)[h % 3] for h in range(H)], dtype=np.float32)
    lab = np.arange(S) // 128
    lt = torch.as_tensor(lab, dtype=torch.int32, device=dev)
    cache = bsa.MaskCache(1, H, C, C, D, delta=8.0, gate_lo=0.4, gate_hi=0.8)
    ref = oracle.HeadMaskCache(8.0, gate_lo=0.4, gate_hi=0.8)
    sig = torch.full((1, H, 1, 1), 0.05, device=dev)
    sig[:, :4] *= 10.0
    g = torch.Generator(device=dev).manual_seed(55)
    qa, ka = q0.float(), k0.float()
    pad = torch.zeros((1, H, Sp - S, D), dtype=torch.bfloat16, device=dev)
    rng = np.random.default_rng(56)
    n_refresh_steps = 0
    for t in range(20):
        if t > 0:
            qa += torch.randn(qa.shape, generator=g, device=dev) * sig
            ka += torch.randn(ka.shape, generator=g, device=dev) * sig
        if t < 2:
            continue  # dense warm-up steps leave the cache untouched
        q, k = qa.to(torch.bfloat16), ka.to(torch.bfloat16)
        r, n = cache.should_refresh(q, k)
        r_ref = ref.should_refresh(_host_means(q), _host_means(k))
        np.testing.assert_array_equal(r.cpu().numpy().astype(bool), r_ref)
        assert n == int(r_ref.sum())
        fin = np.isfinite(ref.last_drift)
        np.testing.assert_allclose(cache.drift.cpu().numpy()[fin], ref.last_drift[fin],
                                   rtol=1e-3, atol=1e-5)
        new = None
        new_ref = np.zeros((1, H, C, C), dtype=bool)  # heads outside `heads`: not compared
        tie_rows = np.zeros((H, C), dtype=bool)
        if n:
            n_refresh_steps += 1
            qp, kp = torch.cat([q, pad], 2), torch.cat([k, pad], 2)
            sc = bsa.antidiagonal_block_scores(qp, kp, 128, 16)
            new = bsa.top_p_block_mask(sc, torch.from_numpy(tau))
            new_g = new.cpu().numpy().astype(bool)
            for h in heads:
                sc_ref = oracle.antidiagonal_block_scores(qp[:, h:h + 1].double().cpu().numpy(),
                                                          kp[:, h:h + 1].double().cpu().numpy(),
                                                          128, 16)
                m_h, tie = oracle.top_p_block_mask(sc_ref, tau[h:h + 1])
                new_ref[0, h] = m_h[0, 0]
                tie_rows[h] = tie[0, 0]
                bad = (new_g[0, h] != m_h[0, 0]).any(-1) & ~tie[0, 0]
                assert not bad.any(), (t, h, np.nonzero(bad))
        m = cache.update(new)
        m_ref = ref.update(new_ref, r_ref)
        mg = m.cpu().numpy().astype(bool)
        out = bsa.centroid_compensated_attention(q, k, v, lt, lt, m)
        out_h = out[0, heads].cpu().numpy()
        for i, h in enumerate(heads):
            diff = (mg[0, h] != m_ref[0, h]).any(-1)
            assert not (diff & ~tie_rows[h]).any()
            rows = rng.choice(S, 64, replace=False)
            rows = np.sort(rows[~diff[lab[rows]]])
            o_ref = oracle.centroid_compensated_attention(
                q[:, h:h + 1].double().cpu().numpy(), k[:, h:h + 1].double().cpu().numpy(),
                v[:, h:h + 1].double().cpu().numpy(), lab, lab, m_ref[:, h:h + 1], rows=rows,
                Cq=C, Ck=C)
            got = out_h[i][rows]
            assert np.abs(got - o_ref[0, 0]).max() <= 2e-2
            assert np.linalg.norm(got - o_ref[0, 0]) / np.linalg.norm(o_ref[0, 0]) <= 5e-3
    # the recipe's expected behaviour: only the first cached step refreshes (the pooled
    # drift stays far below delta, and 4 of 40 heads are under the gate's 40 %)
    assert n_refresh_steps == 1
    assert bsa.device_status()[0] == 0
