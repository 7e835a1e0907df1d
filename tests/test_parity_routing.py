"""GPU parity: SVG-EAR error-aware routing vs the oracle ("Sparse-block compensation",
§SVG-EAR — centroid compensation; the SVG-EAR abstract: a probe estimates each block's
compensation error and the highest error-to-cost blocks are computed exactly).

Protocol (as for top-p): the block errors are compared at a tolerance (fp32 with fast
exponentials against float64); the selection, an exact function of the errors, is
compared bit for bit with the oracle's selection applied to the GPU's own float32
errors; against the oracle's float64 chain, masks may differ only on blocks whose
ratio lies at the selection's cutoff within the error tolerance.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 2e-3


def _bsa():
    import block_sparse_attention_tcgen05_b200 as bsa
    return bsa


def _route(q, k, v, ql, kl, Cq, Ck, density):
    bsa = _bsa()
    mask, err = bsa.error_aware_block_mask(
        q.cuda(), k.cuda(), v.cuda(), torch.as_tensor(ql, dtype=torch.int32).cuda(),
        torch.as_tensor(kl, dtype=torch.int32).cuda(), Cq, Ck, density, return_err=True)
    torch.cuda.synchronize()
    assert bsa.device_status()[0] == 0
    return mask.cpu().numpy().astype(bool), err.cpu().numpy()


def _check_errors(err, ref):
    scale = max(float(np.abs(ref).max()), 1e-30)
    assert np.abs(err - ref).max() <= ERR_RTOL * scale, np.abs(err - ref).max() / scale


def _check_chain(mask, ref_mask, ref_err, ql, kl, Cq, Ck):
    """Blocks where the GPU mask and the float64 chain differ must sit at the cutoff."""
    nk = np.bincount(kl, minlength=Ck)
    nq = np.bincount(ql, minlength=Cq)
    for b in range(mask.shape[0]):
        for h in range(mask.shape[1]):
            diff = mask[b, h] != ref_mask[b, h]
            if not diff.any():
                continue
            ratio = ref_err[b, h] / np.maximum(nk, 1)[None, :]
            valid = (nq[:, None] > 0) & (nk[None, :] > 0)
            kept = ref_mask[b, h] & valid
            cut = ratio[kept].min() if kept.any() else ratio[valid].max()
            assert (np.abs(ratio[diff] - cut) <= 2 * ERR_RTOL * max(cut, ratio[valid].max() * 1e-6)).all()


@pytest.mark.parametrize("dtype,D,Hq,Hkv", [("bf16", 128, 4, 2), ("f32", 64, 2, 2), ("bf16", 64, 3, 1)])
def test_routing_small_uneven_clusters(dtype, D, Hq, Hkv):
    """S = 900 with shuffled uneven clusters, an empty key cluster and an empty query
    cluster, Cq != Ck; densities 0.15 and 0.5."""
    g = np.random.default_rng(31)
    S, Cq, Ck = 900, 11, 14
    ql = g.permutation(np.concatenate([np.arange(Cq - 1), g.integers(0, Cq - 1, S - Cq + 1)]))
    kl = g.permutation(np.concatenate([np.arange(Ck - 1), g.integers(0, Ck - 1, S - Ck + 1)]))
    kl = np.where(kl == 5, Ck - 1, kl)   # key cluster 5 empty, Ck - 1 takes its rows
    q, k, v = wl.gaussian_qkv(1, Hq, Hkv, S, D, dtype, seed=32)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    ref_err = oracle.compensation_errors(qd, kd, vd, ql, kl, Cq, Ck)
    for density in (0.15, 0.5):
        mask, err = _route(q, k, v, ql, kl, Cq, Ck, density)
        _check_errors(err, ref_err)
        same = oracle.route_blocks(err, ql, kl, Cq, Ck, np.float32(density), dtype=np.float32)
        np.testing.assert_array_equal(mask, same)
        ref_mask = oracle.route_blocks(ref_err, ql, kl, Cq, Ck, np.float32(density))
        _check_chain(mask, ref_mask, ref_err, ql, kl, Cq, Ck)
        assert not mask[:, :, Cq - 1].any() and not mask[:, :, :, 5].any()


def test_routing_large_clusters_two_probe_tiles():
    """Key clusters of several hundred keys (several 128-key pieces each, so the running
    reference moves between pieces), 200 query clusters (two 128-probe tiles, the second
    partly padding), GQA 4 over 2 KV heads, bf16 D=128; density 0.3."""
    g = np.random.default_rng(41)
    S, Cq, Ck = 2400, 200, 5
    ql = g.permutation(np.concatenate([np.arange(Cq), g.integers(0, Cq, S - Cq)]))
    kl = np.sort(g.integers(0, Ck, S))
    kl[:Ck] = np.arange(Ck)
    kl = g.permutation(kl)
    q, k, v = wl.gaussian_qkv(1, 4, 2, S, 128, "bf16", seed=42)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    ref_err = oracle.compensation_errors(qd, kd, vd, ql, kl, Cq, Ck)
    mask, err = _route(q, k, v, ql, kl, Cq, Ck, 0.3)
    _check_errors(err, ref_err)
    same = oracle.route_blocks(err, ql, kl, Cq, Ck, np.float32(0.3), dtype=np.float32)
    np.testing.assert_array_equal(mask, same)
    ref_mask = oracle.route_blocks(ref_err, ql, kl, Cq, Ck, np.float32(0.3))
    _check_chain(mask, ref_mask, ref_err, ql, kl, Cq, Ck)


def test_routing_density_edges():
    """Density 1 keeps every block of non-empty clusters, density 0 none."""
    q, k, v = wl.gaussian_qkv(1, 2, 2, 512, 64, "bf16", seed=33)
    lab = np.arange(512) // 64
    m1, _ = _route(q, k, v, lab, lab, 8, 8, 1.0)
    m0, _ = _route(q, k, v, lab, lab, 8, 8, 0.0)
    assert m1.all() and not m0.any()


def test_routing_video_static_then_attention():
    """Video shape (21x30x52 grid, 3x6x8 tiles, 245 clusters, D=128 bf16), 8 heads,
    density 0.22: block errors of two heads against the oracle, the selection bit for
    bit on the GPU's errors, then the compensated attention on the routed mask against
    the oracle on sampled rows (router and attention end to end)."""
    bsa = _bsa()
    grid, tile = (21, 30, 52), (3, 6, 8)
    q, k, v, _ = wl.positional_qkv(1, 8, 8, grid, 128, ell=(3.0, 6.0, 8.0), amp=2.0,
                                   dtype="bf16", seed=3)
    lab, C = oracle.tile_labels(*grid, tile)
    mask, err = _route(q, k, v, lab, lab, C, C, 0.22)
    same = oracle.route_blocks(err, lab, lab, C, C, np.float32(0.22), dtype=np.float32)
    np.testing.assert_array_equal(mask, same)
    cnt = np.bincount(lab, minlength=C)
    dens = [(cnt @ mask[0, h] @ cnt) / 32760 ** 2 for h in range(8)]
    assert all(0.2 < d <= 0.22 for d in dens), dens
    for h in (0, 5):
        ref = oracle.compensation_errors(q[:, h:h + 1].double().numpy(), k[:, h:h + 1].double().numpy(),
                                         v[:, h:h + 1].double().numpy(), lab, lab, C, C)
        _check_errors(err[:, h:h + 1], ref)
    lt = torch.as_tensor(lab, dtype=torch.int32).cuda()
    out = bsa.centroid_compensated_attention(q.cuda(), k.cuda(), v.cuda(), lt, lt,
                                             torch.from_numpy(mask.astype(np.uint8)).cuda())
    got = out.cpu().numpy()
    rows = np.sort(np.random.default_rng(34).choice(32760, 128, replace=False))
    heads = [0, 5]
    ref = oracle.centroid_compensated_attention(
        q[:, heads].double().numpy(), k[:, heads].double().numpy(), v[:, heads].double().numpy(),
        lab, lab, mask[:, heads], rows=rows, Cq=C, Ck=C)
    g = got[:, heads][:, :, rows]
    assert np.abs(g - ref).max() <= 2e-2
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3
    assert bsa.device_status()[0] == 0


@pytest.mark.parametrize("dtype,D,Hq,Hkv", [("bf16", 128, 6, 2), ("f32", 64, 2, 2)])
def test_probe_budget_router(dtype, D, Hq, Hkv):
    """SparsePR's router ("Partition the Support, Reconstruct the Residual": the router
    reserves the probe cost first): cell masses against the oracle at a tolerance, and
    the mask bit for bit against the oracle's budgeted prefix on the GPU's own masses with
    the routing density max(0, density - M / Sq)."""
    bsa = _bsa()
    g = np.random.default_rng(35)
    S, Cq, Ck, M = 2048, 16, 16, 64
    ql = g.permutation(np.arange(S) % Cq)
    kl = g.permutation(np.concatenate([np.arange(Ck - 1), g.integers(0, Ck - 1, S - Ck + 1)]))
    q, k, _ = wl.gaussian_qkv(1, Hq, Hkv, S, D, dtype, seed=36)
    ref_mass = oracle.centroid_mass(q.double().numpy(), k.double().numpy(), ql, kl, Cq, Ck)
    for density in (0.22, 0.5, 0.02):
        mask, mass = bsa.probe_budget_block_mask(
            q.cuda(), k.cuda(), torch.as_tensor(ql, dtype=torch.int32).cuda(),
            torch.as_tensor(kl, dtype=torch.int32).cuda(), Cq, Ck, density, M, return_mass=True)
        mask, mass = mask.cpu().numpy().astype(bool), mass.cpu().numpy()
        assert np.abs(mass - ref_mass).max() <= 1e-4
        route = max(0.0, float(np.float32(density)) - M / S)
        same = oracle.route_blocks(mass, ql, kl, Cq, Ck, route, dtype=np.float32)
        np.testing.assert_array_equal(mask, same)
        nq, nk = np.bincount(ql, minlength=Cq), np.bincount(kl, minlength=Ck)
        pairs = [(nq[:, None] * nk[None, :])[mask[0, h]].sum() for h in range(Hq)]
        assert max(pairs) + M * S <= max(density * S * S, M * S)
    assert bsa.device_status()[0] == 0
