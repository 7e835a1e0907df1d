"""GPU parity: libbsa centroid-compensated / hard-drop attention vs the float64 oracle.

Tolerances (bf16 or fp32 inputs, fp32 accumulation): max-abs error <= 2e-2 and
relative Frobenius error <= 5e-3 against the oracle on the same input values.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_FRO = 5e-3


def _bsa():
    import block_sparse_attention_tcgen05_b200 as bsa
    return bsa


def _check(got, ref, max_abs=MAX_ABS, rel=REL_FRO):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.isfinite(got).all()
    assert err.max() <= max_abs, f"max-abs {err.max():.3e}"
    assert fro <= rel, f"rel-fro {fro:.3e}"
    return err.max(), fro


def _run(q, k, v, ql, kl, mask, Cq, Ck, compensate=True):
    bsa = _bsa()
    dev = torch.device("cuda")
    out = bsa.centroid_compensated_attention(
        q.to(dev), k.to(dev), v.to(dev), torch.as_tensor(ql, dtype=torch.int32, device=dev),
        torch.as_tensor(kl, dtype=torch.int32, device=dev),
        torch.as_tensor(np.asarray(mask), dtype=torch.uint8, device=dev), Cq=Cq, Ck=Ck,
        compensate=compensate)
    torch.cuda.synchronize()
    assert bsa.device_status()[0] == 0
    return out.cpu().numpy()


def _ref(q, k, v, ql, kl, mask, Cq, Ck, compensate=True, rows=None):
    return oracle.centroid_compensated_attention(
        q.double().numpy(), k.double().numpy(), v.double().numpy(), ql, kl, mask,
        compensate=compensate, rows=rows, Cq=Cq, Ck=Ck)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("compensate", [True, False])
def test_tiny_workload(dtype, compensate):
    """B=1, H=2, S=1024, D=64, labels arange//64, 25 % random cluster mask (diagonal
    kept, seed 0)."""
    q, k, v = wl.gaussian_qkv(1, 2, 2, 1024, 64, dtype, seed=0)
    lab = np.arange(1024) // 64
    mask = wl.random_cluster_mask(16, 0.25, seed=0)
    got = _run(q, k, v, lab, lab, mask, 16, 16, compensate)
    _check(got, _ref(q, k, v, lab, lab, mask, 16, 16, compensate))


@pytest.mark.parametrize("D", [64, 128])
def test_ragged_uneven_clusters_gqa_per_head_mask(D):
    """S not a multiple of 128, shuffled labels with uneven sizes (some not multiples
    of 16), Cq != Ck, an empty key cluster, per-head masks, GQA 4:2."""
    g = np.random.default_rng(1)
    S, Cq, Ck = 1000, 11, 13
    ql = g.permutation(np.concatenate([np.arange(Cq), g.integers(0, Cq, S - Cq)]))
    kl = g.permutation(np.concatenate([np.arange(Ck - 1), g.integers(0, Ck - 1, S - Ck + 1)]))
    mask = g.random((4, Cq, Ck)) < 0.3
    q, k, v = wl.gaussian_qkv(1, 4, 2, S, D, "bf16", seed=2)
    for comp in (True, False):
        got = _run(q, k, v, ql, kl, mask, Cq, Ck, comp)
        _check(got, _ref(q, k, v, ql, kl, mask, Cq, Ck, comp))


def test_one_key_per_cluster_equals_dense():
    q, k, v = wl.gaussian_qkv(1, 2, 2, 384, 64, "bf16", seed=3)
    ql = np.arange(384) // 128
    kl = np.random.default_rng(4).permutation(384)
    mask = np.random.default_rng(5).random((3, 384)) < 0.2
    got = _run(q, k, v, ql, kl, mask, 3, 384)
    dense = oracle.dense_attention(q.double().numpy(), k.double().numpy(), v.double().numpy())
    _check(got, dense)


def test_all_kept_equals_dense_and_batch():
    q, k, v = wl.gaussian_qkv(2, 2, 1, 640, 128, "bf16", seed=6)
    lab = np.arange(640) // 80
    mask = np.ones((8, 8), dtype=bool)
    for comp in (True, False):
        got = _run(q, k, v, lab, lab, mask, 8, 8, comp)
        _check(got, oracle.dense_attention(q.double().numpy(), k.double().numpy(),
                                           v.double().numpy()))


def test_all_skipped_rows_hard_drop_zero():
    q, k, v = wl.gaussian_qkv(1, 1, 1, 256, 64, "bf16", seed=7)
    lab = np.arange(256) // 64
    mask = np.eye(4, dtype=bool)
    mask[2, 2] = False  # query cluster 2 keeps nothing
    got = _run(q, k, v, lab, lab, mask, 4, 4, compensate=False)
    assert np.abs(got[0, 0, 128:192]).max() == 0.0
    _check(got, _ref(q, k, v, lab, lab, mask, 4, 4, False))
    got = _run(q, k, v, lab, lab, mask, 4, 4, compensate=True)
    _check(got, _ref(q, k, v, lab, lab, mask, 4, 4, True))


def test_dynamic_mask_workload_shape():
    """B=1, H=8, S=8192, D=64 bf16 with 1-D positional structure; block labels
    arange//128; a random per-head block mask at ~20 % with the diagonal kept."""
    q, k, v, _ = wl.positional_qkv(1, 8, 8, (8192,), 64, ell=(256.0,), amp=2.0, dtype="bf16",
                                   seed=2)
    lab = np.arange(8192) // 128
    mask = np.stack([wl.random_cluster_mask(64, 0.2, seed=10 + h) for h in range(8)])
    rows = np.random.default_rng(11).choice(8192, 512, replace=False)
    got = _run(q, k, v, lab, lab, mask, 64, 64)
    ref = _ref(q, k, v, lab, lab, mask, 64, 64, rows=rows)
    _check(got[:, :, rows], ref)


def test_video_static_tiles_full_size_sampled():
    """B=1, H=40, S=32760 (21x30x52), D=128, 3x6x8 tiles (245 clusters of 144 / 72
    tokens), nearest-22 % tile-pair mask; sampled rows of every head vs the oracle."""
    bsa = _bsa()
    grid, tile = (21, 30, 52), (3, 6, 8)
    q, k, v, _ = wl.positional_qkv(1, 40, 40, grid, 128, ell=(3.0, 6.0, 8.0), amp=2.0,
                                   dtype="bf16", seed=3)
    labels_gpu, C = bsa.tile_labels(*grid, tile)
    lab_ref, C_ref = oracle.tile_labels(*grid, tile)
    assert C == C_ref == 245
    np.testing.assert_array_equal(labels_gpu.cpu().numpy(), lab_ref)
    mask = wl.nearest_pair_mask(wl.tile_centroids(grid, tile), 0.22)
    got = _run(q, k, v, lab_ref, lab_ref, mask, C, C)
    rows = np.random.default_rng(12).choice(32760, 96, replace=False)
    ref = _ref(q, k, v, lab_ref, lab_ref, mask, C, C, rows=rows)
    _check(got[:, :, rows], ref)
    # Coverage: one row in every 128-row query tile of the cluster-sorted order the
    # kernel walks (tokens stably sorted by label), and one row of every cluster (the
    # 35 partial 72-token edge tiles included), on four heads.
    g = np.random.default_rng(13)
    order = np.argsort(lab_ref, kind="stable")
    cover = {int(order[t * 128 + g.integers(0, min(128, 32760 - t * 128))])
             for t in range(-(-32760 // 128))}
    for c in range(C):
        cover.add(int(g.choice(np.nonzero(lab_ref == c)[0])))
    cover = np.array(sorted(cover))
    heads = [0, 13, 26, 39]
    qh, kh, vh = (t[:, heads] for t in (q, k, v))
    ref = _ref(qh, kh, vh, lab_ref, lab_ref, mask, C, C, rows=cover)
    _check(got[:, heads][:, :, cover], ref)


# Calls with at least 148 query-tile CTAs over all heads run without a key-range split
# (one CTA walks every kept key of its tile); the cases below reach that path with short
# sequences and many heads.

@pytest.mark.parametrize("D", [64, 128])
def test_unsplit_ragged_gqa(D):
    """S = 1100 (9 query tiles, the last one ragged), shuffled uneven clusters
    (sizes not multiples of 16), an empty key cluster, Cq != Ck, per-head masks at
    ~30 %, GQA 40:20; compensated and hard drop."""
    g = np.random.default_rng(21)
    S, Cq, Ck, H, Hkv = 1100, 13, 17, 40, 20
    ql = g.permutation(np.concatenate([np.arange(Cq), g.integers(0, Cq, S - Cq)]))
    kl = g.permutation(np.concatenate([np.arange(Ck - 1), g.integers(0, Ck - 1, S - Ck + 1)]))
    mask = g.random((H, Cq, Ck)) < 0.3
    q, k, v = wl.gaussian_qkv(1, H, Hkv, S, D, "bf16", seed=22)
    rows = np.sort(g.choice(S, 160, replace=False))
    for comp in (True, False):
        got = _run(q, k, v, ql, kl, mask, Cq, Ck, comp)
        _check(got[:, :, rows], _ref(q, k, v, ql, kl, mask, Cq, Ck, comp, rows=rows))


def test_unsplit_all_kept_equals_dense():
    """Every block kept over many 128-key chunks: equals dense attention."""
    q, k, v = wl.gaussian_qkv(1, 48, 48, 896, 128, "bf16", seed=23)
    lab = np.arange(896) // 112
    mask = np.ones((8, 8), dtype=bool)
    got = _run(q, k, v, lab, lab, mask, 8, 8, True)
    _check(got, oracle.dense_attention(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy()))


def test_unsplit_large_logit_jumps():
    """Keys 64..127 of every 128 have 20x larger logits, so the running max jumps by far
    more than the lazy-rescale threshold between the two halves of a chunk."""
    g = np.random.default_rng(24)
    S, H, D = 1024, 40, 64
    q = torch.tensor(g.standard_normal((1, H, S, D)) * 0.5, dtype=torch.float64)
    k = torch.tensor(g.standard_normal((1, H, S, D)) * 0.5, dtype=torch.float64)
    # keys 64..127 of every 128 are 20x larger: the second half of a chunk raises the
    # max by far more than the lazy-rescale threshold
    k = k * torch.tensor(1.0 + 19.0 * ((np.arange(S) % 128) >= 64))[None, None, :, None]
    v = torch.tensor(g.standard_normal((1, H, S, D)), dtype=torch.float64)
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    lab = np.arange(S) // 128
    mask = np.random.default_rng(25).random((8, 8)) < 0.6
    np.fill_diagonal(mask, True)
    for comp in (True, False):
        got = _run(q, k, v, lab, lab, mask, 8, 8, comp)
        ref = _ref(q.float(), k.float(), v.float(), lab, lab, mask, 8, 8, comp)
        _check(got, ref)


def test_key_range_at_one_window():
    """Sk + 15 Ck = 65536: 4096 key groups, the size of one CTA's bitset window, here
    taken as two key ranges. 16 clusters of ~4081 tokens (none a multiple of 16), a
    random mask with the diagonal kept; compensated and hard drop; sampled rows vs the
    oracle."""
    S, C = 65536 - 15 * 16, 16
    q, k, v = wl.gaussian_qkv(1, 1, 1, S, 64, "bf16", seed=41)
    lab = (np.arange(S) * C) // S
    mask = wl.random_cluster_mask(C, 0.4, seed=42)
    rows = np.sort(np.random.default_rng(43).choice(S, 96, replace=False))
    for comp in (True, False):
        got = _run(q, k, v, lab, lab, mask, C, C, comp)
        _check(got[:, :, rows], _ref(q, k, v, lab, lab, mask, C, C, comp, rows=rows))


def test_long_key_sequence_split_into_windows():
    """S = 81920 (a long video latent, past one window of 4096 key groups): the key
    groups are split into ranges of at most 4096 per CTA, merged afterwards. 20 clusters
    of 4096 tokens, a random mask with the diagonal kept; compensated and hard drop;
    sampled rows vs the oracle."""
    S, C = 81920, 20
    q, k, v = wl.gaussian_qkv(1, 1, 1, S, 64, "bf16", seed=61)
    lab = (np.arange(S) * C) // S
    mask = wl.random_cluster_mask(C, 0.3, seed=62)
    rows = np.sort(np.random.default_rng(63).choice(S, 96, replace=False))
    for comp in (True, False):
        got = _run(q, k, v, lab, lab, mask, C, C, comp)
        _check(got[:, :, rows], _ref(q, k, v, lab, lab, mask, C, C, comp, rows=rows))


@pytest.mark.parametrize("H,Hkv", [(40, 10), (2, 1)])
def test_per_batch_and_head_masks(H, Hkv):
    """B=2 with a different mask for every (batch, head) (batch and head mask strides),
    grouped-query heads, shuffled uneven clusters; 40 heads run without a key split,
    2 heads with one; compensated and hard drop."""
    g = np.random.default_rng(51)
    B, S, Cq, Ck = 2, 640, 7, 9
    ql = g.permutation(np.concatenate([np.arange(Cq), g.integers(0, Cq, S - Cq)]))
    kl = g.permutation(np.concatenate([np.arange(Ck), g.integers(0, Ck, S - Ck)]))
    mask = g.random((B, H, Cq, Ck)) < 0.35
    q, k, v = wl.gaussian_qkv(B, H, Hkv, S, 64, "bf16", seed=52)
    rows = np.sort(g.choice(S, 128, replace=False))
    for comp in (True, False):
        got = _run(q, k, v, ql, kl, mask, Cq, Ck, comp)
        _check(got[:, :, rows], _ref(q, k, v, ql, kl, mask, Cq, Ck, comp, rows=rows))


def test_plan_reuse_with_new_qkv():
    """A call that reuses the label sorts, key order, tile plan and bitsets of the previous
    call on the same workspace ("Dynamic block masks and head-wise mask reuse": masks and
    the token grid fixed across denoising steps) with new Q, K, V: bit-identical to a
    fresh call on those values, and within tolerance of the oracle. Video-grid tiles
    (72- and 144-token clusters), per-head masks, GQA, bf16 D=128."""
    bsa = _bsa()
    dev = torch.device("cuda")
    grid, tile = (3, 12, 20), (3, 6, 8)
    lab, C = oracle.tile_labels(*grid, tile)
    S = int(np.prod(grid))
    g = np.random.default_rng(51)
    mask = g.random((4, C, C)) < 0.4
    mask[:, np.arange(C), np.arange(C)] = True
    lt = torch.as_tensor(lab, dtype=torch.int32, device=dev)
    mt = torch.as_tensor(mask, dtype=torch.uint8, device=dev)
    q0, k0, v0 = (t.to(dev) for t in wl.gaussian_qkv(1, 4, 2, S, 128, "bf16", seed=52))
    q1, k1, v1 = wl.gaussian_qkv(1, 4, 2, S, 128, "bf16", seed=53)
    ws = torch.empty(bsa.attention_workspace_bytes(q0, k0, C, C), dtype=torch.uint8, device=dev)
    bsa.centroid_compensated_attention(q0, k0, v0, lt, lt, mt, Cq=C, Ck=C, workspace=ws)
    reused = bsa.centroid_compensated_attention(q1.to(dev), k1.to(dev), v1.to(dev), lt, lt, mt,
                                                Cq=C, Ck=C, workspace=ws, reuse_plan=True)
    fresh = bsa.centroid_compensated_attention(q1.to(dev), k1.to(dev), v1.to(dev), lt, lt, mt,
                                               Cq=C, Ck=C)
    torch.cuda.synchronize()
    assert bsa.device_status()[0] == 0
    assert torch.equal(reused, fresh)
    _check(reused.cpu().numpy(), _ref(q1, k1, v1, lab, lab, mask[None], C, C))
