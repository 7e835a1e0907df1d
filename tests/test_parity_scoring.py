"""GPU parity: anti-diagonal block scores and top-p masks vs the oracle."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SCORE_ATOL = 1e-4   # fp32 accumulation of bf16 products vs float64 on the same values


def _bsa():
    import block_sparse_attention_tcgen05_b200 as bsa
    return bsa


def _scores(q, k, block, stride):
    bsa = _bsa()
    sc = bsa.antidiagonal_block_scores(q.cuda(), k.cuda(), block=block, stride=stride)
    torch.cuda.synchronize()
    assert bsa.device_status()[0] == 0
    return sc.cpu().numpy()


@pytest.mark.parametrize("D,stride,block", [(64, 16, 128), (128, 16, 128), (64, 8, 64), (128, 4, 128)])
def test_scores_small(D, stride, block):
    S = 128 * stride * 2  # two strided query tiles
    q, k, _ = wl.gaussian_qkv(1, 2, 2, S, D, "bf16", seed=D + stride)
    got = _scores(q, k, block, stride)
    ref = oracle.antidiagonal_block_scores(q.double().numpy(), k.double().numpy(), block, stride)
    np.testing.assert_allclose(got, ref, atol=SCORE_ATOL, rtol=0)
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-4)


def test_scores_gqa():
    q, k, _ = wl.gaussian_qkv(1, 4, 2, 4096, 64, "bf16", seed=5)
    got = _scores(q, k, 128, 16)
    ref = oracle.antidiagonal_block_scores(q.double().numpy(), k.double().numpy(), 128, 16)
    np.testing.assert_allclose(got, ref, atol=SCORE_ATOL, rtol=0)


@pytest.mark.parametrize("S,D,stride,block", [
    (40960, 64, 16, 128),   # 2560 strided rows: more than one pass's 2048
    (32768, 128, 16, 64),   # 512 key blocks: more than one pass's 256
])
def test_scores_two_pass_long_sequences(S, D, stride, block):
    """Sequences past the one-pass limits take the two-pass path (row statistics first,
    then normalised block sums); same oracle, same tolerance, rows sum to 1."""
    q, k, _ = wl.gaussian_qkv(1, 2, 1, S, D, "bf16", seed=S % 97 + D)
    got = _scores(q, k, block, stride)
    ref = oracle.antidiagonal_block_scores(q.double().numpy(), k.double().numpy(), block, stride)
    np.testing.assert_allclose(got, ref, atol=SCORE_ATOL, rtol=0)
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-4)


def test_top_p_kernel_bit_exact_on_identical_scores():
    """Same float32 scores on both sides, decisions in float32 in the same order."""
    g = np.random.default_rng(0)
    sc = g.dirichlet(np.ones(64) * 0.3, size=(2, 3, 64)).astype(np.float32)
    tau = np.array([0.85, 0.9, 0.95], dtype=np.float32)
    bsa = _bsa()
    got, ties = bsa.top_p_block_mask(torch.from_numpy(sc).cuda(), torch.from_numpy(tau),
                                     return_ties=True)
    ref, ref_tie = oracle.top_p_block_mask(sc, tau, dtype=np.float32)
    np.testing.assert_array_equal(got.cpu().numpy().astype(bool), ref)
    np.testing.assert_array_equal(ties.cpu().numpy().astype(bool), ref_tie)
    # ragged Nk (not a power of two), scalar tau
    sc2 = g.dirichlet(np.ones(245), size=(1, 2, 7)).astype(np.float32)
    got2 = bsa.top_p_block_mask(torch.from_numpy(sc2).cuda(), 0.9)
    ref2, _ = oracle.top_p_block_mask(sc2, 0.9, dtype=np.float32)
    np.testing.assert_array_equal(got2.cpu().numpy().astype(bool), ref2)
    assert (got2.cpu().numpy().sum(-1) >= 1).all()
    # degenerate tau: a tiny tau keeps the arg-max block only; tau = 1 keeps every block
    # up to the first running sum reaching 1 (the whole row when rounding stays below 1)
    for t in (1e-7, 1.0):
        got3 = bsa.top_p_block_mask(torch.from_numpy(sc).cuda(), t).cpu().numpy().astype(bool)
        ref3, _ = oracle.top_p_block_mask(sc, t, dtype=np.float32)
        np.testing.assert_array_equal(got3, ref3)
        if t < 1e-3:
            assert (got3.sum(-1) == 1).all()
            np.testing.assert_array_equal(got3.argmax(-1), sc.argmax(-1))


def test_top_p_tie_rows_reported():
    """Rows built so that a decision is fragile: a running sum landing within 1e-5 of
    tau, and a last kept score within 1e-5 of the first dropped one. The kernel's tie
    flags equal the oracle's (float32 running sums on both sides) bit for bit, and so
    do the masks."""
    rows = np.array([
        [0.5, 0.4, 0.1, 0.0],               # running sum 0.9 at rank 1: |0.9 - tau| = 0
        [0.5, 0.399995, 0.100005, 0.0],     # 0.899995: within 1e-5 below tau
        [0.5, 0.40002, 0.09998, 0.0],       # 0.90002: 2e-5 past tau, no tie
        [0.6, 0.200005, 0.2, -0.0],         # kept 0.200005 vs dropped 0.2: gap 5e-6
        [0.6, 0.21, 0.19, 0.0],             # gap 0.02, running sums far from tau: no tie
        [0.25, 0.25, 0.25, 0.25],           # equal scores: index order decides
    ], dtype=np.float32)
    taus = np.array([0.9, 0.9, 0.9, 0.7, 0.7, 0.6], dtype=np.float32)
    bsa = _bsa()
    for r, t in zip(rows, taus):
        sc = np.abs(r)[None, None, None, :]
        got, ties = bsa.top_p_block_mask(torch.from_numpy(sc).cuda(), float(t), return_ties=True)
        ref, ref_tie = oracle.top_p_block_mask(sc, float(t), dtype=np.float32)
        np.testing.assert_array_equal(got.cpu().numpy().astype(bool), ref)
        np.testing.assert_array_equal(ties.cpu().numpy().astype(bool), ref_tie)
    want = [True, True, False, True, False, True]
    got_all = []
    for r, t in zip(rows, taus):
        _, tie = oracle.top_p_block_mask(np.abs(r)[None, None, None, :], float(t), dtype=np.float32)
        got_all.append(bool(tie.reshape(-1)[0]))
    assert got_all == want, got_all


def test_dynamic_mask_workload_scores_and_masks():
    """B=1, H=8, S=8192, D=64 bf16 with 1-D positional structure; block 128, stride 16,
    tau 0.9. Masks must match the float64 oracle chain bit for bit outside tie rows."""
    bsa = _bsa()
    q, k, _, _ = wl.positional_qkv(1, 8, 8, (8192,), 64, ell=(256.0,), amp=2.0, dtype="bf16",
                                   seed=2)
    got = _scores(q, k, 128, 16)
    ref = oracle.antidiagonal_block_scores(q.double().numpy(), k.double().numpy(), 128, 16)
    np.testing.assert_allclose(got, ref, atol=SCORE_ATOL, rtol=0)
    m_gpu_t, ties_gpu = bsa.top_p_block_mask(torch.from_numpy(got).cuda(), 0.9, return_ties=True)
    m_gpu = m_gpu_t.cpu().numpy().astype(bool)
    # on the GPU's own scores, decided in float32 on both sides: masks and tie flags
    # bit for bit
    m32, tie32 = oracle.top_p_block_mask(got, 0.9, dtype=np.float32)
    np.testing.assert_array_equal(m_gpu, m32)
    np.testing.assert_array_equal(ties_gpu.cpu().numpy().astype(bool), tie32)
    m_ref, tie = oracle.top_p_block_mask(ref, 0.9)
    diff_rows = (m_gpu != m_ref).any(-1)
    assert not (diff_rows & ~tie).any(), f"{int((diff_rows & ~tie).sum())} non-tie rows differ"
    print(f"tie rows {int(tie.sum())}, differing rows {int(diff_rows.sum())}, density "
          f"{m_gpu.mean():.3f}")
    # the chain's last step: compensated attention on the top-p mask, labels arange // 128;
    # sampled rows against the oracle's attention on the oracle's own mask (rows of query
    # blocks whose masks differ, tie rows only, are left out)
    _, _, v, _ = wl.positional_qkv(1, 8, 8, (8192,), 64, ell=(256.0,), amp=2.0, dtype="bf16",
                                   seed=2)
    lab = np.arange(8192) // 128
    lt = torch.as_tensor(lab, dtype=torch.int32).cuda()
    out = bsa.centroid_compensated_attention(q.cuda(), k.cuda(), v.cuda(), lt, lt,
                                             torch.from_numpy(m_gpu.astype(np.uint8)).cuda())
    got = out.cpu().numpy()
    rows = np.sort(np.random.default_rng(21).choice(8192, 512, replace=False))
    ref_o = oracle.centroid_compensated_attention(q.double().numpy(), k.double().numpy(),
                                                  v.double().numpy(), lab, lab, m_ref, rows=rows,
                                                  Cq=64, Ck=64)
    for h in range(8):
        keep = ~diff_rows[0, h][lab[rows]]
        g_h, r_h = got[0, h, rows[keep]], ref_o[0, h, keep]
        assert np.abs(g_h - r_h).max() <= 2e-2
        assert np.linalg.norm(g_h - r_h) / np.linalg.norm(r_h) <= 5e-3
    assert bsa.device_status()[0] == 0


def test_video_reuse_workload_scores_sampled_heads():
    """B=1, H=40, S=32760 padded to 32768 (XAttention pads with zeros), D=128, block 128,
    stride 16; heads 0 and 39 against the oracle."""
    grid = (21, 30, 52)
    q, k, _, _ = wl.positional_qkv(1, 40, 40, grid, 128, ell=(3.0, 6.0, 8.0), amp=2.0,
                                   dtype="bf16", seed=5)
    pad = torch.zeros(1, 40, 8, 128, dtype=torch.bfloat16)
    qp = torch.cat([q, pad], 2).contiguous()
    kp = torch.cat([k, pad], 2).contiguous()
    got = _scores(qp, kp, 128, 16)
    assert got.shape == (1, 40, 256, 256)
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-4)
    for h in (0, 39):
        ref = oracle.antidiagonal_block_scores(qp[:, h:h + 1].double().numpy(),
                                               kp[:, h:h + 1].double().numpy(), 128, 16)
        np.testing.assert_allclose(got[:, h:h + 1], ref, atol=SCORE_ATOL, rtol=0)
