"""Oracle: SparsePR probe selection and probe-fitted residual repair.

Test infrastructure only (see the package docstring).

Sources: "Sparse-block compensation", §SparsePR — probe-fitted residual repair,
§What mlx-arsenal ships (``select_probe_rows``), §Recipe, §Deviations from the papers
(middle-out member, weights normalised to sum 1); "Partition the Support,
Reconstruct the Residual", §Probe-Fitted Residual Reconstruction (M = 64 exact rows,
ridge λ = 0.1, projection on the r = 16 residual subspace, probes stratified across
query groups and ordered by distance to the group centroid, weights |G_a| / m_a).
"""

import numpy as np

from .attention import dense_attention


def _middle_out(n):
    """Member order of a cluster of n rows sorted by index: by |r − (n−1)/2|
    ascending, ties to the lower r (reading of "middle-out member")."""
    r = np.arange(n)
    return sorted(range(n), key=lambda i: (abs(2 * i - (n - 1)), i))


def _round_robin(members, M):
    """Stratify M probes across clusters.

    ``members`` lists, per non-empty cluster in ascending label order, its rows in
    preference order. Reading of "round-robin over query clusters": if M is at
    least the number of clusters C, pass p takes the p-th preferred row of every
    cluster that still has one, until M rows are taken; if M < C, probe i comes
    from cluster floor(i·C / M) (its first preferred row).
    Returns (rows (M,), cluster index of each probe (M,)).
    """
    C = len(members)
    rows, owner = [], []
    if M < C:
        for i in range(M):
            a = (i * C) // M
            rows.append(members[a][0])
            owner.append(a)
    else:
        p = 0
        while len(rows) < M:
            took = False
            for a in range(C):
                if p < len(members[a]) and len(rows) < M:
                    rows.append(members[a][p])
                    owner.append(a)
                    took = True
            if not took:
                break
            p += 1
    return np.asarray(rows, dtype=np.int64), np.asarray(owner, dtype=np.int64)


def _weights(sizes, owner):
    """w = |G_a| / m_a for each probe of cluster a (m_a probes taken from it),
    normalised to sum 1 (mlx deviation: the ridge does not scale with M)."""
    m = np.bincount(owner, minlength=len(sizes)).astype(np.float64)
    w = np.asarray(sizes, dtype=np.float64)[owner] / m[owner]
    return w / w.sum()


def select_probe_rows(labels, M):
    """Head-agnostic probe rows: middle-out member of each query cluster,
    round-robin across clusters. Returns (probe_idx (M,) int64, weights (M,))."""
    lab = np.asarray(labels, dtype=np.int64)
    C = int(lab.max()) + 1
    members, sizes = [], []
    for a in range(C):
        idx = np.nonzero(lab == a)[0]
        if len(idx) == 0:
            continue
        members.append([int(idx[j]) for j in _middle_out(len(idx))])
        sizes.append(len(idx))
    rows, owner = _round_robin(members, M)
    return rows, _weights(sizes, owner)


def select_probe_rows_centroid(q, labels, M):
    """Per (batch, query head) probes ordered by distance to the group centroid.

    For each cluster a the rows are ordered by the Euclidean distance
    ‖q_i − q̄_a‖₂ ascending (q̄_a the mean query of the cluster in that head; ties
    to the lower index), then stratified as in ``select_probe_rows``.
    Returns (probe_idx (B, H, M) int64, weights (B, H, M)).
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, S, D = q.shape
    lab = np.asarray(labels, dtype=np.int64)
    C = int(lab.max()) + 1
    groups = [np.nonzero(lab == a)[0] for a in range(C)]
    groups = [g for g in groups if len(g)]
    sizes = [len(g) for g in groups]
    idx = np.zeros((B, H, M), dtype=np.int64)
    wts = np.zeros((B, H, M))
    for b in range(B):
        for h in range(H):
            members = []
            for g in groups:
                x = q[b, h, g]
                d = np.sqrt(((x - x.mean(axis=0)) ** 2).sum(axis=1))
                order = np.lexsort((g, d))
                members.append([int(g[j]) for j in order])
            rows, owner = _round_robin(members, M)
            idx[b, h] = rows
            wts[b, h] = _weights(sizes, owner)
    return idx, wts


def probe_dense_attention(q, k, v, probe_idx, scale=None):
    """Exact dense attention of the probe rows over all keys (the recipe's SDPA call
    on q[:, :, probe_idx]). ``probe_idx`` is (M,) shared or (B, H, M) per head."""
    q = np.asarray(q, dtype=np.float64)
    pi = np.asarray(probe_idx)
    if pi.ndim == 1:
        return dense_attention(q, k, v, scale=scale, rows=pi)
    B, H, M = pi.shape
    out = np.zeros((B, H, M, np.shape(v)[-1]))
    for b in range(B):
        for h in range(H):
            g = h // (H // np.shape(k)[1])
            out[b, h] = dense_attention(q[b:b + 1, h:h + 1], np.asarray(k)[b:b + 1, g:g + 1],
                                        np.asarray(v)[b:b + 1, g:g + 1], scale=scale,
                                        rows=pi[b, h])[0, 0]
    return out


def standardise(x, eps=1e-6):
    """Column standardisation over all rows: Z = (X − μ) / sqrt(σ² + eps), with μ
    and the population variance σ² per column (reading of "standardized sparse
    output"; eps = 1e-6 keeps constant columns finite)."""
    mu = x.mean(axis=0)
    var = ((x - mu) ** 2).mean(axis=0)
    return (x - mu) / np.sqrt(var + eps)


def probe_residual_correction(out, o_probe, probe_idx, weights, rank=16, lam=0.1,
                              return_parts=False):
    """SparsePR repair of an approximate attention output, per (batch, head).

    With X the approximate output (S × D), Z its standardised form and Z̃ = [Z, 1]:
      R  = O_probe − X[p]                      residual at the M probe rows
      B  = (Z̃_pᵀ W Z̃_p + λ·diag(1,…,1,0))⁻¹ Z̃_pᵀ W R     weighted ridge affine fit
      V_r = top-r eigenvectors of Rᵀ W R       the residual subspace seen at the probes
      X' = X + Z̃ · B · V_r V_rᵀ               applied to every row
    Readings: the intercept column is not penalised; the whole affine prediction is
    projected; every row is corrected (probes are not overwritten with their exact
    values); W = diag(weights). ``probe_idx``/``weights`` are (M,) shared or
    (B, H, M) per head. Returns the repaired (B, H, S, D) array (and, with
    ``return_parts``, a dict of the per-head B, V_r, fit residuals).
    """
    X = np.asarray(out, dtype=np.float64)
    Op = np.asarray(o_probe, dtype=np.float64)
    B_, H, S, D = X.shape
    pi = np.asarray(probe_idx)
    wt = np.asarray(weights, dtype=np.float64)
    res = np.empty_like(X)
    parts = {"coef": np.zeros((B_, H, D + 1, D)), "Vr": np.zeros((B_, H, D, rank)),
             "fit_residual": np.zeros((B_, H, pi.shape[-1], D)), "eig": np.zeros((B_, H, D))}
    for b in range(B_):
        for h in range(H):
            p = pi if pi.ndim == 1 else pi[b, h]
            w = wt if wt.ndim == 1 else wt[b, h]
            x = X[b, h]
            Zt = np.concatenate([standardise(x), np.ones((S, 1))], axis=1)
            Zp = Zt[p]
            R = Op[b, h] - x[p]
            pen = np.eye(D + 1) * lam
            pen[D, D] = 0.0
            A = Zp.T @ (w[:, None] * Zp) + pen
            Y = Zp.T @ (w[:, None] * R)
            coef = np.linalg.solve(A, Y)
            G = R.T @ (w[:, None] * R)
            evals, evecs = np.linalg.eigh(G)
            Vr = evecs[:, ::-1][:, :rank]
            corr = Zt @ (coef @ Vr @ Vr.T)
            res[b, h] = x + corr
            parts["coef"][b, h] = coef
            parts["Vr"][b, h] = Vr
            parts["eig"][b, h] = evals[::-1]
            parts["fit_residual"][b, h] = R - corr[p]
    return (res, parts) if return_parts else res
