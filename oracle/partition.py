"""Oracle: SparsePR Response-Coupled Partitioning (query and key clusters).

Test infrastructure only (see the package docstring).

Source: "Partition the Support, Reconstruct the Residual" (paper summary): queries are
sampled from the current call and keys grouped by their pre-softmax response; keys with
similar response profiles share a K/V block and values follow their keys; centroids of
the key groups then define query coordinates, so that queries with a similar response
direction share a route; one asymmetric pass with no alternating refinement; feature
ranks rK = 48 and rQ = 64; K/V partitions and routes are shared by the query heads of a
KV head (grouped-query attention); the latency includes an online k-means.

The pages name these steps but not their constants. Readings taken here, per (batch,
KV head g) with G = Hq / Hkv query heads h = g·G .. g·G + G − 1:

* Samples: rK query rows, sample s at token floor((s + 1/2) · Sq / rK) of query head
  g·G + (s mod G).
* Key features: f_j = scale · Q_s k_j (rK response logits per key).
* k-means (Lloyd): centroids start at the rows floor((c + 1/2) · N / C); each round
  assigns every row to its nearest centroid (squared Euclidean distance, ties to the
  lower index) and moves every centroid to the mean of its rows (an empty cluster keeps
  its centroid); after ``iters`` rounds a last assignment gives the labels.
* Key groups: Ck clusters of the key features. Their centroids in key space, k̄_c, are
  the means of the keys of each group.
* Query coordinates: rQ' = min(rQ, Ck) groups c_t = floor((t + 1/2) · Ck / rQ'); query
  token i gets x_i = (scale · q_{h,i} · k̄_{c_t}) over t and over the G query heads h of
  the group (rQ'·G values), divided by its Euclidean norm ("response direction"; a zero
  vector stays zero). Query groups: Cq clusters of those coordinates.
"""

import numpy as np


def kmeans(x, C, iters):
    """Labels (N,) of the Lloyd iteration described in the module docstring."""
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    cent = x[(np.arange(C) * 2 + 1) * N // (2 * C)].copy()
    for _ in range(iters + 1):
        d = ((x[:, None, :] - cent[None, :, :]) ** 2).sum(-1)
        lab = np.argmin(d, axis=1)          # first minimum: ties to the lower index
        if _ == iters:
            break
        for c in range(C):
            sel = lab == c
            if sel.any():
                cent[c] = x[sel].mean(0)
    return lab


def response_coupled_partition(q, k, Cq, Ck, r_k=48, r_q=64, iters=8, scale=None,
                               return_features=False):
    """Query labels (B, Hkv, Sq) and key labels (B, Hkv, Sk), one partition per
    (batch, KV head) shared by its query heads (readings in the module docstring).
    With ``return_features`` also the key features (B, Hkv, Sk, rK) and the query
    coordinates (B, Hkv, Sq, rQ'·G)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = D ** -0.5
    rq = min(r_q, Ck)
    ql = np.zeros((B, Hkv, Sq), dtype=np.int64)
    kl = np.zeros((B, Hkv, Sk), dtype=np.int64)
    fk_all = np.zeros((B, Hkv, Sk, r_k))
    xq_all = np.zeros((B, Hkv, Sq, rq * G))
    for b in range(B):
        for g in range(Hkv):
            toks = (np.arange(r_k) * 2 + 1) * Sq // (2 * r_k)
            heads = g * G + np.arange(r_k) % G
            qs = q[b, heads, toks]                          # (rK, D)
            fk = scale * (k[b, g] @ qs.T)                   # (Sk, rK)
            kl[b, g] = kmeans(fk, Ck, iters)
            kbar = np.zeros((Ck, D))
            for c in range(Ck):
                sel = kl[b, g] == c
                if sel.any():
                    kbar[c] = k[b, g, sel].mean(0)
            cols = (np.arange(rq) * 2 + 1) * Ck // (2 * rq)
            xq = np.concatenate([scale * (q[b, g * G + j] @ kbar[cols].T) for j in range(G)],
                                axis=1)                     # (Sq, rQ'·G)
            nrm = np.sqrt((xq ** 2).sum(1, keepdims=True))
            xq = np.where(nrm > 0, xq / np.where(nrm > 0, nrm, 1.0), 0.0)
            ql[b, g] = kmeans(xq, Cq, iters)
            fk_all[b, g], xq_all[b, g] = fk, xq
    if return_features:
        return ql, kl, fk_all, xq_all
    return ql, kl
