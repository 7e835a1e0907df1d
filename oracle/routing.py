"""Oracle: SVG-EAR error-aware routing (which blocks to compute exactly).

Test infrastructure only (see the package docstring).

Source: "Sparse-block compensation", §SVG-EAR — centroid compensation (the paper adds
an error-aware router choosing which blocks to compute exactly) and the SVG-EAR
abstract on the block-sparse attention topic feed (a lightweight probe estimates the
compensation error of every block; the blocks with the highest error-to-cost ratio
are computed exactly, the skipped ones compensated).

The pages name the probe and the ratio but not their formulas. Readings taken here:

* Probe: one query per (batch, query head, query cluster a), the cluster's mean query
  q̄_a.
* Block error: for that probe, with dense logits l_j = scale · q̄_a · k_j, their
  maximum m and Z = Σ_j exp(l_j − m) over every key, the exact contribution of key
  cluster c to the probe's output is E_ac = Σ_{j∈c} exp(l_j − m) v_j / Z and its
  centroid compensation is A_ac = n_c exp(scale · q̄_a · k̄_c − m) v̄_c / Z; the
  error is err_ac = ‖E_ac − A_ac‖₂ (the change of the probe's output when the block
  is compensated instead of computed, to first order).
* Cost: the block's token pairs n_a · n_c. Ratio = n_a · err_ac / (n_a · n_c) =
  err_ac / n_c (the error summed over the cluster's rows per computed pair).
* Selection per (batch, head): blocks with n_a > 0 and n_c > 0 in descending ratio
  (equal ratios: lower a · Ck + c first); keep the longest prefix whose summed cost
  is at most the budget floor(density · Σ_a n_a · Σ_c n_c). Blocks of empty
  clusters are never kept (they hold no pair).
"""

import numpy as np

from .attention import cluster_centroids, kv_head


def _query_centroids(q, q_labels, Cq):
    """Mean query of each cluster, (Cq, D); empty clusters get zeros."""
    lab = np.asarray(q_labels, dtype=np.int64)
    n = np.bincount(lab, minlength=Cq)
    qbar = np.zeros((Cq, q.shape[1]))
    np.add.at(qbar, lab, q)
    nz = n > 0
    qbar[nz] /= n[nz, None]
    return n, qbar


def compensation_errors(q, k, v, q_labels, k_labels, Cq, Ck, scale=None):
    """err (B, Hq, Cq, Ck): the probe-estimated compensation error of every block
    (readings in the module docstring); 0 where either cluster is empty."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = D ** -0.5
    kl = np.asarray(k_labels, dtype=np.int64)
    err = np.zeros((B, Hq, Cq, Ck))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            n_q, qbar = _query_centroids(q[b, h], q_labels, Cq)
            n_k, kbar, vbar = cluster_centroids(k[b, g], v[b, g], kl, Ck)
            for a in np.nonzero(n_q)[0]:
                logits = scale * (k[b, g] @ qbar[a])
                m = logits.max()
                e = np.exp(logits - m)
                Z = e.sum()
                for c in np.nonzero(n_k)[0]:
                    sel = kl == c
                    exact = (e[sel] @ v[b, g, sel]) / Z
                    comp = n_k[c] * np.exp(scale * (qbar[a] @ kbar[c]) - m) * vbar[c] / Z
                    err[b, h, a, c] = np.linalg.norm(exact - comp)
    return err


def route_blocks(err, q_labels, k_labels, Cq, Ck, density, dtype=np.float64):
    """The budgeted prefix selection of SVG-EAR routing, given block errors
    (B, Hq, Cq, Ck): per (batch, head), blocks ranked by err_ac / n_c descending (ties:
    lower a · Ck + c); the longest prefix whose token pairs n_a · n_c sum to at most
    floor(density · Sq · Sk) is kept. ``dtype`` is the precision of the ratio (float32
    when deciding on a kernel's own float32 errors, as the kernel does). Returns a bool
    mask (B, Hq, Cq, Ck)."""
    n_q = np.bincount(np.asarray(q_labels, dtype=np.int64), minlength=Cq).astype(np.int64)
    n_k = np.bincount(np.asarray(k_labels, dtype=np.int64), minlength=Ck).astype(np.int64)
    cost = np.outer(n_q, n_k)
    budget = int(np.floor(float(density) * float(n_q.sum()) * float(n_k.sum())))
    err = np.asarray(err)
    B, Hq = err.shape[:2]
    mask = np.zeros(err.shape, dtype=bool)
    valid = cost > 0
    for b in range(B):
        for h in range(Hq):
            ratio = np.where(valid, err[b, h].astype(dtype) / np.maximum(n_k, 1).astype(dtype)[None, :],
                             dtype(-1.0))
            flat = ratio.reshape(-1)
            idx = np.arange(flat.size)
            order = np.lexsort((idx, -flat))
            total = 0
            for e in order:
                if flat[e] < 0:
                    break
                a, c = divmod(int(e), Ck)
                if total + cost[a, c] > budget:
                    break
                total += int(cost[a, c])
                mask[b, h, a, c] = True
    return mask


def error_aware_block_mask(q, k, v, q_labels, k_labels, Cq, Ck, density, scale=None):
    """SVG-EAR routing: (mask (B, Hq, Cq, Ck) bool, err (B, Hq, Cq, Ck)): the block
    errors of ``compensation_errors`` and the selection of ``route_blocks``."""
    err = compensation_errors(q, k, v, q_labels, k_labels, Cq, Ck, scale)
    return route_blocks(err, q_labels, k_labels, Cq, Ck, density), err


def centroid_mass(q, k, q_labels, k_labels, Cq, Ck, scale=None):
    """Block mass estimate (B, Hq, Cq, Ck): for the mean query q̄_a of each query
    cluster, the softmax over key clusters of scale · q̄_a · k̄_c + ln n_c (empty key
    clusters: 0), the share of q̄_a's attention that falls on each key cluster when
    every key is replaced by its cluster centroid ("Sparse-block compensation",
    §SVG-EAR: a cluster enters the softmax as one term with the log-count prior).
    Rows of empty query clusters are 0."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = D ** -0.5
    kl = np.asarray(k_labels, dtype=np.int64)
    v0 = np.zeros_like(k[0, 0])
    out = np.zeros((B, Hq, Cq, Ck))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            n_q, qbar = _query_centroids(q[b, h], q_labels, Cq)
            n_k, kbar, _ = cluster_centroids(k[b, g], v0, kl, Ck)
            with np.errstate(divide="ignore"):
                logits = scale * (qbar @ kbar.T) + np.log(n_k.astype(np.float64))[None, :]
            m = logits.max(1, keepdims=True)
            e = np.exp(logits - m)
            out[b, h] = e / e.sum(1, keepdims=True)
            out[b, h, n_q == 0] = 0.0
    return out


def probe_budget_block_mask(q, k, q_labels, k_labels, Cq, Ck, density, M, scale=None):
    """SparsePR's router with the probe cost reserved first ("Partition the Support,
    Reconstruct the Residual": executed-pair density is the routing density plus M/Nq,
    and the router reserves the probe cost before routing). Reading: cells are ranked
    by their centroid-estimated attention mass per computed pair (``centroid_mass`` /
    n_c) and the budgeted prefix of ``route_blocks`` is taken with the routing density
    max(0, density − M / Sq). Returns (mask (B, Hq, Cq, Ck) bool, mass)."""
    mass = centroid_mass(q, k, q_labels, k_labels, Cq, Ck, scale)
    Sq = len(np.asarray(q_labels))
    route = max(0.0, float(density) - float(M) / Sq)
    return route_blocks(mass, q_labels, k_labels, Cq, Ck, route), mass
