"""Oracle attention: dense, hard-drop block-sparse, and SVG-EAR centroid-compensated.

Test infrastructure only (see the package docstring).

Notation (per batch b and query head h): q_i, k_j, v_j rows of Q, K, V; a_i the
query-cluster label of row i; l_j the key-cluster label of key j; kept(a, c) the
cluster-level block mask (True = block computed exactly). Under grouped-query
attention the KV head of query head h is h // (Hq / Hkv), so routes and clusters
are shared by the query heads of one KV head ("Partition the Support, Reconstruct
the Residual", §Q, K, and V are permuted into group-major order).
"""

import numpy as np


def kv_head(h, Hq, Hkv):
    """KV head serving query head h: contiguous groups of Hq/Hkv query heads."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def _as64(x):
    return np.asarray(x, dtype=np.float64)


def _softmax_average(logits, values):
    """Row-wise softmax of ``logits`` (−inf allowed) applied to ``values``.

    A row whose logits are all −inf has no term in its softmax; it returns 0 (the
    reading taken for an all-skipped row under hard drop).
    """
    if logits.shape[1] == 0:
        return np.zeros((logits.shape[0], values.shape[1]))
    m = logits.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(logits - m)
    den = e.sum(axis=1)
    num = e @ values
    out = np.zeros_like(num)
    nz = den > 0
    out[nz] = num[nz] / den[nz, None]
    return out


def cluster_centroids(k, v, k_labels, Ck):
    """Cluster sizes n_c and arithmetic-mean centroids k̄_c, v̄_c of one KV head.

    "Sparse-block compensation", §SVG-EAR — centroid compensation: each skipped key
    is replaced by its cluster centroid and its value by the value centroid. The
    centroid is read as the arithmetic mean of the cluster's rows. Empty clusters
    get n_c = 0 and zero centroids; their log-count prior ln 0 = −inf removes them.
    """
    k = _as64(k)
    v = _as64(v)
    lab = np.asarray(k_labels, dtype=np.int64)
    n = np.bincount(lab, minlength=Ck).astype(np.int64)
    kbar = np.zeros((Ck, k.shape[1]))
    vbar = np.zeros((Ck, v.shape[1]))
    np.add.at(kbar, lab, k)
    np.add.at(vbar, lab, v)
    nz = n > 0
    kbar[nz] /= n[nz, None]
    vbar[nz] /= n[nz, None]
    return n, kbar, vbar


def dense_attention(q, k, v, scale=None, rows=None):
    """O_i = Σ_j softmax_j(scale · q_i · k_j) v_j for every (b, h); shape (B, H, R, Dv).

    ``rows`` selects query rows (default all), so large cases can be sampled.
    GQA: K, V have Hkv heads.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, Hq, Sq, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = D ** -0.5
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    out = np.zeros((B, Hq, len(rows), v.shape[-1]))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            logits = scale * (q[b, h, rows] @ k[b, g].T)
            out[b, h] = _softmax_average(logits, v[b, g])
    return out


def _mask_bh(block_mask, b, h):
    """Cluster-level kept mask for (b, h); ``block_mask`` is (Cq, Ck), (H, Cq, Ck)
    or (B, H, Cq, Ck), with size-1 leading dimensions broadcast."""
    m = np.asarray(block_mask).astype(bool)
    if m.ndim == 2:
        return m
    if m.ndim == 3:
        return m[h if m.shape[0] > 1 else 0]
    return m[b if m.shape[0] > 1 else 0, h if m.shape[1] > 1 else 0]


def centroid_compensated_attention(q, k, v, q_labels, k_labels, block_mask, scale=None,
                                   compensate=True, rows=None, Cq=None, Ck=None):
    """SVG-EAR centroid-compensated block-sparse attention (formulation A).

    "Sparse-block compensation", §The problem and §SVG-EAR — centroid compensation:
    for query row i in cluster a, the softmax runs over

    * every key j whose cluster l_j has kept(a, l_j), logit scale · q_i · k_j,
      value v_j, and
    * (compensate) one term per skipped non-empty key cluster c, logit
      scale · q_i · k̄_c + ln n_c, value v̄_c.

    With ``compensate=False`` this is hard drop: the softmax is renormalised over
    kept keys only, and a row with no kept key returns 0. All query rows of one
    cluster share one key set, so the computation runs per query cluster.
    Returns (B, H, R, Dv) float64 for the selected ``rows`` (default all rows).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, Hq, Sq, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = D ** -0.5
    ql = np.asarray(q_labels, dtype=np.int64)
    kl = np.asarray(k_labels, dtype=np.int64)
    Cq = int(ql.max()) + 1 if Cq is None else Cq
    Ck = int(kl.max()) + 1 if Ck is None else Ck
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    out = np.zeros((B, Hq, len(rows), v.shape[-1]))
    for b in range(B):
        stats = [cluster_centroids(k[b, g], v[b, g], kl, Ck) for g in range(Hkv)]
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            n, kbar, vbar = stats[g]
            kept = _mask_bh(block_mask, b, h)
            row_lab = ql[rows]
            for a in np.unique(row_lab):
                sel = np.nonzero(row_lab == a)[0]
                qi = q[b, h, rows[sel]]
                tok = np.nonzero(kept[a, kl])[0]
                logits = [scale * (qi @ k[b, g, tok].T)]
                values = [v[b, g, tok]]
                if compensate:
                    cen = np.nonzero(~kept[a] & (n > 0))[0]
                    logits.append(scale * (qi @ kbar[cen].T) + np.log(n[cen])[None, :])
                    values.append(vbar[cen])
                out[b, h, sel] = _softmax_average(np.concatenate(logits, axis=1),
                                                  np.concatenate(values, axis=0))
    return out


def hard_drop_attention(q, k, v, q_labels, k_labels, block_mask, scale=None, rows=None,
                        Cq=None, Ck=None):
    """Block-sparse attention with skipped blocks dropped and the softmax renormalised
    over kept keys ("Sparse-block compensation", §The problem)."""
    return centroid_compensated_attention(q, k, v, q_labels, k_labels, block_mask, scale,
                                          compensate=False, rows=rows, Cq=Cq, Ck=Ck)


def extended_key_attention(q, k, v, q_labels, k_labels, block_mask, scale=None,
                           compensate=True, Cq=None, Ck=None):
    """Formulation B: one dense softmax over the extended keys.

    "Sparse-block compensation", §No LSE needed: the compensated output equals one
    softmax over keys [K; K̄] and values [V; V̄] with an additive (Sq, Sk + Ck) mask
    that is 0 / −inf on token columns (kept / skipped block) and ln n_c / −inf on
    centroid columns (skipped / kept block). Empty clusters get −inf (ln 0). With
    ``compensate=False`` every centroid column is −inf (hard drop).
    This is an independent route to the same numbers as formulation A.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, Hq, Sq, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = D ** -0.5
    ql = np.asarray(q_labels, dtype=np.int64)
    kl = np.asarray(k_labels, dtype=np.int64)
    Cq = int(ql.max()) + 1 if Cq is None else Cq
    Ck = int(kl.max()) + 1 if Ck is None else Ck
    out = np.zeros((B, Hq, Sq, v.shape[-1]))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            n, kbar, vbar = cluster_centroids(k[b, g], v[b, g], kl, Ck)
            kept = _mask_bh(block_mask, b, h)
            k_ext = np.concatenate([k[b, g], kbar], axis=0)
            v_ext = np.concatenate([v[b, g], vbar], axis=0)
            tok_mask = np.where(kept[ql][:, kl], 0.0, -np.inf)
            with np.errstate(divide="ignore"):
                logn = np.log(n.astype(np.float64))
            if compensate:
                cen_mask = np.where(kept[ql], -np.inf, logn[None, :])
            else:
                cen_mask = np.full((Sq, Ck), -np.inf)
            add = np.concatenate([tok_mask, cen_mask], axis=1)
            logits = scale * (q[b, h] @ k_ext.T) + add
            out[b, h] = _softmax_average(logits, v_ext)
    return out
