"""Oracle: XAttention anti-diagonal block scoring and per-row top-p block selection.

Test infrastructure only (see the package docstring).

Source: "Dynamic block masks and head-wise mask reuse", §XAttention — anti-diagonal
block scoring, §Deviations from the papers (normalised scores, no forced block 0),
§Out of scope (padding: the caller pads to a multiple of the block size and padded
keys still take softmax mass).
"""

import numpy as np

from .attention import kv_head


def antidiagonal_block_scores(q, k, block, stride, logit_scale=None):
    """Block-mass estimate from strided anti-diagonal sums of QKᵀ.

    For every stride × stride sub-block (I, J) of QKᵀ, the anti-diagonal sum is
    A[I, J] = Σ_{t<s} q_{I·s+t} · k_{J·s+s−1−t}  (reading: the anti-diagonal of a
    sub-block is its (t, s−1−t) entries). Each strided row is softmaxed over all
    N/s columns, P = rowsoftmax(logit_scale · A) (reading: logit_scale = 1/sqrt(D)
    applied to the anti-diagonal sum, no extra 1/stride; parity unpinned for that
    convention), then summed per block × block tile and divided by block/stride so
    each row of the (N/b, N/b) result sums to 1.

    q: (B, Hq, N, D), k: (B, Hkv, N, D) with N a multiple of ``block`` and ``block``
    a multiple of ``stride``. Returns (B, Hq, N/block, N/block) float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    s, b = int(stride), int(block)
    if N % b or b % s:
        raise ValueError("N must be a multiple of block and block of stride")
    if logit_scale is None or logit_scale <= 0:
        logit_scale = D ** -0.5
    ns, nb, r = N // s, N // b, b // s
    out = np.zeros((B, Hq, nb, nb))
    for bb in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            # Row I of Qs is q_{Is}, ..., q_{Is+s-1} laid end to end; row J of Kr is
            # k_{Js+s-1}, ..., k_{Js} (reversed inside the stride group), so that
            # Qs[I] . Kr[J] is the anti-diagonal sum of sub-block (I, J).
            Qs = q[bb, h].reshape(ns, s * D)
            Kr = k[bb, g].reshape(ns, s, D)[:, ::-1, :].reshape(ns, s * D)
            A = logit_scale * (Qs @ Kr.T)
            A -= A.max(axis=1, keepdims=True)
            P = np.exp(A)
            P /= P.sum(axis=1, keepdims=True)
            out[bb, h] = P.reshape(nb, r, nb, r).sum(axis=(1, 3)) / r
    return out


def top_p_block_mask(scores, tau, dtype=np.float64, tie_eps=1e-5):
    """Per query block, keep the smallest set of key blocks whose mass reaches τ.

    Reading of "reaches a fraction τ of its total": sort the row's scores in
    descending order (equal scores: lower key-block index first), take the
    inclusive running sum, and keep ranks 0..m where m is the first rank whose
    running sum is ≥ τ. At least one block is kept; key block 0 is not forced. If
    rounding keeps every running sum below τ, the whole row is kept.

    ``tau`` is a scalar or one value per head (H,). ``dtype`` is the precision in
    which the running sum and the comparison are taken: float64 for the oracle
    chain, float32 (sequential running sum in sorted order) when checked against
    a kernel that decides in float32.

    Returns (mask (B, H, Nq, Nk) bool, tie (B, H, Nq) bool). A row is a tie row
    when some running sum lies within ``tie_eps`` of τ or when the last kept and
    the first dropped score differ by at most ``tie_eps``: there a float32 and a
    float64 decision may legitimately differ.
    """
    sc = np.asarray(scores).astype(dtype)
    B, H, Nq, Nk = sc.shape
    tau_h = np.broadcast_to(np.asarray(tau, dtype=np.float64).reshape(-1), (H,)) \
        if np.ndim(tau) else np.full(H, float(tau))
    mask = np.zeros(sc.shape, dtype=bool)
    tie = np.zeros((B, H, Nq), dtype=bool)
    for b in range(B):
        for h in range(H):
            t = dtype(tau_h[h])
            for i in range(Nq):
                row = sc[b, h, i]
                order = np.argsort(-row, kind="stable")
                srt = row[order]
                cum = np.cumsum(srt, dtype=dtype)
                hit = np.nonzero(cum >= t)[0]
                m = int(hit[0]) if len(hit) else Nk - 1
                mask[b, h, i, order[: m + 1]] = True
                near = np.abs(cum.astype(np.float64) - float(tau_h[h])) <= tie_eps
                gap = (m + 1 < Nk) and (float(srt[m]) - float(srt[m + 1]) <= tie_eps)
                tie[b, h, i] = bool(near.any() or gap)
    return mask, tie
