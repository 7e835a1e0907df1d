"""Oracle: executed-pair accounting.

Test infrastructure only (see the package docstring).

Source: "Partition the Support, Reconstruct the Residual", §Q, K, and V are permuted
into group-major order: total executed-pair density is the routing density plus
M / Nq, counted in whole (query group, key group) cells.
"""

import numpy as np


def executed_pairs(q_labels, k_labels, block_mask, H, B=1, M=0, Sk=None):
    """Token pairs computed exactly: Σ over kept cells of n_a · n_c per (b, h), plus
    M · Sk probe pairs per (b, h). Centroid terms are not counted.
    ``block_mask`` is (Cq, Ck), (H, Cq, Ck) or (B, H, Cq, Ck)."""
    ql = np.asarray(q_labels, dtype=np.int64)
    kl = np.asarray(k_labels, dtype=np.int64)
    m = np.asarray(block_mask).astype(bool)
    Cq, Ck = m.shape[-2:]
    na = np.bincount(ql, minlength=Cq).astype(np.int64)
    nc = np.bincount(kl, minlength=Ck).astype(np.int64)
    cell = na[:, None] * nc[None, :]
    mm = np.broadcast_to(m.reshape((1,) * (4 - m.ndim) + m.shape), (B, H, Cq, Ck))
    Sk = len(kl) if Sk is None else Sk
    return int((mm * cell).sum()) + B * H * M * Sk
