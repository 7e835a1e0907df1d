"""Oracle: HEART temporal mask reuse — per-head drift/anchor mask cache.

Test infrastructure only (see the package docstring).

Source: "Dynamic block masks and head-wise mask reuse", §HEART — head-wise temporal
mask reuse (anchor = token means q̄, k̄ and the head's mask; drift = L1 distance;
refresh above δ; layer gate under 40 % / above 80 %), §What mlx-arsenal ships
(``pooled_qk``, ``qk_drift``, ``HeadMaskCache``), §Recipe (all heads refresh on the
first call), §Deviations (relative drift option), "Reuse needs a fixed token grid"
(reset on a grid change).
"""

import numpy as np


def pooled_qk(q, k):
    """Token means q̄, k̄ per (batch, head): shapes (B, H, D) each."""
    return (np.asarray(q, dtype=np.float64).mean(axis=2),
            np.asarray(k, dtype=np.float64).mean(axis=2))


def qk_drift(anchor_q, anchor_k, qbar, kbar, relative=False):
    """‖q̄_anchor − q̄‖₁ + ‖k̄_anchor − k̄‖₁ per (b, h); with ``relative`` divided by
    the anchor's L1 norm ‖q̄_anchor‖₁ + ‖k̄_anchor‖₁ (reading of "divides by the
    anchor's L1 norm")."""
    d = np.abs(anchor_q - qbar).sum(-1) + np.abs(anchor_k - kbar).sum(-1)
    if relative:
        d = d / (np.abs(anchor_q).sum(-1) + np.abs(anchor_k).sum(-1))
    return d


class HeadMaskCache:
    """Two-phase per-head mask cache: ``should_refresh`` then ``update``.

    Readings: per (b, h) anchors; the gate counts the fraction of all (b, h) heads
    of the layer asking for a refresh; strictly under ``gate_lo`` → none refresh,
    strictly above ``gate_hi`` → all refresh (``gate_lo < 0`` disables the gate);
    the first call after construction or ``reset`` refreshes every head; anchors
    move only for refreshed heads, to the pooled values of the call that asked.
    """

    def __init__(self, delta, relative=False, gate_lo=0.4, gate_hi=0.8):
        self.delta = float(delta)
        self.relative = bool(relative)
        self.gate_lo = float(gate_lo)
        self.gate_hi = float(gate_hi)
        self.reset()

    def reset(self):
        """Forget anchors and masks (a grid change invalidates every cached mask)."""
        self.anchor_q = self.anchor_k = None
        self.mask = None
        self._pending = None
        self.last_drift = None

    def should_refresh(self, q, k):
        qbar, kbar = pooled_qk(q, k)
        self._pending = (qbar, kbar)
        if self.anchor_q is None:
            self.last_drift = np.full(qbar.shape[:2], np.inf)
            return np.ones(qbar.shape[:2], dtype=bool)
        d = qk_drift(self.anchor_q, self.anchor_k, qbar, kbar, self.relative)
        self.last_drift = d
        ref = d > self.delta
        if self.gate_lo >= 0:
            frac = ref.mean()
            if frac < self.gate_lo:
                ref[:] = False
            elif frac > self.gate_hi:
                ref[:] = True
        return ref

    def update(self, new_mask, refresh):
        """Cached mask with refreshed heads replaced by ``new_mask``; anchors of the
        refreshed heads move to the pooled values of the last ``should_refresh``."""
        refresh = np.asarray(refresh, dtype=bool)
        qbar, kbar = self._pending
        if self.mask is None:
            self.mask = np.asarray(new_mask, dtype=bool).copy()
            self.anchor_q, self.anchor_k = qbar.copy(), kbar.copy()
            return self.mask.copy()
        if refresh.any():
            nm = np.asarray(new_mask, dtype=bool)
            self.mask[refresh] = nm[refresh]
            self.anchor_q[refresh] = qbar[refresh]
            self.anchor_k[refresh] = kbar[refresh]
        return self.mask.copy()
