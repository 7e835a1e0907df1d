"""A layer's heads split over GPUs, one process per GPU.

Every step of the hot path is independent per (batch, head), so heads shard with no
exchange of attention data; under grouped-query attention the unit is a KV head
together with its query heads ("Partition the Support, Reconstruct the Residual": K/V
partitions and routes are shared by a KV head's query heads). The one step that couples
heads is the mask cache's layer gate ("Dynamic block masks and head-wise mask reuse",
§HEART: under 40 % of the layer's heads asking for a refresh none refresh, above 80 % all
do), which needs the layer-wide refresh count: one integer all-reduce per layer and
step (NCCL over NVLink between GPUs).
"""

import ctypes

import torch
import torch.distributed as dist

from .ops import MaskCache, _call_on, _ptr, _stream


def head_range(Hq, Hkv, world, rank):
    """Query heads [h0, h1) and KV heads [g0, g1) of ``rank`` out of ``world``: the KV
    heads split into contiguous, as-equal-as-possible ranges, each KV head with its
    Hq / Hkv query heads."""
    if Hq % Hkv:
        raise ValueError(f"Hq ({Hq}) must be a multiple of Hkv ({Hkv})")
    if not 0 <= rank < world or world > Hkv:
        raise ValueError(f"rank {rank} of {world} over {Hkv} KV heads")
    g = Hq // Hkv
    g0, g1 = rank * Hkv // world, (rank + 1) * Hkv // world
    return g0 * g, g1 * g, g0, g1


def layer_refresh_count(n_local, group=None, device=None):
    """Refresh count summed over the ranks of ``group`` (one int64 all-reduce; a plain
    return without an initialised process group)."""
    if not dist.is_available() or not dist.is_initialized():
        return int(n_local)
    t = torch.tensor([int(n_local)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(t.item())


class ShardedMaskCache:
    """HEART per-head mask cache for the query heads [h0, h1) of a layer of ``H_layer``
    heads whose other heads live on other ranks.

    The local cache decides per head (drift against its anchors, delta) with no gate of
    its own; ``should_refresh`` then adds the refresh counts of every rank (one integer
    all-reduce over ``group``) and applies the layer gate to the local flags on the
    device (``bsa_mask_cache_layer_gate``), so every rank takes the decision an
    unsharded cache of the whole layer would take.
    """

    def __init__(self, B, H_layer, h0, h1, Cq, Ck, D, delta, relative=False, gate_lo=0.4,
                 gate_hi=0.8, group=None, device="cuda"):
        if not 0 <= h0 < h1 <= H_layer:
            raise ValueError(f"head range [{h0}, {h1}) outside a layer of {H_layer} heads")
        self.B, self.H_layer, self.h0, self.h1 = B, H_layer, h0, h1
        self.gate_lo, self.gate_hi = float(gate_lo), float(gate_hi)
        self.group = group
        self.cache = MaskCache(B, h1 - h0, Cq, Ck, D, delta, relative=relative, gate_lo=-1.0,
                               gate_hi=gate_hi, device=device)

    @property
    def mask(self):
        return self.cache.mask

    def should_refresh(self, q, k):
        """q, k: (B, h1 - h0, S, D) of the local heads. Returns the device uint8
        (B, h1 - h0) refresh flags after the layer gate, and the layer-wide count of heads
        asking for a refresh before it."""
        refresh, n_local = self.cache.should_refresh(q, k, sync=True)
        dev = refresh.device
        comm_dev = dev if dist.is_initialized() and dist.get_backend(self.group) == "nccl" else "cpu"
        n_layer = layer_refresh_count(n_local, self.group, comm_dev)
        _call_on(dev, "bsa_mask_cache_layer_gate", _ptr(self.cache.state), _ptr(refresh),
                 int(n_layer), int(self.B * self.H_layer), ctypes.c_float(self.gate_lo),
                 ctypes.c_float(self.gate_hi), _stream(dev))
        return refresh, n_layer

    def update(self, new_mask):
        """Cached mask of the local heads with the refreshed ones replaced."""
        return self.cache.update(new_mask)

    def reset(self):
        self.cache.reset()

