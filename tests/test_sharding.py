"""CPU: a layer's heads split over ranks (two gloo ranks), the KV-aligned head ranges
and the layer gate's one-integer all-reduce ("Dynamic block masks and head-wise mask
reuse", §HEART: the gate looks at the fraction of the layer's heads asking for a
refresh). The per-head decisions of each rank come from the oracle's cache over the
rank's own heads with no gate; after the all-reduce the gate must give what an
unsharded oracle cache of the whole layer gives."""

import os
import socket
import sys

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_head_ranges_cover_the_layer_on_kv_boundaries():
    from block_sparse_attention_tcgen05_b200.sharding import head_range
    for Hq, Hkv, world in [(40, 40, 2), (40, 40, 8), (24, 8, 2), (24, 8, 8), (24, 8, 3), (48, 6, 4)]:
        got = [head_range(Hq, Hkv, world, r) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == Hq and got[0][2] == 0 and got[-1][3] == Hkv
        for (h0, h1, g0, g1), nxt in zip(got, got[1:] + [None]):
            assert h0 == g0 * (Hq // Hkv) and h1 == g1 * (Hq // Hkv) and h1 > h0
            if nxt is not None:
                assert nxt[0] == h1 and nxt[2] == g1
        sizes = [g1 - g0 for _, _, g0, g1 in got]
        assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        head_range(24, 8, 9, 0)     # more ranks than KV heads
    with pytest.raises(ValueError):
        head_range(10, 4, 2, 0)     # Hq not a multiple of Hkv


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gate(ref, n_layer, n_heads, lo, hi, first):
    if first or lo < 0:
        return ref
    frac = np.float32(n_layer) / np.float32(n_heads)
    if frac < lo:
        return np.zeros_like(ref)
    if frac > hi:
        return np.ones_like(ref)
    return ref


def _rank_main(rank, world, port, H, q_steps, k_steps, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    from block_sparse_attention_tcgen05_b200.sharding import head_range, layer_refresh_count
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        h0, h1, _, _ = head_range(H, H, world, rank)
        local = oracle.HeadMaskCache(delta=1.0, gate_lo=-1)   # this rank's heads, no gate
        full = oracle.HeadMaskCache(delta=1.0)                # the whole layer, gate 0.4 / 0.8
        out = []
        for t, (q, k) in enumerate(zip(q_steps, k_steps)):
            want = full.should_refresh(q, k)
            ref_local = local.should_refresh(q[:, h0:h1], k[:, h0:h1])
            n_layer = layer_refresh_count(int(ref_local.sum()))
            got = _gate(ref_local, n_layer, q.shape[0] * H, 0.4, 0.8, first=(t == 0))
            out.append((bool((got == want[:, h0:h1]).all()), int(n_layer)))
            full.update(np.zeros((q.shape[0], H, 2, 2), dtype=bool), want)
            local.update(np.zeros((q.shape[0], h1 - h0, 2, 2), dtype=bool), got)
        results[rank] = out
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_sharded_gate_matches_the_unsharded_layer(world):
    H, S, D = 10, 6, 3
    g = np.random.default_rng(0)
    q0 = g.standard_normal((1, H, S, D))
    k0 = g.standard_normal((1, H, S, D))
    steps_q, steps_k = [q0], [k0]
    # step 1: heads 0-2 drift by L1 3 (> delta 1): 30 % of the layer -> none refresh;
    # step 2: heads 0-4 (50 %) -> per head, heads 0-4 re-anchor at +1;
    # step 3: heads 0-8 move to +3, every one of them past delta again (90 %) -> all
    for n, shift in ((3, 1.0), (5, 1.0), (9, 3.0)):
        q = q0.copy()
        q[0, :n] += shift
        steps_q.append(q)
        steps_k.append(k0)
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [mp.get_context("spawn").Process(target=_rank_main,
                                             args=(r, world, port, H, steps_q, steps_k, results))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        flags = [ok for ok, _ in results[r]]
        counts = [n for _, n in results[r]]
        assert all(flags), (r, results[r])
        assert counts == [H, 3, 5, 9], counts
