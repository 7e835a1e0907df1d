"""GPU: a layer's heads split over two ranks, each with its own mask cache on the GPU
and the layer gate taken over the summed refresh counts ("Dynamic block masks and
head-wise mask reuse", §HEART). Both ranks run as processes on the one GPU of this
test; their kernels never wait on each other (the count is all-reduced on the host over
gloo). Every step's refresh flags of every rank must equal those of an unsharded oracle
cache over the whole layer."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _steps(H, S, D, seed=0):
    g = np.random.default_rng(seed)
    q0 = g.standard_normal((1, H, S, D)).astype(np.float32)
    k0 = g.standard_normal((1, H, S, D)).astype(np.float32)
    out = [(q0, k0)]
    # pooled means move by `shift` per element in every dim for the first n heads
    for n, shift in ((2, 0.05), (5, 0.05), (9, 0.2), (6, 0.3)):
        q = q0.copy()
        q[0, :n] += shift
        out.append((q, k0))
    return out


def _rank_main(rank, world, port, H, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    from block_sparse_attention_tcgen05_b200.sharding import ShardedMaskCache, head_range
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        S, D, Cq, Ck = 2048, 64, 16, 16
        h0, h1, _, _ = head_range(H, H, world, rank)
        cache = ShardedMaskCache(1, H, h0, h1, Cq, Ck, D, delta=2.0, device="cuda")
        full = oracle.HeadMaskCache(delta=2.0)
        out = []
        for t, (q, k) in enumerate(_steps(H, S, D)):
            want = full.should_refresh(q, k)
            qd = torch.from_numpy(q[:, h0:h1]).contiguous().cuda()
            kd = torch.from_numpy(k[:, h0:h1]).contiguous().cuda()
            got, n_layer = cache.should_refresh(qd, kd)
            got = got.cpu().numpy().astype(bool)
            new = np.random.default_rng(t).random((1, H, Cq, Ck)) < 0.3
            m = cache.update(torch.from_numpy(new[:, h0:h1].astype(np.uint8)).contiguous().cuda())
            ref_m = full.update(new, want)
            out.append((got.tolist(), want[:, h0:h1].tolist(), int(n_layer),
                        bool((m.cpu().numpy().astype(bool) == ref_m[:, h0:h1]).all())))
        import block_sparse_attention_tcgen05_b200 as bsa
        results[rank] = (out, bsa.device_status()[0])
    finally:
        dist.destroy_process_group()


def test_two_rank_layer_gate_on_one_gpu():
    H, world = 10, 2
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, H, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    for r in range(world):
        out, status = results[r]
        assert status == 0
        for t, (got, want, n_layer, mask_ok) in enumerate(out):
            assert got == want, (r, t, got, want, n_layer)
            assert mask_ok, (r, t)
    # the scenario covers the first call, the none / per-head / all branches
    counts = [n for _, _, n, _ in results[0][0]]
    print("layer refresh counts per step:", counts)
