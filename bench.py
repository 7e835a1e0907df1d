#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

Workload: the video-DiT shape with static tiles — B=1, H=40, S=32760 tokens on a
21 x 30 x 52 latent grid, D=128, bf16 Q/K/V with a 3-D positional structure; labels
from 3 x 6 x 8 sliding tiles (245 clusters); the tile-level mask keeps the 22 % of
tile pairs nearest in (t, h, w); skipped tiles are centroid-compensated.
One step = tile_labels + centroid_compensated_attention (label sort, Q gather, K/V
gather with centroids, mask bitsets, fused tcgen05 attention) over one batch.

Metric: effective TFLOP/s on executed pairs (4·D FLOP per token pair inside kept
blocks; centroid terms not counted), with ms per call and % of the measured bf16
tensor peak. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own copy of the workload (weak scaling: the path
shards by heads and needs no collective); the step time is the max over ranks.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GRID = (21, 30, 52)
TILE = (3, 6, 8)
H = 40
D = 128
DENSITY = 0.22
WORKLOAD = ("video_static_tiles: B=1 H=40 S=32760 (21x30x52) D=128 bf16, 3x6x8 tile labels "
            "(245 clusters), nearest-22% tile-pair mask, SVG-EAR compensation")
STA_WINDOW = (3, 3, 5)
WORKLOAD_STA = ("video_static_tiles_sta: B=1 H=40 S=32760 (21x30x52) D=128 bf16, 3x6x8 tile "
                "labels (245 clusters), sliding-tile window (3,3,5) tiles (19% of token pairs), "
                "SVG-EAR compensation")
METRIC = "effective TFLOP/s on executed pairs, centroid-compensated block-sparse attention at 40x32760x128"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="bounded CPU work for the oracle baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--mask", choices=["nearest", "sta"], default="nearest",
                   help="nearest: the 22 %% of tile pairs nearest in (t, h, w) (default); sta: "
                        "the recipe's sliding-tile window of STA_WINDOW tiles")
    p.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                   help="replicas: every rank runs the whole workload (weak scaling, default); "
                        "heads: the layer's 40 heads are split over the ranks (strong scaling)")
    p.add_argument("--heads", type=int, default=H,
                   help="number of heads (default 40; smaller only for profiler captures)")
    return p.parse_args()


def max_over_ranks(values, device, world):
    """Element-wise maximum of per-rank timings over all ranks (every rank gets it):
    a multi-GPU step is as slow as its slowest rank."""
    if world <= 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_tflops(flop_per_rank, world, ms):
    """Whole-job throughput: every rank processes its own copy of the workload."""
    return world * flop_per_rank / (ms * 1e-3) / 1e12


def job_flop(flop_local, heads_local, heads_layer, world, shard):
    """FLOPs of the whole job: N copies of the workload (replicas) or the one layer whose
    heads the ranks share (heads)."""
    if shard == "heads":
        return flop_local / heads_local * heads_layer
    return flop_local * world


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return m, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def roofline_peak(peaks, region_s):
    """The bf16 peak a kernel timed inside a region of ``region_s`` seconds is held to:
    the burst figure for a region shorter than the seconds-long loop the sustained
    figure was measured over (the clocks have not settled under the power cap yet),
    the sustained one otherwise. Returns (key, TFLOP/s)."""
    key = "bf16_tflops" if region_s < 2.0 else "bf16_tflops_sustained"
    return key, float(peaks.get(key, peaks.get("bf16_tflops")))


ATTN_SECTION = b"// ============================================================== attention kernel"


def attention_source_hash():
    """Hash of the source that decides the attention kernel's DRAM traffic: attention.cu
    from the kernel's section to the end (the kernel, its helpers and its launch code;
    the label sorts, mask bitsets and gathers above it are separate kernels) and the
    PTX wrappers it uses."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "block_sparse_attention_tcgen05_b200", "csrc")
    with open(os.path.join(d, "attention.cu"), "rb") as f:
        src = f.read()
    h.update(src[src.index(ATTN_SECTION):])
    with open(os.path.join(d, "ptx.cuh"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the attention kernel from the committed ncu summary,
    or None when the kernel source changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_sha") != attention_source_hash():
        return None
    return rec.get("bytes_per_launch_full_workload")


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait (up to 3 s) for its first sample so
        # that the samples cover the timed region.
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.proc.poll() is None:
            if os.path.getsize(self.file.name) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        self.file.close()
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(q, k, v, labels, mask, seconds):
    """The oracle, as it stands, on the host cores over a bounded sample of the same
    workload: head 0, query rows in chunks of 512 until ``seconds`` of work."""
    import numpy as np

    import oracle
    cores = len(os.sched_getaffinity(0))
    qd = q[:, :1].double().cpu().numpy()
    kd = k[:, :1].double().cpu().numpy()
    vd = v[:, :1].double().cpu().numpy()
    lab = labels.cpu().numpy().astype(np.int64)
    m = mask.cpu().numpy().astype(bool)
    cnt = np.bincount(lab, minlength=m.shape[1])
    kept_keys = (m[lab].astype(np.int64) * cnt[None, :]).sum(1)  # per query row
    order = np.random.default_rng(0).permutation(len(lab))
    t0 = time.perf_counter()
    done, pairs = 0, 0
    while done < len(order) and time.perf_counter() - t0 < seconds:
        rows = np.sort(order[done:done + 512])
        oracle.centroid_compensated_attention(qd, kd, vd, lab, lab, m, rows=rows,
                                              Cq=m.shape[0], Ck=m.shape[1])
        pairs += int(kept_keys[rows].sum())
        done += len(rows)
    dt = time.perf_counter() - t0
    return {"value": pairs * 4 * D / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"head 0, {done} of {len(lab)} query rows (random, in chunks of 512), "
                      f"{pairs:.3e} executed pairs in {dt:.1f} s, float64 NumPy",
            "seconds": round(dt, 2)}


def run_reference(args, rank):
    """--impl reference: the oracle on the host cores, each step a bounded sample."""
    if rank != 0:
        return
    import numpy as np

    import oracle
    from block_sparse_attention_tcgen05_b200 import workloads as wl
    q, k, v, _ = wl.positional_qkv(1, 1, 1, GRID, D, ell=(3.0, 6.0, 8.0), amp=2.0, dtype="bf16",
                                   seed=3)
    lab, C = oracle.tile_labels(*GRID, TILE)
    mask = wl.nearest_pair_mask(wl.tile_centroids(GRID, TILE), DENSITY)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    cnt = np.bincount(lab, minlength=C)
    kept_keys = (mask[lab].astype(np.int64) * cnt[None, :]).sum(1)
    rng = np.random.default_rng(1)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    times, pair_counts = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        pairs = 0
        while time.perf_counter() - t0 < per_step:
            rows = np.sort(rng.choice(len(lab), 256, replace=False))
            oracle.centroid_compensated_attention(qd, kd, vd, lab, lab, mask, rows=rows, Cq=C, Ck=C)
            pairs += int(kept_keys[rows].sum())
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
            pair_counts.append(pairs)
    value = sum(pair_counts) * 4 * D / sum(times) / 1e12
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_per_step": "random 256-row chunks of head 0 "
                   f"for ~{per_step:.1f} s"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"head 0 of 40, random query rows, {sum(pair_counts):.3e} "
                                   "executed pairs over the timed steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import ctypes

    import torch
    import torch.distributed as dist

    import block_sparse_attention_tcgen05_b200 as bsa
    from block_sparse_attention_tcgen05_b200 import _lib
    from block_sparse_attention_tcgen05_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    lib = _lib.load()

    # ---------------------------------------------------------------- inputs (HBM-resident)
    nh = args.heads
    seed = 3 + 1000 * rank
    if args.shard == "heads":
        # this rank's heads of the one layer (KV-aligned ranges; no exchange of data)
        from block_sparse_attention_tcgen05_b200.sharding import head_range
        h0, h1, _, _ = head_range(args.heads, args.heads, world, rank)
        nh, seed = h1 - h0, 3 + h0
    q, k, v = wl.positional_qkv_device(1, nh, nh, GRID, D, ell=(3.0, 6.0, 8.0), amp=2.0,
                                       seed=seed, device=dev)
    labels, C = bsa.tile_labels(*GRID, TILE, device=dev)
    if args.mask == "sta":
        n_tiles = tuple(-(-g // t) for g, t in zip(GRID, TILE))
        mask = bsa.sliding_tile_block_mask(n_tiles, STA_WINDOW, device=dev)
    else:
        mask = torch.as_tensor(wl.nearest_pair_mask(wl.tile_centroids(GRID, TILE), DENSITY),
                               dtype=torch.uint8, device=dev)
    cnt = torch.bincount(labels.long(), minlength=C).double()
    pairs = float(cnt @ mask.double() @ cnt) * nh
    S = q.shape[2]
    flop = pairs * 4 * D
    ws = torch.empty(bsa.attention_workspace_bytes(q, k, C, C), dtype=torch.uint8, device=dev)
    out = torch.empty((1, nh, S, D), dtype=torch.float32, device=dev)

    def step():
        lab, _ = bsa.tile_labels(*GRID, TILE, device=dev)
        bsa.centroid_compensated_attention(q, k, v, lab, lab, mask, Cq=C, Ck=C, out=out, workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, _ = bsa.device_status(dev)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---------------------------------------------------------------- timed region
    _lib.call("bsa_profile_enable", args.steps)
    uuid = getattr(torch.cuda.get_device_properties(dev), "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local))
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    n0 = lib.bsa_launch_count()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    launches = int(lib.bsa_launch_count() - n0)
    ms = e0.elapsed_time(e1) / args.steps
    attn_ms = ctypes.c_float(0.0)
    attn_n = ctypes.c_int(0)
    _lib.call("bsa_profile_read", 0, ctypes.byref(attn_ms), ctypes.byref(attn_n))
    _lib.call("bsa_profile_enable", 0)
    attn_ms_launch = attn_ms.value / max(1, attn_n.value)
    ms, attn_ms_launch = max_over_ranks([ms, attn_ms_launch], dev, world)
    st, _ = bsa.device_status(dev)
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        mh = mask.cpu().pin_memory()
        oh = torch.empty((1, nh, S, D), dtype=torch.float32).pin_memory()
        # Two device copies of a step's inputs and output: step i computes on set i % 2
        # while the upload of step i + 1 and the download of step i - 1 run on their own
        # streams (PCIe carries both directions at once). Every step's upload and
        # download lies inside the timed region.
        sets = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                     m=torch.empty_like(mask), o=torch.empty_like(out)) for _ in range(2)]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        up = [torch.cuda.Event() for _ in range(2)]    # upload into set j done
        done = [torch.cuda.Event() for _ in range(2)]  # compute on set j done
        down = [torch.cuda.Event() for _ in range(2)]  # download of set j's output done

        def upload(i):
            b = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[i % 2])  # step i - 2 no longer reads this set
                for key, h in (("q", qh), ("k", kh), ("v", vh), ("m", mh)):
                    b[key].copy_(h, non_blocking=True)
                up[i % 2].record(s_in)

        def compute(i):
            b = sets[i % 2]
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up[i % 2])
                if i >= 2:
                    s_cmp.wait_event(down[i % 2])  # step i - 2's output has been read
                lab, _ = bsa.tile_labels(*GRID, TILE, device=dev)
                bsa.centroid_compensated_attention(b["q"], b["k"], b["v"], lab, lab, b["m"],
                                                   Cq=C, Ck=C, out=b["o"], workspace=ws)
                done[i % 2].record(s_cmp)

        def download(i):
            b = sets[i % 2]
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i % 2])
                oh.copy_(b["o"], non_blocking=True)
                down[i % 2].record(s_out)

        def run(n):
            upload(0)
            for i in range(n):
                if i + 1 < n:
                    upload(i + 1)
                compute(i)
                download(i)

        run(2)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        run(args.steps)
        b.record(s_out)  # the last download follows every compute and upload
        torch.cuda.synchronize()
        barrier()
        e2e_ms = a.elapsed_time(b) / args.steps
        (e2e_ms,) = max_over_ranks([e2e_ms], dev, world)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, mh))
        d2h = oh.numel() * oh.element_size()
        e2e = {"value": job_flop(flop, nh, args.heads, world, args.shard) / (e2e_ms * 1e-3) / 1e12,
               "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "block_sparse_attention_tcgen05_b200.centroid_compensated_attention",
               "overlap": "upload of step i+1 and download of step i-1 on their own streams "
                          "during step i (double-buffered device tensors)"}
        del qh, kh, vh, oh, sets

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(q, k, v, labels, mask, args.cpu_seconds)

    if rank == 0:
        peaks, src = measured_peaks()
        peak_key, peak = roofline_peak(peaks, ms * args.steps * 1e-3)
        achieved = flop / (attn_ms_launch * 1e-3) / 1e12
        line = {
            "metric": METRIC,
            "value": job_flop(flop, nh, args.heads, world, args.shard) / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "ms_per_call": ms,
            "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "pct_of_bf16_peak": 100.0 * (flop / (ms * 1e-3) / 1e12) / peak,
            "pct_of_bf16_peak_basis": peak_key,
            "config": {
                "workload": WORKLOAD_STA if args.mask == "sta" else WORKLOAD,
                "B": 1, "H": nh, "S": S, "D": D, "clusters": C,
                "executed_pairs_per_call": pairs,
                "executed_pair_density": pairs / (nh * S * S),
                "flop_per_call": flop,
                "l2": "inputs larger than L2 (Q+K+V = %.2f GB per rank)" % (
                    3 * q.numel() * 2 / 1e9),
                "parallelism": ("heads split over %d ranks (strong, no collective on the data path)"
                                if args.shard == "heads" else
                                "replicas x%d (weak, no collective on the data path)") % world,
            },
            "roofline": {
                "kernel": "attn_kernel<128,bf16>",
                "bound": "tensor",
                "achieved": achieved,
                "peak": peak,
                "peak_source": f"{peak_key} of {src} (MEASURED_PEAKS.json); timed region "
                               f"{ms * args.steps:.0f} ms"
                if src == "measured" else f"fallback {peak_key}",
                "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": recorded_traffic(),
                "ms_per_launch": attn_ms_launch,
            },
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
