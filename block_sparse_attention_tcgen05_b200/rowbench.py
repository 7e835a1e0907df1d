"""Per-step measurement of the hot path: each step's kernels timed at its workload
sizes, with its algorithmic work and roofline fraction.

    python -m block_sparse_attention_tcgen05_b200.rowbench [--out FILE] [--calls N]

Steps and sizes follow the method's pipeline: pooled drift/gate of the per-head mask
cache and the anti-diagonal block scoring + top-p selection at the video shape
(H=40, S=32760 padded to 32768, D=128, block 128, stride 16, per-head tau); the
labels -> permutation -> gather -> centroid -> bitset stages and the fused
compensated attention at the video-tile workload (245 clusters, nearest 22 % of tile
pairs); probe selection, probe dense attention and the probe-fitted residual repair
at the grouped-query shape (H=24 query heads over 8 KV heads, S=32768, M=64).

Timing: CUDA events on the launching stream, 5 warm-up calls, median of N calls
(default 20), L2 flushed (a 256 MB write) before every timed call. Latency-class steps
also report ms_pipelined: 20 back-to-back calls between one pair of events, which
hides the host-side launch path that a single timed call of a short kernel includes. Peaks come from
MEASURED_PEAKS.json at the repository root (burst figures: each call is timed alone).
All inputs are synthetic and seeded; nothing here computes reference values.
"""

import argparse
import json
import os
import statistics
import time

import torch

from . import ops
from . import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GRID, TILE, D = (21, 30, 52), (3, 6, 8), 128


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class Timer:
    """Median device time of a callable; the L2 flush before each call is not timed."""

    def __init__(self, dev, calls, warmup=5):
        self.dev, self.calls, self.warmup = dev, calls, warmup
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def __call__(self, fn):
        for _ in range(self.warmup):
            fn()
        torch.cuda.synchronize(self.dev)
        ts = []
        for _ in range(self.calls):
            self.flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(self.dev)
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def pipelined(self, fn, n=20):
        """Mean device time of n back-to-back calls between one pair of events (the
        host enqueues ahead of the GPU, so launch overhead is hidden; no L2 flush)."""
        for _ in range(self.warmup):
            fn()
        torch.cuda.synchronize(self.dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize(self.dev)
        return a.elapsed_time(b) / n


def row(step, what, ms, work, unit, bound, peak):
    """One result: work per call in bytes (HBM rows) or FLOP (tensor rows)."""
    if bound == "hbm":
        achieved = work / (ms * 1e-3) / 1e9
        unit_a = "GB/s"
    elif bound == "tensor":
        achieved = work / (ms * 1e-3) / 1e12
        unit_a = "TFLOP/s"
    else:
        achieved, unit_a = None, None
    return {"step": step, "what": what, "ms": ms, "work": work, "work_unit": unit, "bound": bound,
            "achieved": achieved, "unit": unit_a, "peak": peak if achieved is not None else None,
            "frac": achieved / peak if achieved is not None else None}


def video_inputs(dev, H):
    q, k, v = wl.positional_qkv_device(1, H, H, GRID, D, ell=(3.0, 6.0, 8.0), amp=2.0, seed=3,
                                       device=dev)
    return q, k, v


def bench_cache_and_scoring(timer, dev, hbm, tc, out):
    H, S, Sp = 40, 32760, 32768
    q, k, _ = video_inputs(dev, H)
    # a1: pooled means, drift and gate over Q and K of every head (one read of each)
    cache = ops.MaskCache(1, H, Sp // 128, Sp // 128, D, delta=8.0)
    cache.should_refresh(q, k, sync=False)  # first call: anchors
    ms = timer(lambda: cache.should_refresh(q, k, sync=False))
    out.append(row("a1", "mask cache: pooled means, drift, gate (H=40, S=32760)", ms,
                   2 * q.numel() * q.element_size(), "B", "hbm", hbm))
    # a2: anti-diagonal scoring on Q, K zero-padded to a multiple of the block
    qp = torch.zeros((1, H, Sp, D), dtype=q.dtype, device=dev)
    kp = torch.zeros_like(qp)
    qp[:, :, :S] = q
    kp[:, :, :S] = k
    del q, k
    stride = 16
    ms = timer(lambda: ops.antidiagonal_block_scores(qp, kp, block=128, stride=stride))
    flop = 2.0 * Sp * Sp * D / stride * H
    out.append(row("a2", "anti-diagonal block scores (H=40, S=32768, D=128, stride 16)", ms, flop,
                   "FLOP", "tensor", tc))
    r = out[-1]
    r["hbm_gbs"] = 2 * qp.numel() * qp.element_size() / (ms * 1e-3) / 1e9
    # a3: top-p with tau per head from {0.85, 0.90, 0.95}
    scores = ops.antidiagonal_block_scores(qp, kp, block=128, stride=stride)
    tau = torch.tensor([(0.85, 0.90, 0.95)[h % 3] for h in range(H)], dtype=torch.float32,
                       device=dev)
    ms = timer(lambda: ops.top_p_block_mask(scores, tau))
    out.append(row("a3", "top-p block mask (1x40x256x256 scores)", ms, None, None, "latency", None))
    out[-1]["ms_pipelined"] = timer.pipelined(lambda: ops.top_p_block_mask(scores, tau))
    del qp, kp, scores


def bench_attention(timer, dev, hbm, tc, out):
    import ctypes

    from . import _lib
    H, S = 40, 32760
    q, k, v = video_inputs(dev, H)
    labels, C = ops.tile_labels(*GRID, TILE, device=dev)
    mask = torch.tensor(wl.nearest_pair_mask(wl.tile_centroids(GRID, TILE), 0.22),
                        dtype=torch.uint8, device=dev)
    ws = torch.empty(ops.attention_workspace_bytes(q, k, C, C), dtype=torch.uint8, device=dev)
    o = torch.empty((1, H, S, D), dtype=torch.float32, device=dev)
    cnt = torch.bincount(labels.long(), minlength=C).double()
    pairs = float(cnt @ mask.double() @ cnt) * H

    def call():
        ops.centroid_compensated_attention(q, k, v, labels, labels, mask, Cq=C, Ck=C, out=o,
                                           workspace=ws)
    _lib.call("bsa_profile_enable", timer.calls + timer.warmup)
    ms = timer(call)
    kms, kn = ctypes.c_float(0.0), ctypes.c_int(0)
    _lib.call("bsa_profile_read", 0, ctypes.byref(kms), ctypes.byref(kn))
    _lib.call("bsa_profile_enable", 0)
    kernel_ms = kms.value / max(1, kn.value)
    prep_ms = max(ms - kernel_ms, 1e-6)
    # Q is not copied (the attention kernel gathers its tile's rows by TMA): the bytes
    # that must cross HBM are one read and one write of K and V
    kv_bytes = 2 * k.numel() * k.element_size()
    out.append(row("a4-a7", "key cluster order, label sorts, query tile plan, cluster-major K/V "
                   "gather, centroids, mask bitsets (call minus attention kernel)", prep_ms,
                   2 * kv_bytes, "B", "hbm", hbm))
    out.append(row("a8", f"fused compensated attention kernel ({pairs:.3e} executed pairs x 4D)",
                   kernel_ms, pairs * 4 * D, "FLOP", "tensor", tc))
    out.append(row("a4-a8", "whole attention call", ms, pairs * 4 * D, "FLOP", "tensor", tc))
    # the same call reusing the label sorts, key order, tile plan and bitsets of the
    # previous call on the workspace (labels and mask unchanged, as across denoising
    # steps whose mask cache refreshes no head): only the K/V gather and centroids remain

    def reuse_call():
        ops.centroid_compensated_attention(q, k, v, labels, labels, mask, Cq=C, Ck=C, out=o,
                                           workspace=ws, reuse_plan=True)
    call()
    _lib.call("bsa_profile_enable", timer.calls + timer.warmup)
    ms_r = timer(reuse_call)
    _lib.call("bsa_profile_read", 0, ctypes.byref(kms), ctypes.byref(kn))
    _lib.call("bsa_profile_enable", 0)
    kernel_r = kms.value / max(1, kn.value)
    out.append(row("a4-a7 reused", "K/V gather and centroids only: preparation of a call that "
                   "reuses the previous call's plan (call minus attention kernel)",
                   max(ms_r - kernel_r, 1e-6), 2 * kv_bytes, "B", "hbm", hbm))
    out.append(row("a4-a8 reused", "whole attention call reusing the plan", ms_r, pairs * 4 * D,
                   "FLOP", "tensor", tc))
    # context: the same call with every tile pair kept (dense attention through the same
    # kernel); its time over the sparse call's is the sparse path's speedup
    full = torch.ones_like(mask)

    def dense_call():
        ops.centroid_compensated_attention(q, k, v, labels, labels, full, Cq=C, Ck=C, out=o,
                                           workspace=ws)
    dense_ms = timer(dense_call)
    out.append(row("a4-a8 dense", "the same call with every tile pair kept (context)", dense_ms,
                   float(H) * S * S * 4 * D, "FLOP", "tensor", tc))
    out[-1]["speedup_of_sparse_call"] = dense_ms / ms


def fp32_alu_tflops(dev):
    """CUDA-core fp32 peak of the part: SMs x 128 FMA lanes x 2 FLOP x the maximum SM
    clock (for kernels that run on the FMA pipe rather than the tensor cores)."""
    props = torch.cuda.get_device_properties(dev)
    mhz = 1965.0
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    return props.multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12


def bench_routing_and_sta(timer, dev, hbm, tc, out):
    H = 40
    q, k, v = video_inputs(dev, H)
    labels, C = ops.tile_labels(*GRID, TILE, device=dev)
    S = q.shape[2]
    # f1: SVG-EAR error-aware routing at density 0.22: the probe kernel computes, per
    # head, every query cluster's mean query against every key (logits and the
    # exp-weighted values): 4 D FLOP per (probe, key) pair, on the tensor cores with
    # both operands that are not bf16-exact carried as two bf16 parts (the executed
    # MMA work is about twice this, plus 16-key padding of each cluster's last piece)
    ws = torch.empty(ops._lib.load().bsa_routing_workspace_bytes(ops.make_shape(q, k), C, C),
                     dtype=torch.uint8, device=dev)
    ms = timer(lambda: ops.error_aware_block_mask(q, k, v, labels, labels, C, C, 0.22,
                                                  workspace=ws))
    out.append(row("f1", "SVG-EAR error-aware routing (H=40, 245 probes per head over 32760 "
                   "keys, density 0.22; whole call: sorts, gathers and means, centroid "
                   "logits, probe kernel, normalisation, selection)", ms,
                   4.0 * D * C * S * H, "FLOP", "tensor", tc))
    # f3: the recipe's sliding-tile window mask, (3, 3, 5) tiles, driving the attention
    n_tiles = tuple(-(-g // t) for g, t in zip(GRID, TILE))
    mask = ops.sliding_tile_block_mask(n_tiles, (3, 3, 5), device=dev)
    ws = torch.empty(ops.attention_workspace_bytes(q, k, C, C), dtype=torch.uint8, device=dev)
    o = torch.empty((1, H, S, D), dtype=torch.float32, device=dev)
    cnt = torch.bincount(labels.long(), minlength=C).double()
    pairs = float(cnt @ mask.double() @ cnt) * H
    ms = timer(lambda: ops.centroid_compensated_attention(q, k, v, labels, labels, mask, Cq=C, Ck=C,
                                                          out=o, workspace=ws))
    out.append(row("f3", "compensated attention call on the sliding-tile (3,3,5) window mask "
                   f"({pairs / (H * S * S):.3f} of token pairs)", ms, pairs * 4 * D, "FLOP",
                   "tensor", tc))


def bench_partition(timer, dev, hbm, tc, out):
    """f2 at the grouped-query shape: response-coupled partition of 24 query heads over 8 KV
    heads, S=32768, 256 query and key groups; and the probe-budget router on the result's
    first KV head labels (all 24 heads, density 0.22, M=64)."""
    Hq, Hkv, S = 24, 8, 32768
    g = torch.Generator(device=dev).manual_seed(4)
    q = torch.randn((1, Hq, S, D), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((1, Hkv, S, D), generator=g, device=dev).to(torch.bfloat16)
    C = S // 128
    ws = torch.empty(ops._lib.load().bsa_partition_workspace_bytes(ops.make_shape(q, k), C, C, 48, 64),
                     dtype=torch.uint8, device=dev)
    ms = timer(lambda: ops.response_coupled_partition(q, k, C, C, workspace=ws))
    # FMA-pipe work: key features 2 rK D per key, 9 k-means assignments of 2 C rK per key,
    # query coordinates 2 rQ G D per query row, 9 assignments of 2 C rQ G per query row
    G = Hq // Hkv
    flop = Hkv * S * (2 * 48 * D + 9 * 2 * C * 48 + 2 * 64 * G * D + 9 * 2 * C * 64 * G)
    r = row("f2", "response-coupled partition (24 query / 8 KV heads, S=32768, 256 + 256 groups, "
            "8 k-means rounds)", ms, flop, "FLOP", "alu", None)
    alu = fp32_alu_tflops(dev)
    r.update({"achieved": flop / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "peak": alu,
              "frac": flop / (ms * 1e-3) / 1e12 / alu,
              "peak_note": "fp32 FMA pipe: SMs x 128 lanes x 2 x max SM clock"})
    out.append(r)
    ql, kl = ops.response_coupled_partition(q, k, C, C, workspace=ws)
    qlab, klab = ql[0, 0].contiguous(), kl[0, 0].contiguous()
    ms = timer(lambda: ops.probe_budget_block_mask(q, k, qlab, klab, C, C, 0.22, 64))
    out.append(row("f2r", "probe-budget router (24 heads, 256 x 256 cells, density 0.22, M=64)", ms,
                   None, None, "latency", None))


def bench_probe_and_repair(timer, dev, hbm, tc, out):
    Hq, Hkv, S, M = 24, 8, 32768, 64
    g = torch.Generator(device=dev).manual_seed(4)
    q = torch.randn((1, Hq, S, D), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((1, Hkv, S, D), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((1, Hkv, S, D), generator=g, device=dev).to(torch.bfloat16)
    labels = (torch.arange(S, device=dev) // 128).to(torch.int32)
    C = S // 128
    ms = timer(lambda: ops.select_probe_rows(labels, C, M, q=q))
    out.append(row("a9", "probe selection, nearest-to-centroid members (H=24, 256 clusters, M=64)",
                   ms, None, None, "latency", None))
    out[-1]["ms_pipelined"] = timer.pipelined(lambda: ops.select_probe_rows(labels, C, M, q=q))
    idx, w = ops.select_probe_rows(labels, C, M, q=q)
    ws = torch.empty(ops._lib.load().bsa_probe_attention_workspace_bytes(ops.make_shape(q, k), M),
                     dtype=torch.uint8, device=dev)
    ms = timer(lambda: ops.probe_dense_attention(q, k, v, idx, workspace=ws))
    out.append(row("a10", "probe dense attention (24 heads x 64 rows over 32768 keys)", ms,
                   4.0 * D * M * S * Hq, "FLOP", "tensor", tc))
    o_probe = ops.probe_dense_attention(q, k, v, idx, workspace=ws)
    del q, k, v
    o = torch.randn((1, Hq, S, D), generator=g, device=dev) * 0.1
    rws = torch.empty(ops._lib.load().bsa_repair_workspace_bytes(1, Hq, S, D, M),
                      dtype=torch.uint8, device=dev)
    ms = timer(lambda: ops.probe_residual_correction(o, o_probe, idx, w, workspace=rws))
    out.append(row("a11-a14", "probe-fitted residual repair: column stats, normal equations, "
                   "Cholesky, top-16 subspace, rank-16 apply (out 1x24x32768x128 fp32)", ms,
                   3 * o.numel() * o.element_size(), "B", "hbm", hbm))


def main():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--calls", type=int, default=20)
    p.add_argument("--out", default=None, help="also write the JSON lines to this file")
    p.add_argument("--only", default=None,
                   help="comma-separated groups to run (cache_scoring, attention, routing, "
                        "partition, probe_repair); default all")
    args = p.parse_args()
    groups = set(args.only.split(",")) if args.only else None
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm, tc, src = peaks()
    timer = Timer(dev, args.calls)
    out = []
    t0 = time.time()
    for name, fn in (("cache_scoring", bench_cache_and_scoring), ("attention", bench_attention),
                     ("routing", bench_routing_and_sta), ("partition", bench_partition),
                     ("probe_repair", bench_probe_and_repair)):
        if groups is None or name in groups:
            fn(timer, dev, hbm, tc, out)
            torch.cuda.empty_cache()
    st, _ = ops.device_status(dev)
    if st != 0:
        raise RuntimeError(f"device status {st}")
    lines = [json.dumps(dict(r, peak_source=src)) for r in out]
    print("\n".join(lines))
    print(f"# {len(out)} rows in {time.time() - t0:.1f} s; peaks: HBM {hbm} GB/s, bf16 {tc} TFLOP/s "
          f"({src}, burst)")
    if args.out:
        with open(args.out, "w") as f:
            f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
