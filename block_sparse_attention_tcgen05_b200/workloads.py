"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module only draws random numbers and builds the caller-side inputs of the
video-DiT workloads (Q/K/V with positional structure, caller-chosen block masks,
drift sequences). It holds none of the method's arithmetic: no attention, scoring,
labels, probe selection or repair. Everything is generated in float64 on the CPU and
cast to the workload dtype (round to nearest even), so the oracle and the CUDA path
see the same values.

Workload recipes (video-DiT stand-ins; no model, prompt or dataset is used):
* Gaussian Q/K/V ~ N(0, 1).
* Positional structure: a sinusoid p(x)_j = amp · sin(ω_j · x + φ_j) added to both Q
  and K of a head, with ω_j ~ N(0, diag(ℓ⁻²)) and φ_j ~ U[0, 2π) drawn per head. Its
  expected inner product amp²·D/2 · exp(−½ Σ (Δ_i / ℓ_i)²) decays with the
  spatiotemporal distance Δ, so attention mass concentrates near the diagonal.
* Block masks a caller would build: a seeded random cluster mask with the diagonal
  kept, and the "nearest pairs" static mask keeping every (query tile, key tile)
  pair whose centroid distance is within the smallest radius reaching a density.
"""

import math

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _rng(seed):
    return np.random.default_rng(seed)


def to_dtype(x64, dtype):
    """Cast a float64 array to the workload dtype as a CPU tensor (RNE)."""
    return torch.from_numpy(np.ascontiguousarray(x64)).to(DTYPES[dtype])


def gaussian_qkv(B, Hq, Hkv, S, D, dtype="bf16", seed=0):
    """Q (B,Hq,S,D), K and V (B,Hkv,S,D) with i.i.d. N(0,1) entries."""
    g = _rng(seed)
    q = g.standard_normal((B, Hq, S, D))
    k = g.standard_normal((B, Hkv, S, D))
    v = g.standard_normal((B, Hkv, S, D))
    return to_dtype(q, dtype), to_dtype(k, dtype), to_dtype(v, dtype)


def grid_coords(grid):
    """(S, len(grid)) float64 coordinates of tokens in raster order."""
    axes = [np.arange(n, dtype=np.float64) for n in grid]
    mesh = np.meshgrid(*axes, indexing="ij")
    return np.stack([m.reshape(-1) for m in mesh], axis=1)


def _positional(g, coords, D, ell, amp):
    ell = np.asarray(ell, dtype=np.float64).reshape(1, -1)
    omega = g.standard_normal((D, coords.shape[1])) / ell
    phi = g.uniform(0.0, 2.0 * math.pi, size=D)
    return amp * np.sin(coords @ omega.T + phi[None, :])


def positional_qkv(B, Hq, Hkv, grid, D, ell, amp=2.0, dtype="bf16", seed=0,
                   temperature_range=None):
    """Q, K = N(0,1) + positional sinusoid over ``grid`` (1-D or 3-D), V ~ N(0,1).

    The positional term of query head h is the one of its KV head, so the structure
    is shared under grouped-query attention. With ``temperature_range=(lo, hi)``
    each query head is divided by T_h ~ U[lo, hi]. Returns (q, k, v, temperatures).
    """
    g = _rng(seed)
    coords = grid_coords(grid)
    S = coords.shape[0]
    grp = Hq // Hkv
    k = np.empty((B, Hkv, S, D))
    q = np.empty((B, Hq, S, D))
    for b in range(B):
        for hk in range(Hkv):
            pos = _positional(g, coords, D, ell, amp)
            k[b, hk] = g.standard_normal((S, D)) + pos
            for j in range(grp):
                q[b, hk * grp + j] = g.standard_normal((S, D)) + pos
    v = g.standard_normal((B, Hkv, S, D))
    temps = None
    if temperature_range is not None:
        temps = g.uniform(temperature_range[0], temperature_range[1], size=Hq)
        q = q / temps[None, :, None, None]
    return to_dtype(q, dtype), to_dtype(k, dtype), to_dtype(v, dtype), temps


def random_cluster_mask(C, density, seed=0):
    """(C, C) bool mask with the diagonal kept and extra off-diagonal entries drawn
    without replacement so that round(density · C²) entries are kept."""
    g = _rng(seed)
    m = np.eye(C, dtype=bool)
    want = int(round(density * C * C)) - C
    off = np.flatnonzero(~m.reshape(-1))
    pick = g.choice(off, size=max(want, 0), replace=False)
    m.reshape(-1)[pick] = True
    return m


def tile_centroids(grid, tile):
    """Mean token coordinate of each tile of ``grid`` cut into ``tile``-sized boxes
    (edge tiles partial), in raster order of tiles (t-tile major, then h, then w)."""
    T, H, W = grid
    tt, th, tw = tile
    nT, nH, nW = -(-T // tt), -(-H // th), -(-W // tw)
    cents = np.zeros((nT * nH * nW, 3))
    for it in range(nT):
        for ih in range(nH):
            for iw in range(nW):
                t = np.arange(it * tt, min(T, (it + 1) * tt))
                h = np.arange(ih * th, min(H, (ih + 1) * th))
                w = np.arange(iw * tw, min(W, (iw + 1) * tw))
                cents[(it * nH + ih) * nW + iw] = (t.mean(), h.mean(), w.mean())
    return cents


def raster_block_centroids(grid, block):
    """Mean token coordinate of each run of ``block`` consecutive raster tokens."""
    c = grid_coords(grid)
    S = c.shape[0]
    nb = -(-S // block)
    return np.stack([c[i * block:min(S, (i + 1) * block)].mean(axis=0) for i in range(nb)])


def nearest_pair_mask(centroids, density):
    """Keep every pair (a, c) with ‖x_a − x_c‖ ≤ d*, d* the smallest pair distance at
    which at least ``density`` of all pairs are kept. Symmetric, diagonal kept."""
    x = np.asarray(centroids, dtype=np.float64)
    d = np.sqrt(((x[:, None, :] - x[None, :, :]) ** 2).sum(-1))
    flat = np.sort(d.reshape(-1))
    need = int(math.ceil(density * flat.size))
    dstar = flat[need - 1]
    return d <= dstar + 1e-9


def drift_steps(q0, k0, steps, sigma, boosted_heads, boost, seed=0):
    """Yield (q_t, k_t) for t = 0..steps-1 with cumulative i.i.d. N(0, σ²) drift per
    element and step (σ·boost on ``boosted_heads``), added to the float64 values of
    q0 / k0 and cast back to their dtype."""
    g = _rng(seed)
    dtype = "bf16" if q0.dtype == torch.bfloat16 else "f32"
    q = q0.double().numpy().copy()
    k = k0.double().numpy().copy()
    sig = np.full(q.shape[1], sigma)
    sig[list(boosted_heads)] *= boost
    for t in range(steps):
        if t > 0:
            q += g.standard_normal(q.shape) * sig[None, :, None, None]
            k += g.standard_normal(k.shape) * sig[None, :, None, None]
        yield to_dtype(q, dtype), to_dtype(k, dtype)


def positional_qkv_device(B, Hq, Hkv, grid, D, ell, amp=2.0, seed=0, device="cuda",
                          dtype=torch.bfloat16):
    """The ``positional_qkv`` recipe drawn with torch's generator on ``device`` (fast at
    full video size; the stream of random numbers differs from the NumPy one, the
    distribution and structure are the same)."""
    g = torch.Generator(device=device).manual_seed(seed)
    axes = [torch.arange(n, dtype=torch.float32, device=device) for n in grid]
    mesh = torch.meshgrid(*axes, indexing="ij")
    coords = torch.stack([m.reshape(-1) for m in mesh], dim=1)
    S = coords.shape[0]
    ellt = torch.tensor(ell, dtype=torch.float32, device=device).reshape(1, -1)
    grp = Hq // Hkv
    q = torch.empty((B, Hq, S, D), dtype=dtype, device=device)
    k = torch.empty((B, Hkv, S, D), dtype=dtype, device=device)
    v = torch.empty((B, Hkv, S, D), dtype=dtype, device=device)
    for b in range(B):
        for hk in range(Hkv):
            omega = torch.randn((D, coords.shape[1]), generator=g, device=device) / ellt
            phi = torch.rand((D,), generator=g, device=device) * (2.0 * math.pi)
            pos = amp * torch.sin(coords @ omega.T + phi[None, :])
            k[b, hk] = (torch.randn((S, D), generator=g, device=device) + pos).to(dtype)
            v[b, hk] = torch.randn((S, D), generator=g, device=device).to(dtype)
            for j in range(grp):
                q[b, hk * grp + j] = (torch.randn((S, D), generator=g, device=device) + pos).to(dtype)
    return q, k, v
