"""Torch-facing wrappers of the libbsa C ABI.

Argument marshalling only: tensors are checked, outputs and workspaces are allocated
with torch on the tensors' device, and every step runs in libbsa's CUDA kernels on the
current torch stream. There is no CPU path.
"""

import ctypes
import weakref

import torch

from . import _lib
from ._lib import BSA_BF16, BSA_F32, Shape, call

_DT = {torch.bfloat16: BSA_BF16, torch.float32: BSA_F32}


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need_cuda(*ts):
    """Every tensor passed to one call must sit on one device (the library launches on
    the current device and reads its arguments as plain pointers: a tensor on another
    GPU would be read through a peer address without peer access), be a CUDA tensor and
    be contiguous."""
    present = [t for t in ts if t is not None]
    devs = {t.device for t in present}
    if len(devs) > 1:
        raise ValueError(f"all tensors of one call must be on the same device, got "
                         f"{sorted(str(d) for d in devs)}")
    for t in present:
        if not t.is_cuda:
            raise ValueError("libbsa operates on CUDA tensors only")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _call_on(dev, name, *args):
    """Call an entry point with ``dev`` as the current CUDA device, so that the library
    launches on the device whose stream it is given."""
    with torch.cuda.device(dev):
        return call(name, *args)


def _expect(t, name, dtypes=None, ndims=None, shape=None):
    """Dtype and shape checks made before anything reaches the C ABI, which takes plain
    pointers: a tensor of the wrong element type or size would be read or written past
    its end there."""
    if t is None:
        raise ValueError(f"{name} is required")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {list(dtypes)}")
    if ndims is not None and t.dim() not in ndims:
        raise ValueError(f"{name}: {t.dim()} dimensions, expected {list(ndims)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _expect_qkv(q, k, v=None):
    """q (B,Hq,Sq,D), k and v (B,Hkv,Sk,D), one element type (bf16 or fp32)."""
    _expect(q, "q", tuple(_DT), (4,))
    _expect(k, "k", (q.dtype,), (4,))
    B, Hq, _, D = q.shape
    if k.shape[0] != B or k.shape[3] != D or k.shape[1] <= 0 or Hq % k.shape[1]:
        raise ValueError(f"k: shape {tuple(k.shape)} does not fit q {tuple(q.shape)}")
    if v is not None:
        _expect(v, "v", (q.dtype,), (4,), tuple(k.shape))


def _expect_workspace(workspace):
    if workspace is not None:
        _expect(workspace, "workspace", (torch.uint8,), (1,))


def _workspace(nbytes, dev):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)


def make_shape(q, k):
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if q.dtype not in _DT or k.dtype != q.dtype:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return Shape(B, Hq, Hkv, Sq, Sk, D, _DT[q.dtype])


def device_status(dev=None):
    """Synchronise the current stream and return (status, site) of the device status
    word (status 0 = no bounded wait has timed out since the last read)."""
    dev = dev or torch.device("cuda", torch.cuda.current_device())
    where = ctypes.c_int(0)
    st = _lib.load().bsa_get_device_status(_stream(dev), ctypes.byref(where))
    return st, where.value


def tile_labels(T, H, W, tile, device="cuda"):
    """Labels of a T×H×W token grid cut into ``tile`` boxes: (int32 (T·H·W,), n_tiles)."""
    labels = torch.empty(T * H * W, dtype=torch.int32, device=device)
    n = ctypes.c_int(0)
    _call_on(labels.device, "bsa_tile_labels", T, H, W, int(tile[0]), int(tile[1]), int(tile[2]), _ptr(labels),
         ctypes.byref(n), _stream(labels.device))
    return labels, n.value


def sliding_tile_block_mask(n_tiles, window, device="cuda"):
    """Tile-resolution Sliding Tile Attention mask over a (nT, nH, nW) tile grid with a
    (wt, wh, ww) window in tiles: uint8 (C, C), C = nT·nH·nW, tiles in the order of
    ``tile_labels``."""
    nT, nH, nW = (int(x) for x in n_tiles)
    C = nT * nH * nW
    mask = torch.empty((C, C), dtype=torch.uint8, device=device)
    _call_on(mask.device, "bsa_sliding_tile_block_mask", nT, nH, nW, int(window[0]),
             int(window[1]), int(window[2]), _ptr(mask), _stream(mask.device))
    return mask


def attention_workspace_bytes(q, k, Cq, Ck):
    return _lib.load().bsa_attention_workspace_bytes(make_shape(q, k), int(Cq), int(Ck))


def _mask_strides(block_mask, B, H, Cq, Ck):
    """uint8 mask of shape (Cq,Ck), (H,Cq,Ck) or (B,H,Cq,Ck) (size-1 dims broadcast)
    -> (tensor, batch stride, head stride) in elements."""
    m = block_mask
    if m.dtype == torch.bool:
        m = m.to(torch.uint8)
    if m.dtype != torch.uint8:
        raise ValueError("block_mask must be bool or uint8")
    if m.dim() not in (2, 3, 4):
        raise ValueError(f"block_mask: {m.dim()} dimensions, expected 2, 3 or 4")
    if tuple(m.shape[-2:]) != (Cq, Ck):
        raise ValueError(f"block_mask trailing dims {tuple(m.shape[-2:])} != ({Cq},{Ck})")
    lead = (1,) * (4 - m.dim()) + tuple(m.shape[:-2])
    if lead[0] not in (1, B) or lead[1] not in (1, H):
        raise ValueError(f"block_mask leading dims {tuple(m.shape[:-2])} must be 1 or (B, H) "
                         f"= ({B}, {H})")
    m = m.contiguous().view(*lead, Cq, Ck)
    bs = Cq * Ck * m.shape[1] if m.shape[0] > 1 else 0
    hs = Cq * Ck if m.shape[1] > 1 else 0
    return m, bs, hs


# Workspace address -> the arguments of the last attention call that prepared it (labels
# and mask by identity and in-place version) and the workspace tensor itself (weakly, so a
# new tensor at a recycled address never matches), for calls that reuse that preparation.
_PLANS = {}


def _record_plan(workspace, key):
    """Remember which call prepared ``workspace``; the record goes when the tensor does."""
    ptr = workspace.data_ptr()

    def drop(ref, ptr=ptr):
        rec = _PLANS.get(ptr)
        if rec is not None and rec[1] is ref:
            del _PLANS[ptr]
    _PLANS[ptr] = (key, weakref.ref(workspace, drop))


def _plan_key(shape, q_labels, k_labels, block_mask, Cq, Ck, compensate):
    return (tuple(getattr(shape, f) for f, _ in shape._fields_), Cq, Ck, bool(compensate),
            q_labels.data_ptr(), q_labels._version, tuple(q_labels.shape),
            k_labels.data_ptr(), k_labels._version, tuple(k_labels.shape),
            block_mask.data_ptr(), block_mask._version, tuple(block_mask.shape),
            tuple(block_mask.stride()), block_mask.dtype)


def centroid_compensated_attention(q, k, v, q_labels, k_labels, block_mask, Cq=None, Ck=None,
                                   scale=None, compensate=True, out=None, workspace=None,
                                   reuse_plan=False):
    """SVG-EAR centroid-compensated block-sparse attention (``compensate=False``: hard
    drop). q: (B,Hq,S,D), k/v: (B,Hkv,S,D) bf16 or fp32; labels int32; block_mask
    bool/uint8 (Cq,Ck) / (H,Cq,Ck) / (B,H,Cq,Ck). Returns fp32 (B,Hq,S,D).

    ``reuse_plan=True`` skips the label sorts, key cluster order, query tile plan and
    mask bitsets, reusing those of the last call on ``workspace``; that call must have
    had the same shapes, label and mask tensors (unmodified since), Cq, Ck and
    compensate, and no other call may have used the workspace in between. q, k, v and
    scale may differ (the K/V gather, centroids and attention always run)."""
    _expect_qkv(q, k, v)
    B, Hq, Sq, D = q.shape
    _expect(q_labels, "q_labels", (torch.int32,), (1,), (Sq,))
    _expect(k_labels, "k_labels", (torch.int32,), (1,), (k.shape[2],))
    if out is not None:
        _expect(out, "out", (torch.float32,), (4,), (B, Hq, Sq, D))
    _expect_workspace(workspace)
    Cq = int(block_mask.shape[-2]) if Cq is None else int(Cq)
    Ck = int(block_mask.shape[-1]) if Ck is None else int(Ck)
    m, bs, hs = _mask_strides(block_mask, B, Hq, Cq, Ck)
    shape = make_shape(q, k)
    key = _plan_key(shape, q_labels, k_labels, block_mask, Cq, Ck, compensate)
    rec = _PLANS.get(workspace.data_ptr()) if workspace is not None else None
    if reuse_plan and (rec is None or rec[0] != key or rec[1]() is not workspace):
        raise ValueError("reuse_plan needs the workspace of an earlier call with the same "
                         "shapes, labels, mask, Cq, Ck and compensate (tensors unmodified)")
    _need_cuda(q, k, v, q_labels, k_labels, m, out, workspace)
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=q.device)
    need = _lib.load().bsa_attention_workspace_bytes(shape, Cq, Ck)
    if need == 0:
        raise _lib.BsaError("bsa_attention_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED, _lib.detail())
    if not reuse_plan and (workspace is None or workspace.numel() < need):
        workspace = _workspace(need, q.device)
    if workspace is not None:
        _PLANS.pop(workspace.data_ptr(), None)
    _call_on(q.device, "bsa_centroid_compensated_attention_ex", _ptr(q), _ptr(k), _ptr(v), shape,
             _ptr(q_labels), Cq, _ptr(k_labels), Ck, _ptr(m), bs, hs, float(scale or 0.0),
             1 if compensate else 0, _ptr(out), _ptr(workspace), workspace.numel(),
             _lib.BSA_REUSE_PLAN if reuse_plan else 0, _stream(q.device))
    _record_plan(workspace, key)
    return out


def per_kv_head_attention(q, k, v, q_labels, k_labels, block_mask, Cq=None, Ck=None, scale=None,
                          compensate=True, out=None, workspace=None):
    """The compensated attention with labels per (batch, KV head), as the response-coupled
    partition produces them: q_labels int32 (B, Hkv, Sq), k_labels int32 (B, Hkv, Sk);
    block_mask bool/uint8 (Cq,Ck) / (Hkv,Cq,Ck) / (B,Hkv,Cq,Ck), shared by the query
    heads of a KV head. Returns fp32 (B,Hq,S,D)."""
    _expect_qkv(q, k, v)
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    _expect(q_labels, "q_labels", (torch.int32,), (3,), (B, Hkv, Sq))
    _expect(k_labels, "k_labels", (torch.int32,), (3,), (B, Hkv, Sk))
    if out is not None:
        _expect(out, "out", (torch.float32,), (4,), (B, Hq, Sq, D))
    _expect_workspace(workspace)
    Cq = int(block_mask.shape[-2]) if Cq is None else int(Cq)
    Ck = int(block_mask.shape[-1]) if Ck is None else int(Ck)
    m, bs, gs = _mask_strides(block_mask, B, Hkv, Cq, Ck)
    _need_cuda(q, k, v, q_labels, k_labels, m, out, workspace)
    shape = make_shape(q, k)
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=q.device)
    need = _lib.load().bsa_per_kv_head_attention_workspace_bytes(shape, Cq, Ck)
    if need == 0:
        raise _lib.BsaError("bsa_per_kv_head_attention_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED,
                            _lib.detail())
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    _call_on(q.device, "bsa_per_kv_head_attention", _ptr(q), _ptr(k), _ptr(v), shape, _ptr(q_labels),
             Cq, _ptr(k_labels), Ck, _ptr(m), bs, gs, float(scale or 0.0), 1 if compensate else 0,
             _ptr(out), _ptr(workspace), workspace.numel(), _stream(q.device))
    return out


def error_aware_block_mask(q, k, v, q_labels, k_labels, Cq, Ck, density, scale=None,
                           return_err=False, workspace=None):
    """SVG-EAR error-aware routing: uint8 (B, Hq, Cq, Ck) mask of the blocks to compute
    exactly, the highest compensation-error-per-pair blocks within ``density`` of the
    token pairs (and, with ``return_err``, the fp32 block errors)."""
    _expect_qkv(q, k, v)
    B, Hq, Sq, D = q.shape
    _expect(q_labels, "q_labels", (torch.int32,), (1,), (Sq,))
    _expect(k_labels, "k_labels", (torch.int32,), (1,), (k.shape[2],))
    _expect_workspace(workspace)
    _need_cuda(q, k, v, q_labels, k_labels, workspace)
    shape = make_shape(q, k)
    Cq, Ck = int(Cq), int(Ck)
    need = _lib.load().bsa_routing_workspace_bytes(shape, Cq, Ck)
    if need == 0:
        raise _lib.BsaError("bsa_routing_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED, _lib.detail())
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    mask = torch.empty((B, Hq, Cq, Ck), dtype=torch.uint8, device=q.device)
    err = torch.empty((B, Hq, Cq, Ck), dtype=torch.float32, device=q.device) if return_err else None
    _call_on(q.device, "bsa_error_aware_block_mask", _ptr(q), _ptr(k), _ptr(v), shape,
             _ptr(q_labels), Cq, _ptr(k_labels), Ck, float(density), float(scale or 0.0),
             _ptr(mask), _ptr(err), _ptr(workspace), workspace.numel(), _stream(q.device))
    return (mask, err) if return_err else mask


def probe_budget_block_mask(q, k, q_labels, k_labels, Cq, Ck, density, M, scale=None,
                            return_mass=False, workspace=None):
    """SparsePR's router: uint8 (B, Hq, Cq, Ck) mask of the highest attention-mass-per-pair
    cells within ``density`` of the token pairs after the M probe rows' pairs are
    reserved (and, with ``return_mass``, the fp32 cell masses)."""
    _expect_qkv(q, k)
    B, Hq, Sq, D = q.shape
    _expect(q_labels, "q_labels", (torch.int32,), (1,), (Sq,))
    _expect(k_labels, "k_labels", (torch.int32,), (1,), (k.shape[2],))
    _expect_workspace(workspace)
    _need_cuda(q, k, q_labels, k_labels, workspace)
    shape = make_shape(q, k)
    Cq, Ck = int(Cq), int(Ck)
    need = _lib.load().bsa_routing_workspace_bytes(shape, Cq, Ck)
    if need == 0:
        raise _lib.BsaError("bsa_routing_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED, _lib.detail())
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    mask = torch.empty((B, Hq, Cq, Ck), dtype=torch.uint8, device=q.device)
    mass = torch.empty((B, Hq, Cq, Ck), dtype=torch.float32, device=q.device) if return_mass else None
    _call_on(q.device, "bsa_probe_budget_block_mask", _ptr(q), _ptr(k), shape, _ptr(q_labels), Cq,
             _ptr(k_labels), Ck, float(density), int(M), float(scale or 0.0), _ptr(mask), _ptr(mass),
             _ptr(workspace), workspace.numel(), _stream(q.device))
    return (mask, mass) if return_mass else mask


def response_coupled_partition(q, k, Cq, Ck, r_k=48, r_q=64, iters=8, scale=None, workspace=None):
    """SparsePR Response-Coupled Partitioning: int32 query labels (B, Hkv, Sq) and key
    labels (B, Hkv, Sk), one partition per KV head shared by its query heads."""
    _expect_qkv(q, k)
    _expect_workspace(workspace)
    _need_cuda(q, k, workspace)
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    shape = make_shape(q, k)
    need = _lib.load().bsa_partition_workspace_bytes(shape, int(Cq), int(Ck), int(r_k), int(r_q))
    if need == 0:
        raise _lib.BsaError("bsa_partition_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED, _lib.detail())
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    ql = torch.empty((B, Hkv, Sq), dtype=torch.int32, device=q.device)
    kl = torch.empty((B, Hkv, Sk), dtype=torch.int32, device=q.device)
    _call_on(q.device, "bsa_response_coupled_partition", _ptr(q), _ptr(k), shape, int(Cq), int(Ck),
             int(r_k), int(r_q), int(iters), float(scale or 0.0), _ptr(ql), _ptr(kl),
             _ptr(workspace), workspace.numel(), _stream(q.device))
    return ql, kl


def antidiagonal_block_scores(q, k, block=128, stride=16, logit_scale=None):
    """XAttention block-mass estimate: fp32 (B, Hq, S/block, S/block), rows sum to 1.
    q: (B,Hq,S,D), k: (B,Hkv,S,D) bf16 with S a multiple of ``block`` (the caller pads)."""
    _expect_qkv(q, k)
    B, Hq, S, D = q.shape
    if k.shape[2] != S:
        raise ValueError(f"k has {k.shape[2]} tokens, q has {S}")
    _need_cuda(q, k)
    nb = S // block
    scores = torch.empty((B, Hq, nb, nb), dtype=torch.float32, device=q.device)
    _call_on(q.device, "bsa_antidiagonal_block_scores", _ptr(q), _ptr(k), make_shape(q, k), int(block),
         int(stride), float(logit_scale or 0.0), _ptr(scores), _stream(q.device))
    return scores


def top_p_block_mask(scores, tau, return_ties=False):
    """Per-row top-p selection over fp32 (B,H,Nq,Nk) scores; ``tau`` is a float or an
    (H,) sequence/tensor. Returns a uint8 mask (and uint8 tie flags (B,H,Nq))."""
    _expect(scores, "scores", (torch.float32,), (4,))
    _need_cuda(scores)
    B, H, Nq, Nk = scores.shape
    t = torch.as_tensor(tau, dtype=torch.float32).reshape(-1).to(scores.device)
    if t.numel() not in (1, H):
        raise ValueError("tau must be a scalar or have H entries")
    mask = torch.empty((B, H, Nq, Nk), dtype=torch.uint8, device=scores.device)
    ties = torch.empty((B, H, Nq), dtype=torch.uint8, device=scores.device)
    _call_on(scores.device, "bsa_top_p_block_mask", _ptr(scores), B, H, Nq, Nk, _ptr(t), t.numel(), _ptr(mask),
         _ptr(ties), _stream(scores.device))
    return (mask, ties) if return_ties else mask


def select_probe_rows(labels, C, M, q=None):
    """SparsePR probe rows. Without ``q``: head-agnostic middle-out members, (M,) int32
    indices and (M,) fp32 weights. With ``q`` (B,Hq,S,D): per-head members nearest to
    their cluster's mean query, (B,Hq,M) indices and weights."""
    _expect(labels, "labels", (torch.int32,), (1,))
    S = labels.shape[0]
    if q is not None:
        _expect(q, "q", tuple(_DT), (4,))
        if q.shape[2] != S:
            raise ValueError(f"q has {q.shape[2]} tokens, labels {S}")
    _need_cuda(labels, q)
    dev = labels.device
    if q is not None:
        B, Hq = q.shape[:2]
        shape = make_shape(q, q)
        n_heads = B * Hq
        idx = torch.empty((B, Hq, M), dtype=torch.int32, device=dev)
        w = torch.empty((B, Hq, M), dtype=torch.float32, device=dev)
    else:
        shape = Shape(1, 1, 1, S, S, 64, BSA_BF16)
        n_heads = 1
        idx = torch.empty((M,), dtype=torch.int32, device=dev)
        w = torch.empty((M,), dtype=torch.float32, device=dev)
    need = _lib.load().bsa_probe_select_workspace_bytes(S, int(C), n_heads)
    ws = _workspace(need, dev)
    _call_on(dev, "bsa_select_probe_rows", _ptr(labels), S, int(C), int(M), _ptr(q), shape, _ptr(idx),
         _ptr(w), _ptr(ws), ws.numel(), _stream(dev))
    return idx, w


def probe_dense_attention(q, k, v, probe_idx, scale=None, workspace=None):
    """Exact attention of the probe rows over every key: fp32 (B, Hq, M, D)."""
    _expect_qkv(q, k, v)
    B, Hq, S, D = q.shape
    _expect(probe_idx, "probe_idx", (torch.int32,), (1, 3))
    if probe_idx.dim() == 3 and tuple(probe_idx.shape[:2]) != (B, Hq):
        raise ValueError(f"probe_idx: shape {tuple(probe_idx.shape)}, expected (M,) or ({B}, {Hq}, M)")
    _expect_workspace(workspace)
    _need_cuda(q, k, v, probe_idx, workspace)
    per_head = 1 if probe_idx.dim() == 3 else 0
    M = probe_idx.shape[-1]
    shape = make_shape(q, k)
    out = torch.empty((B, Hq, M, v.shape[-1]), dtype=torch.float32, device=q.device)
    need = _lib.load().bsa_probe_attention_workspace_bytes(shape, int(M))
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    _call_on(q.device, "bsa_probe_dense_attention", _ptr(q), _ptr(k), _ptr(v), shape, _ptr(probe_idx), int(M),
         per_head, float(scale or 0.0), _ptr(out), _ptr(workspace), workspace.numel(),
         _stream(q.device))
    return out


def probe_residual_correction(out, o_probe, probe_idx, weights, rank=16, lam=0.1, workspace=None):
    """SparsePR repair of ``out`` (fp32 (B,H,S,D), updated in place and returned)."""
    _expect(out, "out", (torch.float32,), (4,))
    B, H, S, D = out.shape
    _expect(probe_idx, "probe_idx", (torch.int32,), (1, 3))
    M = probe_idx.shape[-1]
    if probe_idx.dim() == 3 and tuple(probe_idx.shape) != (B, H, M):
        raise ValueError(f"probe_idx: shape {tuple(probe_idx.shape)}, expected (M,) or ({B}, {H}, M)")
    _expect(weights, "weights", (torch.float32,), None, tuple(probe_idx.shape))
    _expect(o_probe, "o_probe", (torch.float32,), (4,), (B, H, M, D))
    _expect_workspace(workspace)
    _need_cuda(out, o_probe, probe_idx, weights, workspace)
    per_head = 1 if probe_idx.dim() == 3 else 0
    need = _lib.load().bsa_repair_workspace_bytes(B, H, S, D, int(M))
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, out.device)
    _call_on(out.device, "bsa_probe_residual_correction", _ptr(out), _ptr(o_probe), _ptr(probe_idx), _ptr(weights),
         per_head, B, H, S, D, int(M), int(rank), float(lam), _ptr(workspace), workspace.numel(),
         _stream(out.device))
    return out


class MaskCache:
    """HEART per-head drift/anchor mask cache; its state is one device byte buffer."""

    def __init__(self, B, H, Cq, Ck, D, delta, relative=False, gate_lo=0.4, gate_hi=0.8,
                 device="cuda"):
        self.shape = (B, H, Cq, Ck, D)
        n = _lib.load().bsa_mask_cache_state_bytes(B, H, Cq, Ck, D)
        self.state = torch.empty(n, dtype=torch.uint8, device=device)
        self.refresh = torch.empty((B, H), dtype=torch.uint8, device=device)
        self.drift = torch.empty((B, H), dtype=torch.float32, device=device)
        self.mask = torch.empty((B, H, Cq, Ck), dtype=torch.uint8, device=device)
        _call_on(self.state.device, "bsa_mask_cache_init", _ptr(self.state), B, H, Cq, Ck, D, float(delta),
             1 if relative else 0, float(gate_lo), float(gate_hi), _stream(self.state.device))

    def should_refresh(self, q, k, sync=True):
        """Device uint8 (B,H) refresh flags; with ``sync`` also the host count."""
        B, H, _, _, D = self.shape
        _expect(q, "q", tuple(_DT), (4,))
        if q.shape[0] != B or q.shape[1] != H or q.shape[3] != D:
            raise ValueError(f"q: shape {tuple(q.shape)} does not fit the cache ({B}, {H}, S, {D})")
        _expect(k, "k", (q.dtype,), (4,), tuple(q.shape))
        _need_cuda(q, k, self.state)
        n = ctypes.c_int(0)
        _call_on(q.device, "bsa_mask_cache_should_refresh", _ptr(self.state), _ptr(q), _ptr(k), make_shape(q, k),
             _ptr(self.refresh), _ptr(self.drift), ctypes.byref(n) if sync else None,
             _stream(q.device))
        return (self.refresh, n.value) if sync else self.refresh

    def update(self, new_mask):
        """Cached mask with the refreshed heads replaced by ``new_mask`` (or None)."""
        nm = None
        if new_mask is not None:
            B, H, Cq, Ck, _ = self.shape
            _expect(new_mask, "new_mask", (torch.bool, torch.uint8), (4,), (B, H, Cq, Ck))
            nm = new_mask.to(torch.uint8).contiguous()
            _need_cuda(nm, self.state)
        _call_on(self.state.device, "bsa_mask_cache_update", _ptr(self.state), _ptr(nm), _ptr(self.refresh),
             _ptr(self.mask), _stream(self.state.device))
        return self.mask

    def reset(self):
        _call_on(self.state.device, "bsa_mask_cache_reset", _ptr(self.state), _stream(self.state.device))
