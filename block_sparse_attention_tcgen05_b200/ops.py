"""Torch-facing wrappers of the libbsa C ABI.

Argument marshalling only: tensors are checked, outputs and workspaces are allocated
with torch on the tensors' device, and every step runs in libbsa's CUDA kernels on the
current torch stream. There is no CPU path.
"""

import ctypes

import torch

from . import _lib
from ._lib import BSA_BF16, BSA_F32, Shape, call

_DT = {torch.bfloat16: BSA_BF16, torch.float32: BSA_F32}


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libbsa operates on CUDA tensors only")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


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
    call("bsa_tile_labels", T, H, W, int(tile[0]), int(tile[1]), int(tile[2]), _ptr(labels),
         ctypes.byref(n), _stream(labels.device))
    return labels, n.value


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
    m = m.contiguous()
    if m.dim() == 2:
        m = m.view(1, 1, Cq, Ck)
    elif m.dim() == 3:
        m = m.view(1, m.shape[0], Cq, Ck)
    if tuple(m.shape[-2:]) != (Cq, Ck):
        raise ValueError(f"block_mask trailing dims {tuple(m.shape[-2:])} != ({Cq},{Ck})")
    bs = Cq * Ck * m.shape[1] if m.shape[0] > 1 else 0
    hs = Cq * Ck if m.shape[1] > 1 else 0
    if (m.shape[0] not in (1, B)) or (m.shape[1] not in (1, H)):
        raise ValueError("block_mask leading dims must be 1 or (B, H)")
    return m, bs, hs


def centroid_compensated_attention(q, k, v, q_labels, k_labels, block_mask, Cq=None, Ck=None,
                                   scale=None, compensate=True, out=None, workspace=None):
    """SVG-EAR centroid-compensated block-sparse attention (``compensate=False``: hard
    drop). q: (B,Hq,S,D), k/v: (B,Hkv,S,D) bf16 or fp32; labels int32; block_mask
    bool/uint8 (Cq,Ck) / (H,Cq,Ck) / (B,H,Cq,Ck). Returns fp32 (B,Hq,S,D)."""
    _need_cuda(q, k, v, q_labels, k_labels, block_mask)
    B, Hq, Sq, D = q.shape
    Cq = int(block_mask.shape[-2]) if Cq is None else int(Cq)
    Ck = int(block_mask.shape[-1]) if Ck is None else int(Ck)
    shape = make_shape(q, k)
    m, bs, hs = _mask_strides(block_mask, B, Hq, Cq, Ck)
    if q_labels.dtype != torch.int32 or k_labels.dtype != torch.int32:
        raise ValueError("labels must be int32")
    if out is None:
        out = torch.empty((B, Hq, Sq, v.shape[-1]), dtype=torch.float32, device=q.device)
    need = _lib.load().bsa_attention_workspace_bytes(shape, Cq, Ck)
    if need == 0:
        raise _lib.BsaError("bsa_attention_workspace_bytes", _lib.BSA_ERR_UNSUPPORTED, _lib.detail())
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, q.device)
    call("bsa_centroid_compensated_attention", _ptr(q), _ptr(k), _ptr(v), shape, _ptr(q_labels),
         Cq, _ptr(k_labels), Ck, _ptr(m), bs, hs, float(scale or 0.0), 1 if compensate else 0,
         _ptr(out), _ptr(workspace), workspace.numel(), _stream(q.device))
    return out
