"""CPU: the Python binding's dtype and shape checks.

The C ABI takes plain pointers, so a tensor of the wrong element type or size would be
read or written past its end inside the kernels. The binding rejects such arguments
before anything reaches the library; these checks run before the device check, so they
are exercised here with CPU tensors (a well-formed CPU call then fails on the device).
"""

import pytest
import torch

import block_sparse_attention_tcgen05_b200 as bsa

B, H, HKV, S, D, C, M = 1, 4, 2, 256, 64, 4, 8


def _qkv(dtype=torch.bfloat16):
    return (torch.zeros(B, H, S, D, dtype=dtype), torch.zeros(B, HKV, S, D, dtype=dtype),
            torch.zeros(B, HKV, S, D, dtype=dtype))


def _labels(n=S):
    return torch.zeros(n, dtype=torch.int32)


def _raises(match, fn, *args, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*args, **kw)


def test_per_kv_head_attention_arguments():
    q, k, v = _qkv()
    ql = torch.zeros(B, HKV, S, dtype=torch.int32)
    mask = torch.ones(HKV, C, C, dtype=torch.uint8)
    f = bsa.per_kv_head_attention
    _raises("q_labels: shape", f, q, k, v, torch.zeros(B, H, S, dtype=torch.int32), ql, mask)
    _raises("k_labels: 1 dimensions", f, q, k, v, ql, _labels(), mask)
    _raises("k_labels: dtype", f, q, k, v, ql, ql.long(), mask)
    _raises("block_mask leading dims", f, q, k, v, ql, ql, torch.ones(H, C, C, dtype=torch.uint8))
    _raises("block_mask trailing dims", f, q, k, v, ql, ql, mask, Cq=C + 1)
    _raises("CUDA tensors only", f, q, k, v, ql, ql, mask)


def test_attention_arguments():
    q, k, v = _qkv()
    lab, mask = _labels(), torch.ones(C, C, dtype=torch.uint8)
    f = bsa.centroid_compensated_attention
    _raises("q: dtype", f, q.half(), k, v, lab, lab, mask)
    _raises("k: dtype", f, q, k.float(), v, lab, lab, mask)
    _raises("v: shape", f, q, k, v[:, :, :128], lab, lab, mask)
    _raises("k: shape", f, q, torch.zeros(B, 3, S, D, dtype=q.dtype), v, lab, lab, mask)
    _raises("q_labels: shape", f, q, k, v, _labels(S - 1), lab, mask)
    _raises("k_labels: dtype", f, q, k, v, lab, lab.long(), mask)
    _raises("out: dtype", f, q, k, v, lab, lab, mask, out=torch.zeros(B, H, S, D, dtype=q.dtype))
    _raises("workspace: dtype", f, q, k, v, lab, lab, mask, workspace=torch.zeros(16))
    _raises("CUDA tensors only", f, q, k, v, lab, lab, mask)


def test_plan_reuse_needs_a_prepared_workspace():
    """reuse_plan skips the label sorts, tile plan and bitsets, which the kernels then
    read from the workspace: the binding refuses it unless the workspace's last
    attention call had the same arguments (no workspace, a fresh one, or a recorded one
    whose mask was modified in place since)."""
    from block_sparse_attention_tcgen05_b200 import ops
    q, k, v = _qkv()
    lab, mask = _labels(), torch.ones(C, C, dtype=torch.uint8)
    ws = torch.zeros(1024, dtype=torch.uint8)
    f = bsa.centroid_compensated_attention
    _raises("reuse_plan needs", f, q, k, v, lab, lab, mask, reuse_plan=True)
    _raises("reuse_plan needs", f, q, k, v, lab, lab, mask, workspace=ws, reuse_plan=True)
    # a record as a successful call leaves it, then an in-place change of the mask
    shape = ops.make_shape(q, k)
    ops._record_plan(ws, ops._plan_key(shape, lab, lab, mask, C, C, True))
    _raises("CUDA tensors only", f, q, k, v, lab, lab, mask, workspace=ws, reuse_plan=True)
    _raises("reuse_plan needs", f, q, k, v, lab, lab, mask, workspace=ws, reuse_plan=True,
            compensate=False)
    mask[0, 0] = 0
    _raises("reuse_plan needs", f, q, k, v, lab, lab, mask, workspace=ws, reuse_plan=True)
    # the record goes with the workspace tensor
    ptr = ws.data_ptr()
    assert ptr in ops._PLANS
    del ws
    assert ptr not in ops._PLANS


def test_scoring_and_top_p_arguments():
    q, k, _ = _qkv()
    _raises("k has", bsa.antidiagonal_block_scores, q, k[:, :, :128])
    _raises("k: dtype", bsa.antidiagonal_block_scores, q, k.float())
    _raises("CUDA tensors only", bsa.antidiagonal_block_scores, q, k)
    _raises("scores: dtype", bsa.top_p_block_mask, torch.zeros(1, H, 2, 2, dtype=torch.float64), 0.9)
    _raises("scores: 3 dimensions", bsa.top_p_block_mask, torch.zeros(H, 2, 2), 0.9)
    _raises("CUDA tensors only", bsa.top_p_block_mask, torch.zeros(1, H, 2, 2), 0.9)


def test_probe_arguments():
    q, k, v = _qkv()
    _raises("labels: dtype", bsa.select_probe_rows, _labels().long(), C, M)
    _raises("q has", bsa.select_probe_rows, _labels(), C, M, q=q[:, :, :128])
    _raises("CUDA tensors only", bsa.select_probe_rows, _labels(), C, M)
    idx = torch.zeros(M, dtype=torch.int32)
    _raises("probe_idx: dtype", bsa.probe_dense_attention, q, k, v, idx.long())
    _raises("probe_idx: shape", bsa.probe_dense_attention, q, k, v,
            torch.zeros(B, H + 1, M, dtype=torch.int32))
    _raises("CUDA tensors only", bsa.probe_dense_attention, q, k, v, idx)


def test_repair_arguments():
    out = torch.zeros(B, H, S, D)
    op = torch.zeros(B, H, M, D)
    idx = torch.zeros(M, dtype=torch.int32)
    w = torch.full((M,), 1.0 / M)
    f = bsa.probe_residual_correction
    _raises("out: dtype", f, out.bfloat16(), op, idx, w)
    _raises("o_probe: shape", f, out, op[:, :, :4], idx, w)
    _raises("weights: shape", f, out, op, idx, w[:4])
    _raises("weights: dtype", f, out, op, idx, w.double())
    _raises("probe_idx: shape", f, out, op, torch.zeros(B, H + 1, M, dtype=torch.int32), w)
    _raises("CUDA tensors only", f, out, op, idx, w)


def test_tensors_on_different_devices_are_refused():
    """Every tensor of one call must be on one device: the library reads plain pointers
    on the current device. A CPU tensor mixed with a tensor on another device (the meta
    device stands in for a second GPU here) is refused before any other device check."""
    q, k, v = _qkv()
    kmeta = torch.empty(k.shape, dtype=k.dtype, device="meta")
    lab, mask = _labels(), torch.ones(C, C, dtype=torch.uint8)
    _raises("same device", bsa.centroid_compensated_attention, q, kmeta, v, lab, lab, mask)
    _raises("same device", bsa.centroid_compensated_attention, q, k, v, lab, lab,
            mask.to("meta"))
    _raises("same device", bsa.antidiagonal_block_scores, q, kmeta)
    idx = torch.zeros(M, dtype=torch.int32)
    _raises("same device", bsa.probe_dense_attention, q, k, v, idx.to("meta"))
    out = torch.zeros(B, H, S, D)
    op = torch.zeros(B, H, M, D)
    w = torch.full((M,), 1.0 / M)
    _raises("same device", bsa.probe_residual_correction, out, op.to("meta"), idx, w)
    _raises("same device", bsa.centroid_compensated_attention, q, k, v, lab, lab, mask,
            workspace=torch.empty(16, dtype=torch.uint8, device="meta"))


def test_mask_shapes_are_checked_before_any_reshape():
    """A mask whose trailing dims are not (Cq, Ck) is refused even when its element
    count matches; leading dims must be 1, H or (B, H)."""
    q, k, v = _qkv()
    lab = _labels()
    f = bsa.centroid_compensated_attention
    _raises("trailing dims", f, q, k, v, lab, lab, torch.ones(H, 2, 8, dtype=torch.uint8),
            Cq=4, Ck=4)
    _raises("trailing dims", f, q, k, v, lab, lab, torch.ones(2, 8, dtype=torch.uint8), Cq=4,
            Ck=4)
    _raises("leading dims", f, q, k, v, lab, lab, torch.ones(H + 1, C, C, dtype=torch.uint8))
    _raises("leading dims", f, q, k, v, lab, lab, torch.ones(2, H, C, C, dtype=torch.uint8))
    _raises("dimensions", f, q, k, v, lab, lab, torch.ones(1, 1, 1, C, C, dtype=torch.uint8))
    _raises("must be bool or uint8", f, q, k, v, lab, lab, torch.ones(C, C))
