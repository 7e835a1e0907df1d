"""GPU test of bsa_probe_residual_correction_noalloc, the repair entry point that takes
its scratch from a buffer built into the library instead of a caller workspace (for
callers that cannot allocate device memory when they call, e.g. a runtime whose device
memory is fixed up front). Its output must equal the workspace entry point's on two
calls in a row.

This file is collected last on purpose, and must pass alone and after the others."""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _case(seed, B, H, S, D, M):
    g = np.random.default_rng(seed)
    out = (g.standard_normal((B, H, S, D)) * 0.1).astype(np.float32)
    idx = g.integers(0, S, (B, H, M)).astype(np.int32)
    w = (g.random((B, H, M)) + 0.5).astype(np.float32)
    w /= w.sum(-1, keepdims=True)
    op = (out[np.arange(B)[:, None, None], np.arange(H)[None, :, None], idx]
          + 0.05 * g.standard_normal((B, H, M, D))).astype(np.float32)
    return out, op, idx, w


def test_noalloc_matches_workspace_entry_point_twice():
    import block_sparse_attention_tcgen05_b200 as bsa
    from block_sparse_attention_tcgen05_b200 import _lib
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed, (B, H, S, D, M, rank) in enumerate([(1, 24, 4096, 128, 64, 16),
                                                  (1, 3, 2000, 64, 100, 8)]):
        out, op, idx, w = _case(seed, B, H, S, D, M)
        ref = bsa.probe_residual_correction(torch.from_numpy(out).cuda(), torch.from_numpy(op).cuda(),
                                            torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(),
                                            rank=rank, lam=0.1).cpu().numpy()
        got_t = torch.from_numpy(out).cuda()
        opt, idxt, wt = (torch.from_numpy(x).cuda() for x in (op, idx, w))
        st = lib.bsa_probe_residual_correction_noalloc(
            ctypes.c_void_p(got_t.data_ptr()), ctypes.c_void_p(opt.data_ptr()),
            ctypes.c_void_p(idxt.data_ptr()), ctypes.c_void_p(wt.data_ptr()), 1, B, H, S, D, M,
            rank, ctypes.c_float(0.1), stream)
        assert st == 0, _lib.detail()
        got = got_t.cpu().numpy()
        corr_ref, corr_got = ref - out, got - out
        assert np.linalg.norm(corr_got - corr_ref) <= 1e-3 * np.linalg.norm(corr_ref)
    assert bsa.device_status()[0] == 0


def test_noalloc_rejects_sizes_beyond_its_buffer():
    from block_sparse_attention_tcgen05_b200 import _lib
    lib = _lib.load()
    fake = ctypes.c_void_p(256)
    # 1 x 512 heads x 128 dims needs far more than the 16 MiB buffer
    st = lib.bsa_probe_residual_correction_noalloc(fake, fake, fake, fake, 1, 1, 512, 4096, 128, 64,
                                                   16, ctypes.c_float(0.1), None)
    assert st == _lib.BSA_ERR_UNSUPPORTED
    assert "16 MiB" in _lib.detail()
