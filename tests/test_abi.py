"""The C ABI without a GPU: libbsa.so builds, loads, exports every entry point that
include/bsa.h declares, sizes workspaces, and rejects bad arguments on the host
before any CUDA call."""

import ctypes
import os
import re

import pytest

from block_sparse_attention_tcgen05_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    names = declared_functions()
    assert len(names) >= 18
    assert set(names) == set(_lib.SIGNATURES), set(names) ^ set(_lib.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.bsa_status_string(0) == b"BSA_OK"
    assert lib.bsa_status_string(-4) == b"BSA_ERR_TIMEOUT"
    assert lib.bsa_version() >= 100


def test_workspace_queries(lib):
    sh = _lib.Shape(1, 40, 40, 32760, 32760, 128, _lib.BSA_BF16)
    n = lib.bsa_attention_workspace_bytes(sh, 245, 245)
    # the permuted K and V copies dominate (Q rows are gathered by the attention kernel
    # itself): about 2 x 40 x 36k x 128 x 2 bytes
    assert 0.6e9 < n < 0.9e9
    assert lib.bsa_attention_workspace_bytes(_lib.Shape(1, 1, 1, 100, 100, 96, 0), 1, 1) == 0
    assert lib.bsa_repair_workspace_bytes(1, 24, 32768, 128, 64) > 0
    assert lib.bsa_repair_workspace_bytes(1, 24, 32768, 96, 64) == 0
    assert lib.bsa_mask_cache_state_bytes(1, 40, 256, 256, 128) >= 40 * 256 * 256
    assert lib.bsa_probe_select_workspace_bytes(1024, 16, 1) > 0


def _err(lib, status):
    return status, _lib.detail()


def fake_ptr():
    """A non-null, 256-byte aligned address that is never dereferenced: every call given
    it is rejected on the host before any launch."""
    return ctypes.c_void_p(1 << 20)


def test_host_side_argument_errors(lib):
    null = ctypes.c_void_p(0)
    sh = _lib.Shape(1, 2, 2, 1024, 1024, 64, _lib.BSA_BF16)
    st = lib.bsa_centroid_compensated_attention(null, null, null, sh, null, 16, null, 16, null, 0,
                                                0, 0.0, 1, null, null, 0, null)
    assert st == _lib.BSA_ERR_INVALID_ARG
    bad = _lib.Shape(1, 3, 2, 1024, 1024, 64, _lib.BSA_BF16)
    st = lib.bsa_centroid_compensated_attention(null, null, null, bad, null, 16, null, 16, null, 0,
                                                0, 0.0, 1, null, null, 0, null)
    assert st == _lib.BSA_ERR_INVALID_ARG and "Hkv" in _lib.detail()
    d96 = _lib.Shape(1, 2, 2, 1024, 1024, 96, _lib.BSA_BF16)
    st = lib.bsa_centroid_compensated_attention(null, null, null, d96, null, 16, null, 16, null, 0,
                                                0, 0.0, 1, null, null, 0, null)
    assert st == _lib.BSA_ERR_UNSUPPORTED
    # empty sequences, and key ranges past the limit of 16-bit key-group indices
    # (Sk + 15 Ck <= 2^20 - 128)
    empty = _lib.Shape(1, 2, 2, 0, 1024, 64, _lib.BSA_BF16)
    st = lib.bsa_centroid_compensated_attention(null, null, null, empty, null, 16, null, 16, null,
                                                0, 0, 0.0, 1, null, null, 0, null)
    assert st == _lib.BSA_ERR_INVALID_ARG
    assert lib.bsa_attention_workspace_bytes(empty, 16, 16) == 0
    lim = (1 << 20) - 128
    at_max = _lib.Shape(1, 1, 1, 1024, lim - 15 * 16, 64, _lib.BSA_BF16)
    assert lib.bsa_attention_workspace_bytes(at_max, 16, 16) > 0
    past = _lib.Shape(1, 1, 1, 1024, lim - 15 * 16 + 1, 64, _lib.BSA_BF16)
    assert lib.bsa_attention_workspace_bytes(past, 16, 16) == 0
    st = lib.bsa_centroid_compensated_attention(fake_ptr(), fake_ptr(), fake_ptr(), past, fake_ptr(),
                                                16, fake_ptr(), 16, fake_ptr(), 0, 0, 0.0, 1,
                                                fake_ptr(), fake_ptr(), 1 << 30, null)
    assert st == _lib.BSA_ERR_UNSUPPORTED and str(lim) in _lib.detail()
    # the flagged entry point: unknown flag bits, and the usual checks with the
    # plan-reuse flag set
    st = lib.bsa_centroid_compensated_attention_ex(null, null, null, sh, null, 16, null, 16, null,
                                                   0, 0, 0.0, 1, null, null, 0, 2, null)
    assert st == _lib.BSA_ERR_INVALID_ARG and "flags" in _lib.detail()
    st = lib.bsa_centroid_compensated_attention_ex(null, null, null, sh, null, 16, null, 16, null,
                                                   0, 0, 0.0, 1, null, null, 0,
                                                   _lib.BSA_REUSE_PLAN, null)
    assert st == _lib.BSA_ERR_INVALID_ARG and "null" in _lib.detail()
    st = lib.bsa_centroid_compensated_attention_ex(fake_ptr(), fake_ptr(), fake_ptr(), sh,
                                                   fake_ptr(), 16, fake_ptr(), 16, fake_ptr(), 0, 0,
                                                   0.0, 1, fake_ptr(), fake_ptr(), 256,
                                                   _lib.BSA_REUSE_PLAN, null)
    assert st == _lib.BSA_ERR_WORKSPACE
    # scoring: S not a multiple of the block
    fake = ctypes.c_void_p(256)
    s2 = _lib.Shape(1, 1, 1, 1000, 1000, 64, _lib.BSA_BF16)
    assert lib.bsa_antidiagonal_block_scores(fake, fake, s2, 128, 16, 0.0, fake, null) == \
        _lib.BSA_ERR_INVALID_ARG
    # top-p: too many key blocks, bad tau count
    assert lib.bsa_top_p_block_mask(fake, 1, 2, 4, 2048, fake, 1, fake, null, null) == \
        _lib.BSA_ERR_UNSUPPORTED
    assert lib.bsa_top_p_block_mask(fake, 1, 2, 4, 16, fake, 3, fake, null, null) == \
        _lib.BSA_ERR_INVALID_ARG
    # repair: rank outside [1, D], workspace too small
    assert lib.bsa_probe_residual_correction(fake, fake, fake, fake, 0, 1, 1, 100, 64, 8, 65, 0.1,
                                             fake, 1 << 30, null) == _lib.BSA_ERR_INVALID_ARG
    assert lib.bsa_probe_residual_correction(fake, fake, fake, fake, 0, 1, 1, 100, 64, 8, 16, 0.1,
                                             fake, 16, null) == _lib.BSA_ERR_WORKSPACE
    # tile labels
    assert lib.bsa_tile_labels(0, 1, 1, 1, 1, 1, fake, None, null) == _lib.BSA_ERR_INVALID_ARG


def test_per_kv_head_attention_host_errors(lib):
    """The per-KV-head call rejects a bad head split and null pointers on the host, and
    sizes its workspace for one (batch, KV head) problem."""
    null = ctypes.c_void_p(0)
    sh = _lib.Shape(2, 6, 2, 4096, 4096, 64, _lib.BSA_BF16)
    one = _lib.Shape(1, 3, 1, 4096, 4096, 64, _lib.BSA_BF16)
    assert lib.bsa_per_kv_head_attention_workspace_bytes(sh, 16, 16) == \
        lib.bsa_attention_workspace_bytes(one, 16, 16) > 0
    bad = _lib.Shape(1, 5, 2, 4096, 4096, 64, _lib.BSA_BF16)
    assert lib.bsa_per_kv_head_attention_workspace_bytes(bad, 16, 16) == 0
    st = lib.bsa_per_kv_head_attention(null, null, null, bad, null, 16, null, 16, null, 0, 0, 0.0, 1,
                                       null, null, 0, null)
    assert st == _lib.BSA_ERR_INVALID_ARG
    st = lib.bsa_per_kv_head_attention(null, null, null, sh, null, 16, null, 16, null, 0, 0, 0.0, 1,
                                       null, null, 0, null)
    assert st == _lib.BSA_ERR_INVALID_ARG and "null" in _lib.detail()


def test_python_binding_refuses_cpu_tensors():
    import torch

    import block_sparse_attention_tcgen05_b200 as bsa
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    lab = torch.zeros(128, dtype=torch.int32)
    with pytest.raises(ValueError):
        bsa.centroid_compensated_attention(q, q, q, lab, lab, torch.ones(1, 1, dtype=torch.uint8))


def test_noalloc_repair_returns_the_workspace_entry_points_status(lib):
    """The allocation-free repair runs the same argument checks, with the same status
    codes, as bsa_probe_residual_correction before it looks at its buffer's size."""
    fake = fake_ptr()
    null = ctypes.c_void_p(0)
    cases = [
        ((0, 1, 1, 100, 96, 8, 16, 0.1), _lib.BSA_ERR_UNSUPPORTED),    # head dim 96
        ((0, 1, 1, 100, 64, 1025, 16, 0.1), _lib.BSA_ERR_UNSUPPORTED),  # M > 1024
        ((0, 1, 1, 100, 64, 8, 65, 0.1), _lib.BSA_ERR_INVALID_ARG),     # rank > D
        ((0, 1, 1, 100, 64, 8, 16, -1.0), _lib.BSA_ERR_INVALID_ARG),    # lambda < 0
        ((0, 1, 0, 100, 64, 8, 16, 0.1), _lib.BSA_ERR_INVALID_ARG),     # H = 0
    ]
    for (ph, B, H, S, D, M, r, lam), want in cases:
        st_ws = lib.bsa_probe_residual_correction(fake, fake, fake, fake, ph, B, H, S, D, M, r,
                                                  lam, fake, 1 << 30, null)
        st_na = lib.bsa_probe_residual_correction_noalloc(fake, fake, fake, fake, ph, B, H, S, D,
                                                          M, r, lam, null)
        assert st_ws == st_na == want, (D, M, r, lam, st_ws, st_na)
    # null output pointer: both INVALID_ARG
    assert lib.bsa_probe_residual_correction_noalloc(null, fake, fake, fake, 0, 1, 1, 100, 64, 8,
                                                     16, 0.1, null) == _lib.BSA_ERR_INVALID_ARG
