"""ctypes loader for libbsa.so and its C declarations (mirrors include/bsa.h)."""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK = 0
BSA_ERR_INVALID_ARG = -1
BSA_REUSE_PLAN = 1
BSA_ERR_UNSUPPORTED = -2
BSA_ERR_CUDA = -3
BSA_ERR_TIMEOUT = -4
BSA_ERR_WORKSPACE = -5
BSA_BF16 = 0
BSA_F32 = 1


class BsaError(RuntimeError):
    """A libbsa entry point returned a non-zero status."""

    def __init__(self, fn, status, detail):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({detail})")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("Sq", ctypes.c_int), ("Sk", ctypes.c_int), ("D", ctypes.c_int),
                ("dtype", ctypes.c_int)]


_vp, _i, _f, _sz, _i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64
_ip = ctypes.POINTER(ctypes.c_int)

# name -> (restype, argtypes)
SIGNATURES = {
    "bsa_status_string": (ctypes.c_char_p, [_i]),
    "bsa_last_error_detail": (None, [ctypes.c_char_p, _sz]),
    "bsa_version": (_i, []),
    "bsa_get_device_status": (_i, [_vp, _ip]),
    "bsa_wait_timeout_selftest": (_i, [ctypes.c_longlong, _vp]),
    "bsa_launch_count": (ctypes.c_longlong, []),
    "bsa_profile_enable": (_i, [_i]),
    "bsa_profile_read": (_i, [_i, ctypes.POINTER(ctypes.c_float), _ip]),
    "bsa_tile_labels": (_i, [_i, _i, _i, _i, _i, _i, _vp, _ip, _vp]),
    "bsa_sliding_tile_block_mask": (_i, [_i, _i, _i, _i, _i, _i, _vp, _vp]),
    "bsa_antidiagonal_block_scores": (_i, [_vp, _vp, Shape, _i, _i, _f, _vp, _vp]),
    "bsa_top_p_block_mask": (_i, [_vp, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "bsa_attention_workspace_bytes": (_sz, [Shape, _i, _i]),
    "bsa_centroid_compensated_attention": (
        _i, [_vp, _vp, _vp, Shape, _vp, _i, _vp, _i, _vp, _i64, _i64, _f, _i, _vp, _vp, _sz, _vp]),
    "bsa_centroid_compensated_attention_ex": (
        _i, [_vp, _vp, _vp, Shape, _vp, _i, _vp, _i, _vp, _i64, _i64, _f, _i, _vp, _vp, _sz, _i, _vp]),
    "bsa_per_kv_head_attention_workspace_bytes": (_sz, [Shape, _i, _i]),
    "bsa_per_kv_head_attention": (
        _i, [_vp, _vp, _vp, Shape, _vp, _i, _vp, _i, _vp, _i64, _i64, _f, _i, _vp, _vp, _sz, _vp]),
    "bsa_routing_workspace_bytes": (_sz, [Shape, _i, _i]),
    "bsa_error_aware_block_mask": (
        _i, [_vp, _vp, _vp, Shape, _vp, _i, _vp, _i, _f, _f, _vp, _vp, _vp, _sz, _vp]),
    "bsa_probe_budget_block_mask": (
        _i, [_vp, _vp, Shape, _vp, _i, _vp, _i, _f, _i, _f, _vp, _vp, _vp, _sz, _vp]),
    "bsa_partition_workspace_bytes": (_sz, [Shape, _i, _i, _i, _i]),
    "bsa_response_coupled_partition": (
        _i, [_vp, _vp, Shape, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _sz, _vp]),
    "bsa_probe_select_workspace_bytes": (_sz, [_i, _i, _i]),
    "bsa_select_probe_rows": (_i, [_vp, _i, _i, _i, _vp, Shape, _vp, _vp, _vp, _sz, _vp]),
    "bsa_probe_attention_workspace_bytes": (_sz, [Shape, _i]),
    "bsa_probe_dense_attention": (_i, [_vp, _vp, _vp, Shape, _vp, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "bsa_repair_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "bsa_probe_residual_correction": (
        _i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "bsa_probe_residual_correction_noalloc": (
        _i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "bsa_mask_cache_state_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "bsa_mask_cache_init": (_i, [_vp, _i, _i, _i, _i, _i, _f, _i, _f, _f, _vp]),
    "bsa_mask_cache_should_refresh": (_i, [_vp, _vp, _vp, Shape, _vp, _vp, _ip, _vp]),
    "bsa_mask_cache_layer_gate": (_i, [_vp, _vp, _i, _i, _f, _f, _vp]),
    "bsa_mask_cache_update": (_i, [_vp, _vp, _vp, _vp, _vp]),
    "bsa_mask_cache_reset": (_i, [_vp, _vp]),
}

_lib = None


def load():
    """Load libbsa.so (built in-tree by ``build.py``). Raises if it is missing: there is
    no fallback implementation."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libbsa.so not found at {LIB_PATH}; build it with "
                "`python -m block_sparse_attention_tcgen05_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name, None)
            if fn is None:
                continue
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def detail():
    buf = ctypes.create_string_buffer(512)
    load().bsa_last_error_detail(buf, 512)
    return buf.value.decode(errors="replace")


def check(fn_name, status):
    if status != BSA_OK:
        raise BsaError(fn_name, status, detail())
    return status


def call(name, *args):
    """Call an int-returning entry point and raise BsaError on a non-zero status."""
    return check(name, getattr(load(), name)(*args))
