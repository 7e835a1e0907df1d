"""Training-free block-sparse attention for video DiTs on NVIDIA B200 (sm_100a).

The compute path lives in ``libbsa.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/bsa.h``). This package is its thin Python binding: it checks
arguments, allocates outputs and workspaces with torch and calls the library on the
current CUDA stream. It has no CPU fallback; a missing library raises.
"""

from ._lib import BsaError, load as load_library  # noqa: F401
from .ops import (  # noqa: F401
    MaskCache,
    antidiagonal_block_scores,
    attention_workspace_bytes,
    centroid_compensated_attention,
    device_status,
    error_aware_block_mask,
    per_kv_head_attention,
    probe_dense_attention,
    probe_budget_block_mask,
    probe_residual_correction,
    response_coupled_partition,
    select_probe_rows,
    sliding_tile_block_mask,
    tile_labels,
    top_p_block_mask,
)
