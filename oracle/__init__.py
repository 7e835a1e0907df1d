"""Oracle: a plain, slow, float64 CPU statement of what the block-sparse attention
hot path computes.

THIS PACKAGE IS TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (``block_sparse_attention_tcgen05_b200``) never imports it and
shares no code, table or helper with it.

Every function takes the values the GPU path is handed (bf16 or fp32), upcast to
float64, and follows the definitions on the source pages:

* "Sparse-block compensation" (mlx-arsenal research notes): hard drop, SVG-EAR
  centroid compensation, the extended-key ``[K; K̄]`` identity, SparsePR probe
  selection and probe-fitted residual repair, ``tile_labels``.
* "Dynamic block masks and head-wise mask reuse" (mlx-arsenal research notes):
  XAttention anti-diagonal scoring, top-p block masks, the HEART per-head
  drift/anchor mask cache.
* "Partition the Support, Reconstruct the Residual" (paper summary): probe
  stratification by distance to the group centroid, GQA sharing, executed-pair
  accounting.

Readings taken where the pages are silent are stated in each function's docstring.
Functions whose conventions no page fixes say "parity unpinned".
"""

from .attention import (  # noqa: F401
    cluster_centroids,
    dense_attention,
    hard_drop_attention,
    centroid_compensated_attention,
    extended_key_attention,
    kv_head,
)
from .scoring import antidiagonal_block_scores, top_p_block_mask  # noqa: F401
from .labels import sliding_tile_block_mask, sta_token_mask, tile_labels  # noqa: F401
from .repair import (  # noqa: F401
    select_probe_rows,
    select_probe_rows_centroid,
    probe_dense_attention,
    probe_residual_correction,
    standardise,
)
from .cache import HeadMaskCache, pooled_qk, qk_drift  # noqa: F401
from .accounting import executed_pairs  # noqa: F401
from .partition import kmeans, response_coupled_partition  # noqa: F401
from .routing import (  # noqa: F401
    centroid_mass,
    compensation_errors,
    error_aware_block_mask,
    probe_budget_block_mask,
    route_blocks,
)
