"""Sparse global attention over N views (GSA) and dense global attention on B200.

The compute lives in ``lib/libgsa.so`` (CUDA for sm_100a, C ABI in
``include/gsa.h``); this package is its Python binding.
"""

from ._lib import FORWARD_STEPS, GsaError, GsaShape, GsaSizes, LIB_PATH, load  # noqa: F401
from .api import (  # noqa: F401
    GsaLayer,
    Shape,
    check_device_error,
    selftest_exp2,
    compressed_attn,
    dense_global_attn,
    dense_global_attn_mma,
    derive,
    forward,
    forward_noalloc,
    forward_timed,
    guide_logits,
    frame_attn,
    sga_workspace_size,
    new_sga_workspace,
    sga_attn,
    gate_combine,
    new_workspace,
    noalloc_check_device_error,
    pool_kv,
    selected_attn,
    topk_blocks,
    workspace_offsets,
    workspace_size,
    workspace_view,
)
