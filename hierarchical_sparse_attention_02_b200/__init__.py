"""B200-native hot path of Zyphra Hierarchical Attention (ZHA).

The computation lives in libzha.so (hand-written CUDA for sm_100a behind the C ABI of
include/zha.h); ``api`` is a thin ctypes binding with the same function names.
"""
from .api import (Geometry, ZhaError, check_geom, empty_tree, empty_workspace, launch_count,  # noqa: F401
                  leaf_cap, reference_block, tree_bytes, tree_level, workspace_bytes, zha_append, zha_build_tree,
                  zha_decode, zha_dense_decode, zha_flat_index, zha_route, zha_route_schedule, zha_route_topk,
                  zha_sparse_attn,
                  zha_sparse_attn_noalloc, zha_check_bounded_wait, zha_prefill_attn)
from ._lib import (ZHA_OP_ATTN, ZHA_OP_DECODE, ZHA_OP_DENSE, ZHA_OP_FLAT, ZHA_OP_PREFILL, ZHA_OP_ROUTE,  # noqa: F401
                   load as load_library)
