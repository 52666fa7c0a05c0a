"""ctypes view of libzha.so (the C ABI of include/zha.h).

Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzha.so")

ZHA_OK, ZHA_ERR_INVALID_ARG, ZHA_ERR_UNSUPPORTED, ZHA_ERR_CAPACITY, ZHA_ERR_CUDA, ZHA_ERR_DEVICE = range(6)
ZHA_F32, ZHA_BF16 = 0, 1
ZHA_OP_ROUTE, ZHA_OP_ATTN, ZHA_OP_DECODE, ZHA_OP_DENSE, ZHA_OP_FLAT, ZHA_OP_PREFILL = 1, 2, 3, 4, 5, 6

# every symbol include/zha.h declares, in declaration order
EXPORTS = [
    "zha_status_str", "zha_check_geom", "zha_tree_bytes", "zha_tree_level", "zha_workspace_bytes",
    "zha_leaf_cap", "zha_build_tree", "zha_append", "zha_route", "zha_route_schedule", "zha_route_topk", "zha_sparse_attn",
    "zha_prefill_attn", "zha_decode",
    "zha_dense_decode", "zha_flat_index", "zha_sparse_attn_noalloc", "zha_check_bounded_wait", "zha_launch_count",
    "zha_last_error", "zha_trace", "zha_trace_count",
]
ZHA_NOALLOC_SCRATCH_BYTES = 16 << 20
ZHA_TRACE_ATTN, ZHA_TRACE_ROUTE_SCORE, ZHA_TRACE_ROUTE_SELECT, ZHA_TRACE_ROUTE_FUSED = 1, 2, 3, 4


class Geom(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("leaf", ctypes.c_int32), ("branch", ctypes.c_int32), ("depth", ctypes.c_int32),
                ("R", ctypes.c_int32), ("t_cap", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("rope_pairs", ctypes.c_int32)]


class Buf(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


class LevelLayout(ctypes.Structure):
    _fields_ = [("n_cap", ctypes.c_int64), ("span", ctypes.c_int64), ("k_route_off", ctypes.c_size_t),
                ("b_hat_off", ctypes.c_size_t), ("F_off", ctypes.c_size_t), ("k_state_off", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I32, _I64, _F64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
_G = ctypes.POINTER(Geom)

_SIGS = {
    "zha_status_str": (ctypes.c_char_p, [_I32]),
    "zha_check_geom": (_I32, [_G]),
    "zha_tree_bytes": (_SZ, [_G]),
    "zha_tree_level": (_I32, [_G, _I32, ctypes.POINTER(LevelLayout)]),
    "zha_workspace_bytes": (_SZ, [_G, _I32, _I32]),
    "zha_leaf_cap": (_I64, [_G]),
    "zha_build_tree": (_I32, [_G, _P, _I64, _P, Buf, _P, _P]),
    "zha_append": (_I32, [_G, _P, _P, _P, _P, _I64, _I32, _P, Buf, _P, _P]),
    "zha_route": (_I32, [_G, _P, _P, _I32, _F64, Buf, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_route_schedule": (_I32, [_G, _P, _P, _I32, _P, Buf, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_route_topk": (_I32, [_G, _P, _P, _I32, _P, Buf, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_sparse_attn": (_I32, [_G, _P, _P, _P, _P, _I32, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_prefill_attn": (_I32, [_G, _P, _P, _P, _P, _I32, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_decode": (_I32, [_G, _P, _P, _P, _P, _P, _I64, _P, _F64, Buf, _P, _P, _I32, _P, Buf, _P, _P]),
    "zha_dense_decode": (_I32, [_G, _P, _P, _P, _P, _I32, _P, _P, Buf, _P, _P]),
    "zha_flat_index": (_I32, [_G, _P, _P, _P, _P, _I32, _F64, _P, _P, _I32, _P, Buf, _P, _P]),
    "zha_sparse_attn_noalloc": (_I32, [_G, _P, _P, _P, _P, _I32, _P, _P, _I32, _P, _P, _P, _P]),
    "zha_check_bounded_wait": (_I32, [_I64, _P, _P, _P]),
    "zha_launch_count": (_I64, []),
    "zha_last_error": (ctypes.c_char_p, []),
    "zha_trace": (None, [_I32, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p), _I32]),
    "zha_trace_count": (_I32, [_I32]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """The loaded library (built in-tree by ``build.py``); raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libzha.so is not built ({path}); run "
                           "`python -m hierarchical_sparse_attention_02_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
