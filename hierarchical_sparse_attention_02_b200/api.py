"""Python binding of the ZHA C ABI: argument marshalling only.

Every function takes torch tensors on the current CUDA device, passes their
device pointers and the current stream to the function of the same name in
libzha.so, and raises ``ZhaError`` on a non-zero status.  All computation runs
in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib


class ZhaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = _lib.load()
        msg = f"{fn}: {lib.zha_status_str(status).decode()} (status {status})"
        if status == _lib.ZHA_ERR_CUDA:
            msg += f": {lib.zha_last_error().decode()}"
        super().__init__(msg)
        self.status = status


@dataclass(frozen=True)
class Geometry:
    B: int
    Hq: int
    Hkv: int
    t_cap: int
    depth: int
    R: int = 4
    d: int = 128
    leaf: int = 64
    branch: int = 16
    dtype: torch.dtype = torch.bfloat16
    rope_pairs: int = 0          # > 0: qref carries that many rotary frequencies after the references

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def c(self) -> _lib.Geom:
        return _lib.Geom(self.B, self.Hq, self.Hkv, self.d, self.leaf, self.branch, self.depth, self.R,
                         self.t_cap, _lib.ZHA_BF16 if self.dtype == torch.bfloat16 else _lib.ZHA_F32,
                         self.rope_pairs)


def reference_block(qref: torch.Tensor, inv_freq: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The reference-query argument of the tree calls: q_hat [Hkv, R, d] fp32, followed by the
    rotary frequencies (fp32) of a RoPE model when there are any (geometry rope_pairs =
    len(inv_freq))."""
    q = qref.float().contiguous().reshape(-1)
    if inv_freq is None or inv_freq.numel() == 0:
        return q
    return torch.cat([q, inv_freq.to(device=q.device, dtype=torch.float32).reshape(-1)])


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the ZHA library must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the ZHA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _buf(t: torch.Tensor) -> _lib.Buf:
    return _lib.Buf(t.data_ptr(), t.numel() * t.element_size())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise ZhaError(fn, status)


def check_geom(g: Geometry) -> int:
    return _lib.load().zha_check_geom(ctypes.byref(g.c()))


def tree_bytes(g: Geometry) -> int:
    return _lib.load().zha_tree_bytes(ctypes.byref(g.c()))


def tree_level(g: Geometry, level: int) -> _lib.LevelLayout:
    out = _lib.LevelLayout()
    _check("zha_tree_level", _lib.load().zha_tree_level(ctypes.byref(g.c()), level, ctypes.byref(out)))
    return out


def workspace_bytes(g: Geometry, nq: int, op: int) -> int:
    return _lib.load().zha_workspace_bytes(ctypes.byref(g.c()), nq, op)


def leaf_cap(g: Geometry) -> int:
    return _lib.load().zha_leaf_cap(ctypes.byref(g.c()))


def launch_count() -> int:
    return _lib.load().zha_launch_count()


def empty_tree(g: Geometry, device="cuda") -> torch.Tensor:
    return torch.empty(tree_bytes(g), dtype=torch.uint8, device=device)


def empty_workspace(g: Geometry, nq: int, op: int, device="cuda") -> torch.Tensor:
    return torch.empty(workspace_bytes(g, nq, op), dtype=torch.uint8, device=device)


def _qref(g, qref: torch.Tensor):
    """The reference block the library reads: Hkv*R*d fp32 values, plus g.rope_pairs
    frequencies (reference_block); a shorter tensor would be read past its end."""
    need = g.Hkv * g.R * g.d + g.rope_pairs
    if qref.dtype != torch.float32 or qref.numel() != need:
        raise ValueError(f"qref: expected {need} fp32 values (Hkv*R*d references + {g.rope_pairs} "
                         f"rotary frequencies), got {qref.numel()} {qref.dtype}")
    return _ptr(qref)


def zha_build_tree(g, K, T, qref, tree, dev_status, stream=None):
    _check("zha_build_tree", _lib.load().zha_build_tree(
        ctypes.byref(g.c()), _ptr(K), T, _qref(g, qref), _buf(tree), _ptr(dev_status), _stream(stream)))


def zha_append(g, K, V, k_new, v_new, t_old, qref, tree, dev_status, stream=None):
    _check("zha_append", _lib.load().zha_append(
        ctypes.byref(g.c()), _ptr(K), _ptr(V), _ptr(k_new), _ptr(v_new), t_old, k_new.shape[1],
        _qref(g, qref), _buf(tree), _ptr(dev_status), _stream(stream)))


def zha_route(g, Q, q_pos, p, tree, leaf_ids, leaf_cnt, ws, dev_status, level_cnt=None, level_ids=None,
              stream=None):
    _check("zha_route", _lib.load().zha_route(
        ctypes.byref(g.c()), _ptr(Q), _ptr(q_pos), Q.shape[1], float(p), _buf(tree), _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(level_cnt), _ptr(level_ids), _buf(ws), _ptr(dev_status),
        _stream(stream)))


def zha_route_schedule(g, Q, q_pos, p_levels, tree, leaf_ids, leaf_cnt, ws, dev_status, level_cnt=None,
                       level_ids=None, stream=None):
    """zha_route with one threshold per level: p_levels[l-1] for level l (len == depth)."""
    if len(p_levels) != g.depth:
        raise ValueError(f"p_levels holds {len(p_levels)} thresholds for {g.depth} levels")
    arr = (ctypes.c_double * g.depth)(*[float(x) for x in p_levels])
    _check("zha_route_schedule", _lib.load().zha_route_schedule(
        ctypes.byref(g.c()), _ptr(Q), _ptr(q_pos), Q.shape[1], arr, _buf(tree), _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(level_cnt), _ptr(level_ids), _buf(ws), _ptr(dev_status),
        _stream(stream)))


def zha_route_topk(g, Q, q_pos, k_levels, tree, leaf_ids, leaf_cnt, ws, dev_status, level_cnt=None,
                   level_ids=None, stream=None):
    """The tree walk with a fixed-count selector: level l keeps its k_levels[l-1] best candidates."""
    if len(k_levels) != g.depth:
        raise ValueError(f"k_levels holds {len(k_levels)} counts for {g.depth} levels")
    arr = (ctypes.c_int32 * g.depth)(*[int(x) for x in k_levels])
    _check("zha_route_topk", _lib.load().zha_route_topk(
        ctypes.byref(g.c()), _ptr(Q), _ptr(q_pos), Q.shape[1], arr, _buf(tree), _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(level_cnt), _ptr(level_ids), _buf(ws), _ptr(dev_status),
        _stream(stream)))


def zha_sparse_attn(g, Q, K, V, q_pos, leaf_ids, leaf_cnt, O, ws, dev_status, lse=None, stream=None):
    _check("zha_sparse_attn", _lib.load().zha_sparse_attn(
        ctypes.byref(g.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_pos), Q.shape[1], _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(O), _ptr(lse), _buf(ws), _ptr(dev_status), _stream(stream)))


def zha_prefill_attn(g, Q, K, V, q_pos, leaf_ids, leaf_cnt, O, ws, dev_status, lse=None, stream=None):
    """zha_sparse_attn for many queries per sequence, one tensor-core tile of queries at a time."""
    _check("zha_prefill_attn", _lib.load().zha_prefill_attn(
        ctypes.byref(g.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_pos), Q.shape[1], _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(O), _ptr(lse), _buf(ws), _ptr(dev_status), _stream(stream)))


def zha_sparse_attn_noalloc(g, Q, K, V, q_pos, leaf_ids, leaf_cnt, O, dev_status, lse=None, stream=None):
    """zha_sparse_attn with the library's own fixed device scratch instead of a workspace."""
    _check("zha_sparse_attn_noalloc", _lib.load().zha_sparse_attn_noalloc(
        ctypes.byref(g.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_pos), Q.shape[1], _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(O), _ptr(lse), _ptr(dev_status), _stream(stream)))


def zha_decode(g, q, k_new, v_new, K, V, T, qref, p, tree, leaf_ids, leaf_cnt, O, ws, dev_status,
               stream=None):
    _check("zha_decode", _lib.load().zha_decode(
        ctypes.byref(g.c()), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(K), _ptr(V), T, _qref(g, qref), float(p),
        _buf(tree), _ptr(leaf_ids), _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(O), _buf(ws), _ptr(dev_status),
        _stream(stream)))


def zha_dense_decode(g, Q, K, V, q_pos, O, ws, dev_status, lse=None, stream=None):
    _check("zha_dense_decode", _lib.load().zha_dense_decode(
        ctypes.byref(g.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_pos), Q.shape[1], _ptr(O), _ptr(lse),
        _buf(ws), _ptr(dev_status), _stream(stream)))


def zha_flat_index(g, Q, K, V, q_pos, p, leaf_ids, leaf_cnt, O, ws, dev_status, stream=None):
    _check("zha_flat_index", _lib.load().zha_flat_index(
        ctypes.byref(g.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_pos), Q.shape[1], float(p), _ptr(leaf_ids),
        _ptr(leaf_cnt), leaf_ids.shape[-1], _ptr(O), _buf(ws), _ptr(dev_status), _stream(stream)))


def zha_check_bounded_wait(polls: int, dev_status, out, stream=None):
    """The failure-detection check of the bounded device waits (out: int64 [4] on the device)."""
    _check("zha_check_bounded_wait", _lib.load().zha_check_bounded_wait(
        int(polls), _ptr(dev_status), _ptr(out), _stream(stream)))
