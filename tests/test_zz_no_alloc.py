"""zha_sparse_attn_noalloc: the sparse attention for callers that cannot provide a workspace.

Such callers (an engine plugin that receives only its operator's buffers, a process whose
device memory belongs to another allocator) get the attention with the library's own fixed
16 MiB device scratch array.  The GPU test checks, through the C ABI, that two calls in a
row, with different queries, give what zha_sparse_attn (caller workspace) gives for the
same inputs.  This file is named to be collected last.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import zha_synth as S
from hierarchical_sparse_attention_02_b200 import _lib
from hierarchical_sparse_attention_02_b200 import build as zbuild


def test_noalloc_rejects_oversize_before_any_launch():
    """Host-side: a geometry whose scratch cannot fit returns ZHA_ERR_CAPACITY (no GPU needed)."""
    zbuild.build()
    lib = _lib.load()
    g = _lib.Geom(B=64, Hq=64, Hkv=8, d=128, leaf=64, branch=16, depth=3, R=4, t_cap=1 << 20, dtype=1,
                  rope_pairs=0)
    fake = ctypes.c_void_p(0x1000)
    n0 = lib.zha_launch_count()
    assert lib.zha_sparse_attn_noalloc(ctypes.byref(g), fake, fake, fake, fake, 1, fake, fake, 8, fake, None,
                                       fake, None) == _lib.ZHA_ERR_CAPACITY
    assert lib.zha_sparse_attn_noalloc(ctypes.byref(g), None, fake, fake, fake, 1, fake, fake, 8, fake, None,
                                       fake, None) == _lib.ZHA_ERR_INVALID_ARG
    assert lib.zha_launch_count() == n0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    import hierarchical_sparse_attention_02_b200 as Z
    zbuild.build()
    Z.load_library()
    dev = "cuda"
    # 128 (sequence, KV head) units: the default split would need ~26 MiB of scratch, so
    # this also exercises the enlarged split that fits the fixed array
    w = S.scaled(S.workload("batched-decode-128k"), T=40000 + 21, B=32, n_centres=512)
    g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=w.depth, R=w.R)
    assert Z.workspace_bytes(g, 1, Z.ZHA_OP_ATTN) > _lib.ZHA_NOALLOC_SCRATCH_BYTES
    C, K, V = S.clustered_kv(w, dev)
    qref = S.reference_queries(w, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tree = Z.empty_tree(g, dev)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    pos = torch.full((w.B, 1), w.T - 1, dtype=torch.int64, device=dev)
    cap = Z.leaf_cap(g)
    ws_route = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE, dev)
    ws_attn = Z.empty_workspace(g, 1, Z.ZHA_OP_ATTN, dev)
    for call in range(2):
        q = S.queries(w, C, 1, dev, step=call)
        ids = torch.empty(w.B, 1, w.Hq, cap, dtype=torch.int32, device=dev)
        cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=dev)
        Z.zha_route(g, q, pos, 0.95, tree, ids, cnt, ws_route, st)
        want = torch.empty(w.B, 1, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
        want_lse = torch.empty(w.B, 1, w.Hq, dtype=torch.float32, device=dev)
        Z.zha_sparse_attn(g, q, K, V, pos, ids, cnt, want, ws_attn, st, lse=want_lse)
        got = torch.full_like(want, float("nan"))
        got_lse = torch.full_like(want_lse, float("nan"))
        Z.zha_sparse_attn_noalloc(g, q, K, V, pos, ids, cnt, got, st, lse=got_lse)
        torch.cuda.synchronize()
        assert st.item() == 0
        err = (got.float() - want.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, (call, err.max().item())
        assert np.allclose(got_lse.cpu().numpy(), want_lse.cpu().numpy(), atol=1e-3, rtol=1e-4)


@pytest.mark.gpu
def test_noalloc_fp32_cache_at_the_enlarged_split():
    """fp32 caches take the CUDA-core split kernel; with 128 units the default split needs
    more than the fixed array, so the enlarged split (and its combine) runs; the result
    must be zha_sparse_attn's at the fp32 tolerance, on two calls in a row."""
    import hierarchical_sparse_attention_02_b200 as Z
    zbuild.build()
    Z.load_library()
    dev = "cuda"
    w = S.scaled(S.workload("tiny-decode-f32"), T=40000 + 21, B=32, n_centres=256)
    w = dataclasses.replace(w, Hq=32, Hkv=4)
    g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=w.depth, R=w.R, dtype=torch.float32)
    assert Z.workspace_bytes(g, 1, Z.ZHA_OP_ATTN) > _lib.ZHA_NOALLOC_SCRATCH_BYTES
    C, K, V = S.clustered_kv(w, dev)
    qref = S.reference_queries(w, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tree = Z.empty_tree(g, dev)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    pos = torch.full((w.B, 1), w.T - 1, dtype=torch.int64, device=dev)
    cap = Z.leaf_cap(g)
    ws_route = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE, dev)
    ws_attn = Z.empty_workspace(g, 1, Z.ZHA_OP_ATTN, dev)
    for call in range(2):
        q = S.queries(w, C, 1, dev, step=call)
        ids = torch.empty(w.B, 1, w.Hq, cap, dtype=torch.int32, device=dev)
        cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=dev)
        Z.zha_route(g, q, pos, 0.9, tree, ids, cnt, ws_route, st)
        want = torch.empty(w.B, 1, w.Hq, w.d, dtype=torch.float32, device=dev)
        Z.zha_sparse_attn(g, q, K, V, pos, ids, cnt, want, ws_attn, st)
        got = torch.full_like(want, float("nan"))
        Z.zha_sparse_attn_noalloc(g, q, K, V, pos, ids, cnt, got, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.isfinite(got).all()
        assert (got - want).abs().max().item() <= 1e-4, call
