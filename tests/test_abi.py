"""The C-ABI library on the host: it loads, exports every symbol include/zha.h declares,
and rejects bad arguments before it enqueues anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

from hierarchical_sparse_attention_02_b200 import _lib
from hierarchical_sparse_attention_02_b200 import build as zbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    zbuild.build()
    return _lib.load()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "zha.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+(zha_[a-z_]+)\s*\(", src, flags=re.M)


def test_exports_every_declared_symbol(lib):
    decl = declared_symbols()
    assert len(decl) == 22
    assert sorted(decl) == sorted(_lib.EXPORTS)
    for name in decl:
        assert hasattr(lib, name), name


def geom(**kw):
    base = dict(B=2, Hq=16, Hkv=2, d=128, leaf=64, branch=16, depth=3, R=4, t_cap=65536, dtype=1, rope_pairs=0)
    base.update(kw)
    return _lib.Geom(**base)


def test_status_strings(lib):
    assert lib.zha_status_str(0) == b"ok"
    assert lib.zha_status_str(3) == b"capacity exceeded"
    assert lib.zha_status_str(99) == b"unknown status"


@pytest.mark.parametrize("kw,code", [
    ({}, 0), ({"d": 64}, 2), ({"leaf": 32}, 2), ({"Hq": 15}, 1), ({"Hq": 64, "Hkv": 2}, 2),
    ({"R": 17}, 2), ({"R": 0}, 1), ({"R": 3}, 2), ({"R": 16}, 0), ({"R": 1}, 0), ({"depth": 9}, 2), ({"branch": 1}, 2), ({"t_cap": 1000}, 1),
    ({"dtype": 7}, 2), ({"rope_pairs": 65}, 1), ({"rope_pairs": -1}, 1), ({"rope_pairs": 64}, 0),
    ({"rope_pairs": 16}, 0), ({"B": 0}, 1),
    # a cache whose byte count (at 4 bytes per element) passes 2^48: 2^20 * 2 * 2^28 * 512 = 2^58
    ({"B": 1 << 20, "t_cap": 1 << 28}, 2),
    # the largest cache of the decode workloads (16M keys) is well inside the bound
    ({"B": 1, "Hq": 8, "Hkv": 1, "depth": 6, "t_cap": 1 << 24}, 0),
])
def test_check_geom(lib, kw, code):
    assert lib.zha_check_geom(ctypes.byref(geom(**kw))) == code


def test_sizes(lib):
    g = geom()
    assert lib.zha_leaf_cap(ctypes.byref(g)) == 1024
    tb = lib.zha_tree_bytes(ctypes.byref(g))
    lv = _lib.LevelLayout()
    total = 0
    for level in (1, 2, 3):
        assert lib.zha_tree_level(ctypes.byref(g), level, ctypes.byref(lv)) == 0
        assert lv.span == 64 * 16 ** (level - 1)
        assert lv.n_cap == 65536 // lv.span
        assert lv.k_route_off % 256 == 0 and lv.k_state_off % 256 == 0
        total = lv.k_state_off + 2 * 2 * lv.n_cap * 4 * 128 * 4
    assert tb >= total
    assert lib.zha_tree_level(ctypes.byref(g), 4, ctypes.byref(lv)) == 1
    for op in (1, 2, 3, 4, 5):
        assert lib.zha_workspace_bytes(ctypes.byref(g), 1, op) > 0
    assert lib.zha_workspace_bytes(ctypes.byref(g), 0, 1) == 0
    assert lib.zha_workspace_bytes(ctypes.byref(g), 1, 9) == 0
    assert lib.zha_tree_bytes(ctypes.byref(geom(d=64))) == 0


def test_host_side_rejections_enqueue_nothing(lib):
    """Invalid calls return before any launch; the pointers are never dereferenced."""
    g = geom()
    fake = ctypes.c_void_p(0x1000)
    buf = _lib.Buf(0x1000, 1 << 40)
    small = _lib.Buf(0x1000, 16)
    n0 = lib.zha_launch_count()
    # the bounded-wait check: polls outside [1, 2^32], null pointers
    for polls, st, out in ((0, fake, fake), (1 << 33, fake, fake), (100, None, fake), (100, fake, None)):
        assert lib.zha_check_bounded_wait(polls, st, out, None) == 1
    # p outside (0, 1]
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert lib.zha_route(ctypes.byref(g), fake, fake, 1, p, buf, fake, fake, 8, None, None, buf, fake, None) == 1
    # null pointers
    assert lib.zha_route(ctypes.byref(g), None, fake, 1, 0.9, buf, fake, fake, 8, None, None, buf, fake, None) == 1
    assert lib.zha_sparse_attn(ctypes.byref(g), fake, fake, fake, fake, 1, fake, fake, 8, fake, None, buf, None,
                               None) == 1
    # buffers too small
    assert lib.zha_build_tree(ctypes.byref(g), fake, 100, fake, small, fake, None) == 3
    assert lib.zha_route(ctypes.byref(g), fake, fake, 1, 0.9, buf, fake, fake, 8, None, None, small, fake,
                         None) == 3
    # positions beyond the cache
    assert lib.zha_build_tree(ctypes.byref(g), fake, 65537, fake, buf, fake, None) == 1
    assert lib.zha_decode(ctypes.byref(g), fake, fake, fake, fake, fake, 65536, fake, 0.9, buf, fake, fake, 8,
                          fake, buf, fake, None) == 1
    assert lib.zha_append(ctypes.byref(g), fake, fake, fake, fake, 65000, 600, fake, buf, fake, None) == 1
    # bad geometry
    bad = geom(d=256)
    assert lib.zha_decode(ctypes.byref(bad), fake, fake, fake, fake, fake, 5, fake, 0.9, buf, fake, fake, 8,
                          fake, buf, fake, None) == 2
    assert lib.zha_launch_count() == n0


def test_sizes_that_would_overflow_are_rejected(lib):
    """Per-call arrays past 2^48 bytes: the workspace size is 0 and every entry point that
    takes nq returns ZHA_ERR_UNSUPPORTED before it enqueues anything."""
    g = geom()
    fake = ctypes.c_void_p(0x1000)
    buf = _lib.Buf(0x1000, (1 << 64) - 1)
    huge = (1 << 31) - 1          # 2 * huge * 16 heads * 1026 chunks * 8 bytes > 2^48
    for op in (1, 2, 3, 4, 5):
        assert lib.zha_workspace_bytes(ctypes.byref(g), huge, op) == 0
    assert lib.zha_workspace_bytes(ctypes.byref(g), 1 << 20, 1) > 0
    n0 = lib.zha_launch_count()
    assert lib.zha_route(ctypes.byref(g), fake, fake, huge, 0.9, buf, fake, fake, 8, None, None, buf, fake,
                         None) == 2
    assert lib.zha_sparse_attn(ctypes.byref(g), fake, fake, fake, fake, huge, fake, fake, 8, fake, None, buf,
                               fake, None) == 2
    assert lib.zha_dense_decode(ctypes.byref(g), fake, fake, fake, fake, huge, fake, None, buf, fake, None) == 2
    assert lib.zha_flat_index(ctypes.byref(g), fake, fake, fake, fake, huge, 0.9, fake, fake, 8, fake, buf,
                              fake, None) == 2
    assert lib.zha_sparse_attn_noalloc(ctypes.byref(g), fake, fake, fake, fake, huge, fake, fake, 8, fake,
                                       None, fake, None) == 2
    assert lib.zha_launch_count() == n0


def test_route_schedule_rejections(lib):
    """Per-level thresholds: a null array or any level outside (0, 1] is rejected before any
    launch; only the first `depth` entries are read."""
    g = geom()                                  # depth 3
    fake = ctypes.c_void_p(0x1000)
    buf = _lib.Buf(0x1000, 1 << 40)
    n0 = lib.zha_launch_count()
    arr = lambda *v: (ctypes.c_double * len(v))(*v)  # noqa: E731
    for bad in (arr(0.9, 0.0, 0.9), arr(0.9, 0.9, 1.5), arr(float("nan"), 0.9, 0.9), arr(-1.0, 1.0, 1.0)):
        assert lib.zha_route_schedule(ctypes.byref(g), fake, fake, 1, bad, buf, fake, fake, 8, None, None, buf,
                                      fake, None) == 1
    assert lib.zha_route_schedule(ctypes.byref(g), fake, fake, 1, None, buf, fake, fake, 8, None, None, buf,
                                  fake, None) == 1
    good = arr(0.9, 1.0, 0.5, 7.0)             # the fourth entry is past the depth: never read
    assert lib.zha_route_schedule(ctypes.byref(g), fake, fake, 1, good, buf, fake, fake, 8, None, None,
                                  _lib.Buf(0x1000, 16), fake, None) == 3
    assert lib.zha_launch_count() == n0


def test_reference_block_layout_and_size_check():
    """The tree calls read Hkv*R*d reference values plus rope_pairs frequencies: the binding
    builds that block and refuses a tensor of another size before calling the library."""
    import torch
    import hierarchical_sparse_attention_02_b200 as Z
    qref = torch.randn(2, 4, 128)
    f = torch.tensor([1.0, 0.5, 0.25])
    qb = Z.reference_block(qref, f)
    assert qb.shape == (2 * 4 * 128 + 3,) and qb.dtype == torch.float32
    assert torch.equal(qb[:-3].view(2, 4, 128), qref) and torch.equal(qb[-3:], f)
    assert torch.equal(Z.reference_block(qref), qref.reshape(-1))
    g = Z.Geometry(B=1, Hq=8, Hkv=2, t_cap=4096, depth=2, R=4, rope_pairs=3)
    n0 = Z.launch_count()
    with pytest.raises(ValueError, match="qref"):
        Z.zha_build_tree(g, None, 0, qref.reshape(-1), None, None)          # frequencies missing
    with pytest.raises(ValueError, match="qref"):
        Z.zha_decode(g, None, None, None, None, None, 0, qref.double(), 0.9, None, None, None, None, None,
                     None)                                                   # fp64, not fp32
    assert Z.launch_count() == n0


def test_route_topk_rejections(lib):
    """Per-level counts: a null array or a count below 1 is rejected before any launch."""
    g = geom()                                  # depth 3
    fake = ctypes.c_void_p(0x1000)
    buf = _lib.Buf(0x1000, 1 << 40)
    n0 = lib.zha_launch_count()
    arr = lambda *v: (ctypes.c_int32 * len(v))(*v)  # noqa: E731
    for bad in (arr(4, 0, 4), arr(-1, 4, 4), arr(4, 4, -7)):
        assert lib.zha_route_topk(ctypes.byref(g), fake, fake, 1, bad, buf, fake, fake, 8, None, None, buf,
                                  fake, None) == 1
    assert lib.zha_route_topk(ctypes.byref(g), fake, fake, 1, None, buf, fake, fake, 8, None, None, buf,
                              fake, None) == 1
    assert lib.zha_route_topk(ctypes.byref(g), fake, fake, 1, arr(1, 2, 3, 0), buf, fake, fake, 8, None, None,
                              _lib.Buf(0x1000, 16), fake, None) == 3
    assert lib.zha_launch_count() == n0


def _prototypes():
    """name -> (return type, [parameter types]) of every prototype in include/zha.h."""
    src = open(os.path.join(ROOT, "include", "zha.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*((?:const\s+)?[a-z_0-9]+\s*\*?)\s*(zha_[a-z_]+)\s*\(([^)]*)\)\s*;", src, flags=re.M):
        params = [p.strip() for p in m.group(3).replace("\n", " ").split(",") if p.strip() and p.strip() != "void"]
        types = [re.sub(r"\s*\b[a-z_A-Z0-9]+$", "", p).strip() if not p.endswith("*") else p for p in params]
        out[m.group(2)] = (m.group(1).replace(" ", ""), [t.replace(" ", "") for t in types])
    return out


_C_TO_CTYPES = {
    "int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "double": ctypes.c_double, "size_t": ctypes.c_size_t,
    "zha_status": ctypes.c_int32, "zha_buf": "Buf", "constchar*": ctypes.c_char_p, "void": None,
}


def test_ctypes_signatures_match_the_header():
    """Every entry point's ctypes signature has the header's parameter count and, parameter by
    parameter, the same kind (pointer, 32/64-bit integer, double, buffer struct): a mismatch
    would pass garbage through the ABI on a GPU."""
    protos = _prototypes()
    assert sorted(protos) == sorted(_lib._SIGS)
    for name, (ret, params) in protos.items():
        cret, cargs = _lib._SIGS[name]
        assert len(cargs) == len(params), (name, params)
        want_ret = _C_TO_CTYPES.get(ret)
        assert cret == want_ret, (name, ret, cret)
        for i, (p, c) in enumerate(zip(params, cargs)):
            if p.endswith("*"):                       # any pointer
                assert c is ctypes.c_void_p or issubclass(c, ctypes._Pointer), (name, i, p, c)
            else:
                want = _C_TO_CTYPES[p]
                assert (c is _lib.Buf) if want == "Buf" else (c is want), (name, i, p, c)


def test_struct_layouts_match_the_header(tmp_path):
    """zha_geom, zha_buf and zha_level_layout as the C compiler lays them out (sizes and field
    offsets, from a program compiled against include/zha.h) equal the ctypes structures."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = {"zha_geom": [f for f, _ in _lib.Geom._fields_],
              "zha_buf": [f for f, _ in _lib.Buf._fields_],
              "zha_level_layout": [f for f, _ in _lib.LevelLayout._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "zha.h"', "int main(void) {"]
    for s, fs in fields.items():
        lines.append(f'  printf("{s} size %zu\\n", sizeof({s}));')
        for f in fs:
            lines.append(f'  printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for s, cls in (("zha_geom", _lib.Geom), ("zha_buf", _lib.Buf), ("zha_level_layout", _lib.LevelLayout)):
        assert got[(s, "size")] == ctypes.sizeof(cls), s
        for f in fields[s]:
            assert got[(s, f)] == getattr(cls, f).offset, (s, f)


def test_prefill_host_rejections_enqueue_nothing(lib):
    """zha_prefill_attn serves bf16 caches only and checks its pointers, sizes and workspace
    on the host, before anything is enqueued; its workspace grows with the query count."""
    g = geom()
    fake = ctypes.c_void_p(0x1000)
    buf = _lib.Buf(0x1000, 1 << 40)
    n0 = lib.zha_launch_count()
    op = _lib.ZHA_OP_PREFILL
    w16 = lib.zha_workspace_bytes(ctypes.byref(g), 16, op)
    w64 = lib.zha_workspace_bytes(ctypes.byref(g), 64, op)
    assert 0 < w16 < w64
    small = _lib.Buf(0x1000, w16 - 1)

    def call(gg, q_pos=fake, nq=16, ids=fake, cap=8, ws=buf, st=fake):
        return lib.zha_prefill_attn(ctypes.byref(gg), fake, fake, fake, q_pos, nq, ids, fake, cap, fake, None,
                                    ws, st, None)

    assert call(geom(dtype=0)) == _lib.ZHA_ERR_UNSUPPORTED            # fp32 caches
    assert call(geom(d=256)) == _lib.ZHA_ERR_UNSUPPORTED              # bad geometry
    assert call(g, q_pos=None) == _lib.ZHA_ERR_INVALID_ARG            # positions are required
    assert call(g, nq=0) == _lib.ZHA_ERR_INVALID_ARG
    assert call(g, ids=None) == _lib.ZHA_ERR_INVALID_ARG
    assert call(g, cap=0) == _lib.ZHA_ERR_INVALID_ARG
    assert call(g, st=None) == _lib.ZHA_ERR_INVALID_ARG
    assert call(g, ws=small) == _lib.ZHA_ERR_CAPACITY                 # workspace one byte short
    assert lib.zha_launch_count() == n0
