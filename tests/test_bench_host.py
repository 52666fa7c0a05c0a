"""Host-side pieces of bench.py, on the CPU: the per-level frontier statistics, the
near-cutoff count of oracle routes, and the CPU-oracle reference arm's JSON line."""
import json
import math
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import zha_oracle as zo  # noqa: E402


def test_frontier_stats_per_level():
    # 3 heads, depth 3: head 0 routes levels 3..1, head 1 only levels 2..1, head 2 nothing
    lc = np.zeros((1, 1, 3, 3, 2), np.int32)
    lc[0, 0, 0] = [[40, 10], [64, 8], [4, 2]]
    lc[0, 0, 1] = [[20, 5], [16, 4], [0, 0]]
    out = bench.frontier_stats(lc)
    assert [o["level"] for o in out] == [3, 2, 1]
    top, mid, leaf = out
    assert top["heads"] == 1 and top["candidates_mean"] == 4 and top["kept_max"] == 2
    assert mid["heads"] == 2 and mid["candidates_mean"] == 40 and mid["kept_p50"] == 6
    assert leaf["heads"] == 2 and leaf["candidates_max"] == 40 and leaf["kept_mean"] == 7.5


def test_near_cutoff_count_of_oracle_routes():
    d = 8
    rng = np.random.default_rng(3)
    K = rng.standard_normal((256, d))
    qref = rng.standard_normal((2, d)) / math.sqrt(d)
    tree = zo.build_tree(K, 256, qref, depth=2, leaf=4, branch=4, route_storage="f64")
    routes = [zo.route(rng.standard_normal(d), 255, tree, 0.9) for _ in range(5)]
    out = bench.near_cutoff_count(routes)
    assert out["heads"] == 5 and out["levels"] == 10
    want = sum(min(s.margin, s.gap) < 1e-4 for r in routes for s in r.sel.values())
    assert out["near_cutoff"] == want
    # a route whose top level holds two equal scores is near-cutoff there (gap 0)
    flat = zo.build_tree(np.ones((64, d)), 64, qref, depth=2, leaf=4, branch=4, route_storage="f64")
    r = zo.route(np.ones(d), 63, flat, 0.5)
    assert bench.near_cutoff_count([r])["near_cutoff"] == 2


def test_reference_arm_line_on_cpu():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny-decode-f32", "--steps", "1", "--warmup", "0",
                          "--cpu-seconds", "0.5"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    for key in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "e2e"):
        assert key in line


def _gpu_layout(routes_by_head, depth, n_cap):
    """Oracle routes of one sequence's heads in zha_route's level_cnt / level_ids layout."""
    Hq = len(routes_by_head)
    lc = np.zeros((1, 1, Hq, depth, 2), np.int32)
    lids = np.full((1, 1, Hq, sum(n_cap.values())), -1, np.int32)
    for h, r in enumerate(routes_by_head):
        off = 0
        for l in range(2, depth + 1):
            if l in r.sel:
                lc[0, 0, h, l - 1] = (len(r.cand[l]), r.sel[l].m)
                lids[0, 0, h, off:off + r.sel[l].m] = r.sel[l].ids
            off += n_cap[l]
        lc[0, 0, h, 0] = (len(r.cand[1]), r.sel[1].m)
    return lc, lids


def test_candidate_unions_match_the_oracle_candidate_sets():
    d, leaf, branch, depth = 8, 4, 4, 3
    T = 4 * 4 * 4 * 3 + 4 * 4 + 3 * 4 + 2          # orphans at levels 1 and 2
    rng = np.random.default_rng(8)
    C = rng.standard_normal((4, d))
    K = C[rng.integers(0, 4, T + 1)] + 0.3 * rng.standard_normal((T + 1, d))
    qref = rng.standard_normal((2, d)) / math.sqrt(d)
    tree = zo.build_tree(K, T + 1, qref, depth=depth, leaf=leaf, branch=branch, route_storage="f64")
    G = 4
    routes = [zo.route(2 * C[h % 4] + 0.3 * rng.standard_normal(d), T, tree, 0.6) for h in range(2 * G)]
    n_cap = {l: (T + 1) // (leaf * branch ** (l - 1)) for l in range(2, depth + 1)}
    lc, lids = _gpu_layout(routes, depth, n_cap)
    v = leaf * (T // leaf)
    nvis = {l: v // (leaf * branch ** (l - 1)) for l in range(1, depth + 1)}
    got = bench.candidate_unions(lc, lids, n_cap, nvis, G, branch)
    assert sorted(got) == [1, 2, 3]
    for l in (1, 2, 3):
        want = np.mean([len(np.unique(np.concatenate([r.cand[l] for r in routes[g:g + G]])))
                        for g in (0, G)])
        assert got[l] == want


def test_paper_model_terms():
    line = {"dtype": "bf16", "steps": 10, "gpu_launches": 80,
            "config": {"workload": "w", "B": 2, "Hq": 16, "Hkv": 2, "d": 128, "R": 4, "T": 65536,
                       "leaf": 64, "branch": 16, "depth": 3},
            "frontier": {"levels": [
                {"level": 2, "candidates_mean": 64.0, "candidates_max": 64, "candidates_group_union": 64.0},
                {"level": 1, "candidates_mean": 900.0, "candidates_max": 950, "candidates_group_union": 1000.0}]},
            # depth 3 with an empty top level: three launches per kind, level 3 first
            "stages_ms": {"route_score_per_launch": [0.004, 0.01, 0.02],
                          "route_select_per_launch": [0.003, 0.005, 0.01],
                          "attention": 0.05, "step": 0.1, "stage_sum": 0.095},
            "kv_touched": {"mean": 0.5}, "tree_build": {"ms": 0.4},
            "roofline": {"algorithmic_bytes_per_launch": 1e8, "launches_per_step": 1.0}}
    peaks = {"hbm_gbs": 5000.0, "bf16_tflops": 1000.0}
    m = bench.paper_model(line, peaks)
    rows = {r["stage"]: r for r in m["rows"]}
    r1 = rows["route score L1"]
    # 2 B Hq R d K flops; R (s d + 4) B Hkv K_grp + s d B Hq bytes
    assert r1["flops"] == 2 * 2 * 16 * 4 * 128 * 900.0
    assert r1["bytes"] == 4 * (2 * 128 + 4) * 2 * 2 * 1000.0 + 2 * 128 * 2 * 16
    assert r1["model_ms"] == pytest.approx(max(1e3 * r1["flops"] / 40e12, 1e3 * r1["bytes"] / 5e12, 0.01))
    assert r1["measured_ms"] == 0.02 and rows["route score L2"]["measured_ms"] == 0.01
    # the wave term: the top level's launch (level 2 here) calibrates tau
    assert rows["route score L2"]["waves_ms"] == 0.01 and rows["route select L1"]["waves_ms"] == 0.005
    assert rows["route select L2"]["bytes"] == 12 * 2 * 16 * 64.0
    att = rows["attention"]
    assert att["bytes"] == 1e8 and att["model_ms"] == pytest.approx(1e3 * 1e8 / 5e12)
    assert att["measured_over_model"] == pytest.approx(0.05 / att["model_ms"])
    # launch overhead: the gaps between kernels plus the launches of the empty level 3
    assert m["launch_gaps_ms"] == pytest.approx(0.005 + 0.004 + 0.003) and m["launches_per_step"] == 8
    assert rows["route L3 (empty)"]["measured_ms"] == pytest.approx(0.007)


def test_oracle_pool_parity_check_on_cpu():
    """The bench's CPU-oracle pool: a step on spawned workers, then the parity summary of
    GPU-shaped results made up on the host (the oracle's own lists and outputs: all exact;
    one list with a far-off chunk: a failure)."""
    import zha_synth as S
    w = S.scaled(S.workload("batched-decode-128k"), T=4096 + 70, B=1, n_centres=64)
    pool = bench.OraclePool.from_workload(w, 0.9, "cpu", workers=3)
    try:
        r = bench.oracle_sample(pool, 30.0)
        assert r["heads"] == w.Hq and r["value"] > 0 and len(r["flags"]) == w.Hq
        one = S.scaled(w, T=w.T, B=1)
        C, K, V = S.clustered_kv(one, "cpu")
        kn, vn = S.new_tokens(one, C, 1, "cpu")
        q = S.queries(one, C, 1, "cpu")[0, 0].double().numpy()
        K[:, :, w.T], V[:, :, w.T] = kn[:, 0], vn[:, 0]
        qref = S.reference_queries(one, "cpu").double().numpy()
        leaves, outs = {}, {}
        for hk in range(w.Hkv):
            tree = zo.build_tree(K[0, hk], w.T + 1, qref[hk], w.depth)
            for h in range(hk * w.G, (hk + 1) * w.G):
                rt, o, _ = zo.decode_head(q[h], K[0, hk], V[0, hk], w.T, tree, 0.9)
                leaves[h], outs[h] = rt.leaves, o
        got = pool.check(leaves, outs)
        assert got["heads"] == w.Hq and got["exact"] == w.Hq and got["failed"] == 0
        assert got["max_abs_err"] < 1e-12
        bad = dict(leaves)
        bad[3] = np.union1d(leaves[3], [w.T // 64 - 1])[-len(leaves[3]) - 1:]
        if len(leaves[3]) == w.T // 64:
            bad[3] = leaves[3][1:]
        got = pool.check(bad, outs)
        assert got["exact"] == w.Hq - 1 and got["failed"] + got["near_cutoff_mismatch"] == 1
    finally:
        pool.close()


def test_paper_model_with_the_fused_top_levels():
    """Lines whose small top levels share one fused launch: the per-level lists start at the
    first level launched on its own, and the fused levels form one row."""
    line = {"dtype": "bf16", "steps": 10, "gpu_launches": 80,
            "config": {"workload": "w", "B": 4, "Hq": 32, "Hkv": 4, "d": 128, "R": 4, "T": 1 << 20,
                       "leaf": 64, "branch": 16, "depth": 5},
            "frontier": {"levels": [
                {"level": 4, "candidates_mean": 4.0, "candidates_max": 4},
                {"level": 3, "candidates_mean": 64.0, "candidates_max": 64},
                {"level": 2, "candidates_mean": 976.0, "candidates_max": 976},
                {"level": 1, "candidates_mean": 14700.0, "candidates_max": 14750}]},
            "stages_ms": {"route_fused": 0.01, "route_fused_per_launch": [0.01],
                          "route_score_per_launch": [0.02, 0.15], "route_select_per_launch": [0.015, 0.04],
                          "attention": 1.2, "step": 1.5, "stage_sum": 1.435},
            "kv_touched": {"mean": 0.8}, "tree_build": {"ms": 3.6},
            "roofline": {"algorithmic_bytes_per_launch": 8e9, "launches_per_step": 1.0}}
    m = bench.paper_model(line, {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0})
    rows = {r["stage"]: r for r in m["rows"]}
    assert rows["route fused L4..L3"]["measured_ms"] == 0.01
    assert rows["route score L2"]["measured_ms"] == 0.02 and rows["route score L1"]["measured_ms"] == 0.15
    assert rows["route select L1"]["measured_ms"] == 0.04
    assert "route score L4" not in rows and "route score L3" not in rows
    assert m["launch_gaps_ms"] == pytest.approx(1.5 - 1.435)


def test_paper_model_wave_term_needs_a_one_wave_launch():
    """The wave term of the score and select rows is calibrated from the highest level
    launched on its own only when that level lies above the leaves.  When every level above
    the leaves is fused, no launch of those kernels fits one wave: the level-1 rows keep only
    their flop and byte terms.  The fused row takes its own launch as its wave term."""
    line = {"dtype": "bf16", "steps": 10, "gpu_launches": 60,
            "config": {"workload": "w", "B": 32, "Hq": 32, "Hkv": 4, "d": 128, "R": 4, "T": 1 << 17,
                       "leaf": 64, "branch": 16, "depth": 3},
            "frontier": {"levels": [
                {"level": 3, "candidates_mean": 8.0, "candidates_max": 8},
                {"level": 2, "candidates_mean": 128.0, "candidates_max": 128},
                {"level": 1, "candidates_mean": 1936.0, "candidates_max": 1936,
                 "candidates_group_union": 2048.0}]},
            "stages_ms": {"route_fused": 0.06, "route_fused_per_launch": [0.06],
                          "route_score_per_launch": [0.149], "route_select_per_launch": [0.045],
                          "attention": 1.25, "step": 1.55, "stage_sum": 1.504},
            "kv_touched": {"mean": 0.87}, "tree_build": {"ms": 3.6},
            "roofline": {"algorithmic_bytes_per_launch": 8.6e9, "launches_per_step": 1.0}}
    m = bench.paper_model(line, {"hbm_gbs": 6448.4, "bf16_tflops": 1725.8})
    rows = {r["stage"]: r for r in m["rows"]}
    fused = rows["route fused L3..L2"]
    assert fused["waves_ms"] == 0.06 and fused["model_ms"] == pytest.approx(0.06)
    score, select = rows["route score L1"], rows["route select L1"]
    assert score["waves_ms"] == 0.0 and select["waves_ms"] == 0.0
    # no wave term: the score row is its fp64 flops (2 B Hq R d K) over the fp64 tensor rate
    flops = 2.0 * 32 * 32 * 4 * 128 * 1936.0
    assert score["model_ms"] == pytest.approx(1e3 * flops / (bench.FP64_TENSOR_TFLOPS * 1e12))
    assert score["bound"] == "fp64 tensor"
    # the select row is its bytes (12 B Hq K) over the copy bandwidth
    assert select["model_ms"] == pytest.approx(1e3 * 12.0 * 32 * 32 * 1936.0 / (6448.4e9))
    assert select["bound"] == "hbm"
    # a line whose highest separate level lies above the leaves does calibrate from it
    line2 = dict(line)
    line2["config"] = dict(line["config"], depth=3)
    line2["stages_ms"] = dict(line["stages_ms"], route_fused=0.0, route_fused_per_launch=[],
                              route_score_per_launch=[0.013, 0.02, 0.149],
                              route_select_per_launch=[0.011, 0.013, 0.045])
    m2 = bench.paper_model(line2, {"hbm_gbs": 6448.4, "bf16_tflops": 1725.8})
    rows2 = {r["stage"]: r for r in m2["rows"]}
    assert rows2["route score L1"]["waves_ms"] == 0.013 and rows2["route select L2"]["waves_ms"] == 0.011
    assert rows2["route score L3"]["bound"] == "latency (one wave)"
