"""Host-side pieces of bench.py, on the CPU: the per-level frontier statistics, the
near-cutoff count of oracle routes, and the CPU-oracle reference arm's JSON line."""
import json
import math
import os
import subprocess
import sys

import numpy as np

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
