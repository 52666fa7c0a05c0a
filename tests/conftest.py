import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The routing tallies of the GPU parity tests (heads whose kept sets equal the
    oracle's at every level, heads that differ only at a near cutoff, mismatches), one line
    per comparison and a total, so that they are visible in a quiet run."""
    reps, seen = [], set()
    for mod in ("tests.zha_cases", "zha_cases"):       # the tests import it as tests.zha_cases
        cases = sys.modules.get(mod)
        for name, r in (cases.ROUTE_REPORTS if cases is not None else []):
            if id(r) not in seen and r.heads and "test_gpu" in name:
                seen.add(id(r))
                reps.append((name, r))
    if not reps:
        return
    terminalreporter.section("routing against the oracle (GPU tests)")
    for name, r in reps:
        status = "" if r.ok() else "  FAILED: " + "; ".join(r.problems())
        terminalreporter.write_line(f"{name}: {r.summary()}{status}")
    heads = sum(r.heads for _, r in reps)
    exact = sum(r.exact for _, r in reps)
    near = sum(r.near_cutoff for _, r in reps)
    bad = sum(len(r.mismatched) for _, r in reps)
    terminalreporter.write_line(f"total: {exact} exact, {near} near-cutoff mismatches, {bad} mismatched "
                                f"of {heads} heads in {len(reps)} comparisons")
