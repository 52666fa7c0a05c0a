"""The multi-GPU benchmark path on the host: two gloo ranks, world size 2.

Each rank runs an independent replica (the path shards over (sequence, KV head) units with
no exchange), so the only cross-rank operations are the barrier and the maximum of the
per-rank step times; the whole-job rate is the units of all ranks over the slowest rank's
time (weak scaling).  The per-rank inputs differ (the seed is offset by the rank).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import zha_synth as S
        # replicas draw different data (bench offsets the seed by 1000 * rank)
        w = S.scaled(S.workload("batched-decode-128k"), T=256, B=1, n_centres=8)
        wr = S.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank}) if rank else w
        k = S.clustered_kv(wr)[1]
        bench.barrier(ws)
        ms_local = 2.0 + rank                       # rank 1 is the slower one
        ms, value = bench.whole_job_rate(1024, ms_local, ws)
        out[rank] = (ms, value, float(k.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    (ms0, v0, k0), (ms1, v1, k1) = out[0], out[1]
    assert ms0 == ms1 == 3.0                      # every rank reports the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 1024 / 3.0e-3)
    assert k0 != k1                               # independent replicas


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.whole_job_rate(10, 2.0, 1) == (2.0, 10 / 2.0e-3)
