"""Benchmark of the ZHA decode hot path on B200.

One step = one decode token for every sequence of the workload: append the new key/value
(and summarise any node it completes), route every query head top-down with top-p, and
attend over the selected index set (zha_decode: all kernels of the hot path).  Inputs are
seeded synthetic clustered keys; the KV cache (8 GiB for the default workload) is larger
than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl zha|reference]
                    [--workload NAME] [--p P] [--path zha|dense|flat|prefill]

The default workload is the 1M-token decode (long-decode-1m).  `--path prefill` times the
query-tile prefill attention (zha_prefill_attn) on the chunked-prefill workload against the
per-query path over the same leaf lists.  `--sweep` runs the crossover sweep over T,
`--segment N` the structured variant of the generator, and `--model FILE` the pages' roofline
model over saved bench lines (no GPU work).

Multi-GPU: one process per GPU (torchrun); every rank runs its own independent replica of
the workload (the path shards over (sequence, KV head) units with no exchange), so the
scaling is weak and the reported value is the sum over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import zha_synth as S  # noqa: E402

DEFAULT_WORKLOAD = "long-decode-1m"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="zha", choices=["zha", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(S.WORKLOADS))
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU budget of one sampled oracle step, per worker process")
    ap.add_argument("--cpu-workers", type=int, default=0,
                    help="oracle worker processes (0: one per host core, at most one per query head)")
    ap.add_argument("--segment", type=int, default=0,
                    help="structured keys: runs of this many positions share a cluster centre "
                         "(a variant of the generator, not one of the five workloads)")
    ap.add_argument("--rope", type=int, default=0, metavar="H",
                    help="rotary tree: reference queries rotated with H RoPE frequencies (base 10000 "
                         "over 2H dims; the keys stay as generated)")
    ap.add_argument("--graph", action="store_true",
                    help="capture the step once in a CUDA graph and replay it in the timed loop "
                         "(the dominant kernel's duration then comes from traced, uncaptured steps)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--n-new", type=int, default=None,
                    help="prefill path: appended queries (default: the workload's 4096)")
    ap.add_argument("--path", default="zha", choices=["zha", "dense", "flat", "prefill"],
                    help="zha: the hot path (default); dense / flat: the baselines on the same inputs; "
                         "prefill: the query-tile attention of the chunked-prefill workload")
    ap.add_argument("--sweep", action="store_true",
                    help="crossover sweep over T and depth against the dense kernel (one JSON line each)")
    ap.add_argument("--model", metavar="FILE", default=None,
                    help="no GPU work: read bench JSON lines of the zha path from FILE and print the "
                         "pages' roofline model of each beside its measured stage times")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# process group
# ---------------------------------------------------------------------------


def dist_setup(n):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The maximum of x over the ranks (NCCL on the GPU, gloo on the host)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, ms_local: float, ws: int) -> tuple:
    """(slowest rank's ms per step, whole-job units per second): every rank processes
    `units_per_rank` units per step (weak scaling), the job takes as long as its slowest rank."""
    ms = max_over_ranks(ms_local, ws)
    return ms, ws * units_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        self.why = None
        # the physical GPU: CUDA_VISIBLE_DEVICES may renumber devices, nvidia-smi does not
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        index = str(device)
        if vis:
            parts = [p.strip() for p in vis.split(",") if p.strip()]
            if device < len(parts):
                index = parts[device]
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", index, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.PIPE)
        except Exception as e:  # noqa: BLE001
            self.proc = None
            self.why = f"nvidia-smi unavailable: {type(e).__name__}: {e}"
        self.t_start = self.t_end = None

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.why], "samples": 0}
        t_busy_end = time.time()
        time.sleep(0.25)
        self.proc.terminate()
        err = b""
        try:
            _, err = self.proc.communicate(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        import datetime
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], parts[4], ts))
            except ValueError:
                continue
        # samples from the start of the timed region on (the end-to-end steps that follow it
        # keep the GPU on the same work)
        if self.t_start is not None:
            busy = [r for r in rows if self.t_start - 0.05 <= r[4] <= t_busy_end]
            rows = busy or rows
        os.unlink(self.path)
        if not rows:
            msg = (err or b"").decode(errors="replace").strip()[:200]
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no samples: {msg}"], "samples": 0}
        # keep the samples taken while the GPU was busy (highest-clock half if the tail idles)
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the attention
# gather kernel, from ncu captures of the 1M-token decode at batch 1 (4 of its 16 KV units)
# and of the batched 128K decode at batch 4 (16 of its 128 KV units), each valid while the
# kernel source is the one that was captured.
PROFILED_TRAFFIC = {
    "long-decode-1m": {"bytes": 2.149206784e9 + 18.750208e6, "units": 4,
                       "source": "hierarchical_sparse_attention_02_b200/csrc/zha_attn_tc.cu",
                       "sha1": "66fb0e96b0d9ccbdee5e0bc5c25088c89c77ee09"},
    "batched-decode-128k": {"bytes": 1.075083776e9 + 11.032576e6, "units": 16,
                            "source": "hierarchical_sparse_attention_02_b200/csrc/zha_attn_tc.cu",
                            "sha1": "66fb0e96b0d9ccbdee5e0bc5c25088c89c77ee09"},
}


def profiled_traffic(w, units: int):
    import hashlib
    rec = PROFILED_TRAFFIC.get(w.name)
    if rec is None:
        return None
    try:
        digest = hashlib.sha1(open(os.path.join(ROOT, rec["source"]), "rb").read()).hexdigest()
    except OSError:
        return None
    if digest != rec["sha1"]:
        return None                                      # the kernel changed since the capture
    return rec["bytes"] * units / rec["units"]           # traffic grows with the units gathered


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------


NEAR_CUTOFF = 1e-4      # a level whose cutoff margin or boundary gap is below this is "near-cutoff"


def near_cutoff_count(routes) -> dict:
    """Near-cutoff levels among oracle routes: (query head, level) pairs whose cumulative
    mass at the cutoff lies within NEAR_CUTOFF of p, or whose two candidates at the
    boundary differ by less than NEAR_CUTOFF in softmax mass.  There a one-ulp difference
    in a score may legitimately change the kept set."""
    return near_cutoff_from_flags([[min(s.margin, s.gap) for s in r.sel.values()] for r in routes])


def near_cutoff_from_flags(flags) -> dict:
    """The same from per-head lists of min(margin, gap), one entry per routed level."""
    levels = sum(len(f) for f in flags)
    near = sum(int(x < NEAR_CUTOFF) for f in flags for x in f)
    return {"heads": len(flags), "levels": levels, "near_cutoff": near, "threshold": NEAR_CUTOFF}


def frontier_stats(level_cnt: np.ndarray) -> list:
    """Per-level frontier sizes from zha_route's level counts [..., depth, 2] (candidates,
    kept) of every query head: mean / p50 / max over the heads that route that level."""
    lc = np.asarray(level_cnt).reshape(-1, level_cnt.shape[-2], 2)
    out = []
    for l in range(lc.shape[1], 0, -1):
        c, k = lc[:, l - 1, 0], lc[:, l - 1, 1]
        on = c > 0
        if not on.any():
            continue
        out.append({"level": l, "heads": int(on.sum()),
                    "candidates_mean": float(c[on].mean()), "candidates_p50": float(np.median(c[on])),
                    "candidates_max": int(c[on].max()),
                    "kept_mean": float(k[on].mean()), "kept_p50": float(np.median(k[on])),
                    "kept_max": int(k[on].max())})
    return out


FP64_TENSOR_TFLOPS = 40.0      # nominal dense fp64 tensor-core rate of a B200 (no measured figure here)


def paper_model(line: dict, peaks: dict) -> dict:
    """The pages' decode roofline model (arXiv 2610.42112 §V-A, App. D-B) with this GPU's
    constants, set against the measured stage times of one bench line of the zha path.

    Per stage x, Phi_x = max(FLOPs_x / P_x, bytes_x / BW, t_waves).  The worker-wave term
    needs a per-block latency tau_x; it is calibrated here as the measured time of the same
    kernel's launch at the highest level launched on its own when that level is above the
    leaves (its few candidates fit in one wave, so tau is the kernel's fixed latency and the
    wave count is taken as 1).  The fused launch of the small top levels is its own one-wave
    calibration.  A line whose only separately launched level is the leaf level has no
    one-wave launch of the score and select kernels: their wave term is then left out
    (t_waves = 0).  Counts follow App. D-B1
    with this implementation's element sizes:
      routing, level l:  FLOPs = 2 B Hq R d K_l (every head scores its own candidates, on the
                         fp64 tensor cores here); bytes = R (s d + 4) B Hkv K_l^grp + s d B Hq
                         (each node of a KV group's candidate union K_l^grp is read once;
                         without the union in the line, the largest per-head frontier, a
                         lower bound, stands in for it);
      scan, level l:     bytes = 12 B Hq K_l (an fp64 score and an int32 id per candidate,
                         one pass: the select keeps the scores in shared memory);
      attention:         FLOPs = 2 B Hq (d_k + d_v) K_0; bytes = the bench's gathered bytes
                         (K_0 union rows of K and V per KV group) + split partials (d_v + 2
                         fp32 values per head and split), i.e. bytes_attn,split;
      tree (decode):     amortised: one leaf summary per `leaf` appended tokens per unit,
                         64 d s read + R (d s + 4 d + 8) written (parents add 1/branch of it);
      launches:          lambda = step time minus the traced kernels' time, plus the
                         launches of levels above the top one (no visible node there).
    """
    cfg = line["config"]
    B, Hq, Hkv, d, R = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], cfg["R"]
    leaf = cfg.get("leaf", 64)
    s = 2 if line["dtype"] == "bf16" else 4
    bw = peaks["hbm_gbs"] * 1e9
    p16 = peaks["bf16_tflops"] * 1e12
    p64 = FP64_TENSOR_TFLOPS * 1e12
    st = line["stages_ms"]
    levels = line["frontier"]["levels"]               # top level first
    depth = cfg["depth"]
    top = levels[0]["level"]
    # one score and one select launch per level launched on its own, top level first (lines
    # that also timed the empty levels above the top start at level `depth`); the small top
    # levels may instead share one fused launch (route_fused), above the per-level ones
    per_s = st.get("route_score_per_launch") or ([st["route_score"]] if st.get("route_score") else [])
    per_x = st.get("route_select_per_launch") or ([st["route_select"]] if st.get("route_select") else [])
    n_sep = len(per_s)                                # levels n_sep .. 1 launched on their own
    first = depth if n_sep == depth else n_sep
    fused_ms = st.get("route_fused", 0.0) or 0.0
    score_ms = lambda l: per_s[first - l] if l <= first else None      # noqa: E731
    select_ms = lambda l: per_x[first - l] if l <= first else None     # noqa: E731
    sep_top = min(top, first)
    tau = {"score": score_ms(sep_top), "select": select_ms(sep_top)} if sep_top > 1 else {}

    def row(stage, kind, flops, byts, peak, unit, measured):
        t_f, t_b = 1e3 * flops / peak, 1e3 * byts / bw
        t_w = tau.get(kind, 0.0)
        model = max(t_f, t_b, t_w)
        bound = "latency (one wave)" if model == t_w and t_w > 0 else (unit if t_f > t_b else "hbm")
        return {"stage": stage, "flops": flops, "bytes": byts, "flops_ms": t_f, "bytes_ms": t_b,
                "waves_ms": t_w, "model_ms": model, "bound": bound, "measured_ms": measured}

    rows = []
    fused = []
    for f in levels:
        l = f["level"]
        k_head = f["candidates_mean"]
        k_grp = f.get("candidates_group_union", f["candidates_max"])
        r_s = row(f"route score L{l}", "score", 2.0 * B * Hq * R * d * k_head,
                  R * (s * d + 4) * B * Hkv * k_grp + s * d * B * Hq, p64, "fp64 tensor", score_ms(l))
        r_x = row(f"route select L{l}", "select", 0.0, 12.0 * B * Hq * k_head, p64, "alu", select_ms(l))
        if l > first:                                 # inside the fused launch
            fused += [r_s, r_x]
        else:
            rows += [r_s, r_x]
    if fused:
        rows.insert(0, {"stage": f"route fused L{top}..L{first + 1}", "flops": sum(r["flops"] for r in fused),
                        "bytes": sum(r["bytes"] for r in fused), "flops_ms": sum(r["flops_ms"] for r in fused),
                        "bytes_ms": sum(r["bytes_ms"] for r in fused), "waves_ms": fused_ms,
                        "model_ms": max(sum(r["flops_ms"] for r in fused), sum(r["bytes_ms"] for r in fused),
                                        fused_ms),
                        "bound": "latency (one wave)", "measured_ms": fused_ms})
    T1 = cfg["T"] + 1
    k0 = line["kv_touched"]["mean"] * T1
    byts = line["roofline"]["algorithmic_bytes_per_launch"] * line["roofline"]["launches_per_step"]
    rows.append(row("attention", "attention", 2.0 * B * Hq * 2 * d * k0, byts, p16, "bf16 tensor",
                    st["attention"]))
    leaf_bytes = leaf * d * s + R * (d * s + 4 * d + 8)
    byts = B * Hkv * leaf_bytes / leaf * (1 + 1 / max(1, cfg.get("branch", 16) - 1))
    rows.append(row("tree (amortised per step)", "tree", 4.0 * R * d * B * Hkv, byts, p64, "fp64 tensor",
                    line["tree_build"]["ms"] / cfg["T"]))
    # levels above the top one have no visible node: their score and select launches are
    # launch overhead only (the lambda_l of the model), with the gaps between kernels
    empty = 0.0
    for l in range(first, top, -1):
        if score_ms(l) is None:
            continue
        t = score_ms(l) + select_ms(l)
        empty += t
        rows.append({"stage": f"route L{l} (empty)", "flops": 0.0, "bytes": 0.0, "flops_ms": 0.0,
                     "bytes_ms": 0.0, "waves_ms": 0.0, "model_ms": 0.0, "bound": "launch only",
                     "measured_ms": t})
    kernels = sum(r["model_ms"] for r in rows)
    lam = max(0.0, st["step"] - st["stage_sum"]) + empty
    for r in rows:
        r["measured_over_model"] = r["measured_ms"] / r["model_ms"] if r["model_ms"] > 0 else None
    return {"workload": cfg["workload"], "rows": rows, "model_kernels_ms": kernels,
            "measured_step_ms": st["step"], "launch_gaps_ms": lam,
            "launches_per_step": line["gpu_launches"] / line["steps"],
            "model_step_ms": kernels + lam,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                      "fp64_tensor_tflops": FP64_TENSOR_TFLOPS}}


def candidate_unions(level_cnt: np.ndarray, level_ids: np.ndarray, n_cap: dict, nvis: dict, G: int,
                     branch: int) -> dict:
    """Per level, the mean over KV groups of the size of the group's candidate union (the
    nodes the score kernel reads once per group), from zha_route's level counts
    [B, nq, Hq, depth, 2] and kept ids [B, nq, Hq, sum_{l>=2} n_cap(l)] (one query per
    sequence).  At the top level every head's candidates are the visible nodes; below it,
    the children of the union of the heads' kept parents plus the orphans (visible nodes
    whose parent is not visible)."""
    B, _, Hq, depth, _ = level_cnt.shape
    offs, off = {}, 0
    for l in range(2, depth + 1):
        offs[l] = off
        off += n_cap[l]
    top = max((l for l in range(1, depth + 1) if nvis.get(l, 0) >= 1), default=0)
    out = {}
    for l in range(top, 0, -1):
        sizes = []
        for b in range(B):
            for g0 in range(0, Hq, G):
                if l == top:
                    sizes.append(nvis[top])
                    continue
                kept = set()
                for h in range(g0, g0 + G):
                    n = int(level_cnt[b, 0, h, l, 1])            # kept at level l + 1
                    kept.update(level_ids[b, 0, h, offs[l + 1]:offs[l + 1] + n].tolist())
                sizes.append(branch * len(kept) + nvis[l] - branch * nvis[l + 1])
        out[l] = float(np.mean(sizes))
    return out


class _Bf16Rows:
    """A [t_cap, d] bf16 array held as its raw 16-bit patterns, read row by row as float32
    (exact: a bf16 value is the upper half of the fp32 with the same value).  It gives the
    oracle's row readers (slices and index arrays) float values without a full fp32 copy."""

    def __init__(self, bits: np.ndarray):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, idx):
        return (np.asarray(self.bits[idx]).astype(np.uint32) << 16).view(np.float32)


def _oracle_worker(conn, spec):
    """One process of the CPU-oracle pool (spawned: it never touches CUDA).

    It attaches the shared K / V of sequence 0, builds the oracle's tree of every KV unit
    its heads belong to (untimed: the step's prior state), then on each "step" message
    routes and attends its query heads one at a time (zo.decode_head) until the step's
    CPU budget is spent, and answers with the heads done and the seconds taken.  A
    "check" message compares the GPU's leaf lists and outputs of its heads with the
    oracle's results of the last step."""
    from multiprocessing import shared_memory
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass
    from oracle import zha_oracle as zo
    shms = [shared_memory.SharedMemory(name=n) for n in (spec["k_name"], spec["v_name"])]
    dt = np.uint16 if spec["dtype"] == "bf16" else np.float32
    arrs = [np.ndarray(spec["shape"], dtype=dt, buffer=m.buf) for m in shms]
    rows = (lambda a: _Bf16Rows(a)) if spec["dtype"] == "bf16" else (lambda a: a)
    K = {hk: rows(arrs[0][hk]) for hk in spec["units"]}
    V = {hk: rows(arrs[1][hk]) for hk in spec["units"]}
    T, G = spec["T"], spec["G"]
    t0 = time.perf_counter()
    trees = {hk: zo.build_tree(K[hk], T + 1, spec["qref"][hk], spec["depth"], route_storage=spec["route_storage"],
                               inv_freq=spec["inv_freq"]) for hk in spec["units"]}
    conn.send(("ready", time.perf_counter() - t0))
    last = {}
    while True:
        msg = conn.recv()
        if msg[0] == "stop":
            break
        if msg[0] == "step":
            budget = msg[1]
            last = {}
            t0 = time.perf_counter()
            for h in spec["heads"]:
                r, o, _ = zo.decode_head(spec["q"][h], K[h // G], V[h // G], T, trees[h // G], spec["p"])
                last[h] = (r, o)
                if time.perf_counter() - t0 >= budget:
                    break
            conn.send(("done", len(last), time.perf_counter() - t0,
                       [[(min(s.margin, s.gap)) for s in r.sel.values()] for r, _ in last.values()]))
        if msg[0] == "check":
            gpu = msg[1]                                 # h -> (leaf ids, output row)
            out = []
            for h, (r, o) in last.items():
                leaves, og = gpu[h]
                near = any(min(s.margin, s.gap) < NEAR_CUTOFF for s in r.sel.values())
                same = np.array_equal(np.asarray(leaves, np.int64), r.leaves)
                if not same:                             # the oracle's attention over the GPU's list
                    o, _ = zo.attention(spec["q"][h], K[h // G], V[h // G], zo.index_set(leaves, T))
                out.append((h, same, near, float(np.abs(np.asarray(og, np.float64) - o).max())))
            conn.send(("checked", out))
    for m in shms:
        m.close()


class OraclePool:
    """The CPU oracle on the host cores: spawned worker processes, one BLAS thread each,
    over the query heads of sequence 0 of a workload (contiguous blocks of heads, so a
    worker builds the trees of one or two KV units).  The sample's K / V sit in shared
    memory; nothing is copied per step."""

    def __init__(self, w: S.Workload, p: float, K0, V0, q0, qref, inv_freq=None, workers: int = 0):
        """K0, V0: [Hkv, t_cap, d] of sequence 0 with the step's new token at position T;
        q0: [Hq, d] its queries; qref: [Hkv, R, d] (torch tensors on any device)."""
        import multiprocessing as mp
        from multiprocessing import shared_memory
        bf16 = w.dtype == "bf16"
        self.w, self.p = w, p
        self.shms = []
        names = []
        for X in (K0, V0):
            x = X.cpu()
            a = (x.view(torch.int16).numpy().view(np.uint16) if bf16 else x.numpy())
            m = shared_memory.SharedMemory(create=True, size=a.nbytes)
            np.ndarray(a.shape, dtype=a.dtype, buffer=m.buf)[...] = a
            self.shms.append(m)
            names.append(m.name)
            shape = a.shape
        cpus = os.cpu_count() or 1
        cap = max(1, int(32 * (1 << 20) // max(1, w.T)))      # bounds the trees held per unit
        self.n = workers or max(1, min(cpus, w.Hq, cap))
        self.cpus = cpus
        qc = q0.double().cpu().numpy()
        qr = qref.double().cpu().numpy()
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        per = [list(range(i * w.Hq // self.n, (i + 1) * w.Hq // self.n)) for i in range(self.n)]
        for heads in per:
            units = sorted({h // w.G for h in heads})
            spec = {"k_name": names[0], "v_name": names[1], "shape": shape, "dtype": w.dtype, "units": units,
                    "heads": heads, "q": {h: qc[h] for h in heads}, "qref": {u: qr[u] for u in units},
                    "T": w.T, "G": w.G, "depth": w.depth, "p": p,
                    "route_storage": "bf16" if bf16 else "f32", "inv_freq": inv_freq}
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_oracle_worker, args=(b, spec), daemon=True)
            pr.start()
            self.conns.append(a)
            self.procs.append(pr)
        self.build_s = max(c.recv()[1] for c in self.conns)

    @classmethod
    def from_workload(cls, w: S.Workload, p: float, device: str, inv_freq=None, workers: int = 0):
        """A pool over sequence 0 of the workload drawn afresh by the seeded generator."""
        one = S.scaled(w, T=w.T, B=1)
        C, K, V = S.clustered_kv(one, device)
        qref = S.reference_queries(one, device)
        kn, vn = S.new_tokens(one, C, 1, device)
        q = S.queries(one, C, 1, device)
        K[:, :, w.T] = kn[:, 0]
        V[:, :, w.T] = vn[:, 0]
        return cls(w, p, K[0], V[0], q[0, 0], qref, inv_freq=inv_freq, workers=workers)

    def step(self, budget: float):
        """One sampled step: every worker routes and attends its heads for at most `budget`
        seconds (at least one head each).  Returns (heads done, wall seconds, near flags)."""
        t0 = time.perf_counter()
        for c in self.conns:
            c.send(("step", budget))
        res = [c.recv() for c in self.conns]
        wall = time.perf_counter() - t0
        return sum(r[1] for r in res), wall, [m for r in res for m in r[3]]

    def check(self, leaves: dict, outputs: dict):
        """Compare the GPU's leaf lists and outputs (dicts over heads of sequence 0) with the
        oracle's results of the last step: a parity summary."""
        for c, pr_heads in zip(self.conns, self._heads()):
            c.send(("check", {h: (leaves[h], outputs[h]) for h in pr_heads}))
        rows = [x for c in self.conns for x in c.recv()[1]]
        return {"heads": len(rows), "exact": sum(1 for r in rows if r[1]),
                "near_cutoff_mismatch": sum(1 for r in rows if not r[1] and r[2]),
                "failed": sum(1 for r in rows if not r[1] and not r[2]),
                "max_abs_err": max((r[3] for r in rows), default=None),
                "rule": "leaf lists equal to the oracle's, or differing only for a head with a level whose "
                        f"cutoff margin or boundary gap is under {NEAR_CUTOFF}; the output against the oracle's "
                        "attention over the GPU's own list"}

    def _heads(self):
        w = self.w
        return [list(range(i * w.Hq // self.n, (i + 1) * w.Hq // self.n)) for i in range(self.n)]

    def close(self):
        for c in self.conns:
            try:
                c.send(("stop",))
            except Exception:  # noqa: BLE001
                pass
        for pr in self.procs:
            pr.join(timeout=30)
        for m in self.shms:
            m.close()
            m.unlink()


def oracle_sample(pool: OraclePool, seconds: float) -> dict:
    """Query-heads/s of the CPU oracle over one sampled step of the pool."""
    heads, wall, flags = pool.step(seconds)
    return {"value": heads / wall, "heads": heads, "wall_s": wall, "flags": flags}


def stage_breakdown(lib, step, stream, nb, ms_step):
    """Per-step GPU time of the traced kernels, from nb extra (untimed) steps whose
    score, select and attention launches are bracketed by CUDA events on their stream.
    With a chunked decode the routing of later chunks runs concurrently with attention,
    so the stage sum exceeds the step time by the overlap."""
    from hierarchical_sparse_attention_02_b200 import _lib
    kinds = {"route_fused": _lib.ZHA_TRACE_ROUTE_FUSED, "route_score": _lib.ZHA_TRACE_ROUTE_SCORE,
             "route_select": _lib.ZHA_TRACE_ROUTE_SELECT, "attention": _lib.ZHA_TRACE_ATTN}
    cap = nb * 64                     # <= 8 chunks x 8 levels per step
    ev = {}
    for name, kid in kinds.items():
        a = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
        b = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
        for e in a + b:
            e.record(stream)
        ev[name] = (a, b)
    torch.cuda.synchronize()
    keep = []
    for name, kid in kinds.items():
        a, b = ev[name]
        arr_s = (ctypes.c_void_p * cap)(*[ctypes.c_void_p(e.cuda_event) for e in a])
        arr_e = (ctypes.c_void_p * cap)(*[ctypes.c_void_p(e.cuda_event) for e in b])
        keep.append((arr_s, arr_e))
        lib.zha_trace(kid, arr_s, arr_e, cap)
    for _ in range(nb):
        step()
    torch.cuda.synchronize()
    out = {}
    for name, kid in kinds.items():
        n = lib.zha_trace_count(kid)
        lib.zha_trace(kid, None, None, 0)
        a, b = ev[name]
        t = [x.elapsed_time(y) for x, y in zip(a[:n], b[:n])]
        out[name] = sum(t) / nb
        per = n // nb                 # launches per step, in launch order (top level first)
        out[name + "_per_launch"] = [round(sum(t[j::per]) / nb, 4) for j in range(per)]
    out["stage_sum"] = sum(out[k] for k in kinds)
    out["step"] = ms_step
    out["steps"] = nb
    return out


def run_reference(args, w, p, ws, rank):
    """The reference arm: the CPU oracle as it stands, on the host cores (a pool of
    spawned worker processes, one BLAS thread each), on sampled steps of the workload:
    each step routes and attends the query heads of sequence 0 (at most `cpu_seconds`
    of CPU per worker).  value = query heads per second of that sample; ms_per_step is
    the measured wall time of one sampled step."""
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    per_step = max(0.5, 150.0 / max(1, K + W))
    freq = (10000.0 ** (-np.arange(args.rope, dtype=np.float64) / args.rope)).astype(np.float32).astype(
        np.float64) if args.rope else None
    pool = OraclePool.from_workload(w, p, dev, inv_freq=freq, workers=args.cpu_workers)
    try:
        rates = []
        for i in range(W + K):
            r = oracle_sample(pool, min(per_step, args.cpu_seconds))
            if i >= W:
                rates.append(r)
    finally:
        pool.close()
    value = statistics.median(r["value"] for r in rates)
    ms = 1e3 * statistics.median(r["wall_s"] for r in rates)
    heads = rates[0]["heads"]
    line = {
        "metric": "ZHA decode query-heads/s", "value": value, "unit": "query-heads/s", "n_gpus": 1,
        "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**config_of(w, p), **({"rope_pairs": args.rope} if args.rope else {})}, "impl": "reference",
        "step_sample": f"{heads} of the {w.B * w.Hq} query heads of a full step (sequence 0); "
                       "ms_per_step is the measured wall time of that sample",
        "cpu_baseline": {"value": value, "unit": "query-heads/s", "cores": pool.n, "host_cpus": pool.cpus,
                         "kind": "oracle",
                         "sample": f"{heads} query heads of sequence 0 per step, fp64 numpy, {pool.n} worker "
                                   f"processes x 1 thread (tree built untimed, {pool.build_s:.1f} s)"},
        "e2e": {"value": value, "unit": "query-heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, p):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "depth": w.depth,
            "leaf": w.leaf, "branch": w.branch, "R": w.R, "p": p, "n_centres": w.n_centres,
            "kv_bytes": 2 * w.B * w.Hkv * w.T * w.d * (2 if w.dtype == "bf16" else 4),
            "l2": "no flush: the KV cache read per step is larger than the 126 MB L2",
            **({"segment": w.segment, "generator": "structured variant: keys share a centre over runs "
                "of `segment` positions; queries take a segment's centre"} if w.segment else {})}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------


SWEEP_T = (16384, 32768, 65536, 131072, 262144, 524288, 1048576, 2097152)


def run_sweep(args):
    """Crossover sweep: ms per decode step of zha_decode at every depth L = 1..6, of the
    dense kernel and of the flat indexer, for T in SWEEP_T at the long-decode head geometry (B=4, Hq=32, Hkv=4),
    on the same seeded inputs per T (with --segment, the structured variant of the generator).
    One JSON line per (T, path, depth)."""
    import dataclasses
    import hierarchical_sparse_attention_02_b200 as Z
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    base = S.workload("long-decode-1m")
    p = args.p if args.p is not None else base.p[0]
    for T in SWEEP_T:
        w = S.scaled(base, T=T)
        if args.segment > 0:          # the structured variant of the generator
            w = dataclasses.replace(w, segment=args.segment)
        tag = {"segment": args.segment} if args.segment > 0 else {}
        C, K, V = S.clustered_kv(w, dev)
        qref = S.reference_queries(w, dev)
        k_new, v_new = S.new_tokens(w, C, 1, dev)
        q = S.queries(w, C, 1, dev)
        del C
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        O = torch.empty(w.B, 1, w.Hq, w.d, dtype=torch.bfloat16, device=dev)

        def timed(fn):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(args.steps):
                fn()
            b.record()
            torch.cuda.synchronize()
            if st.item() != 0:
                raise RuntimeError(f"device status {st.item()}")
            return a.elapsed_time(b) / args.steps

        best = None
        for L in range(1, 7):
            wl = dataclasses.replace(w, depth=L)
            g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=L, R=w.R)
            tree = Z.empty_tree(g, dev)
            Z.zha_build_tree(g, K, w.T, qref, tree, st)
            wsb = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE, dev)
            ids = torch.empty(w.B, 1, w.Hq, Z.leaf_cap(g), dtype=torch.int32, device=dev)
            cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=dev)
            ms = timed(lambda: Z.zha_decode(g, q, k_new, v_new, K, V, w.T, qref, p, tree, ids, cnt, O, wsb, st))
            touched = float((cnt.double() * 64 + 1).mean().item()) / (w.T + 1)
            print(json.dumps({"sweep": "crossover", "T": T, "path": "zha", "depth": L, "p": p,
                              "ms_per_step": ms, "kv_touched_approx": touched, **tag}), flush=True)
            best = min(best, ms) if best is not None else ms
            del tree, wsb, ids, cnt
        g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=1, R=w.R)
        wsd = Z.empty_workspace(g, 1, Z.ZHA_OP_DENSE, dev)
        pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=dev)
        ms_dense = timed(lambda: Z.zha_dense_decode(g, q, K, V, pos, O, wsd, st))
        print(json.dumps({"sweep": "crossover", "T": T, "path": "dense", "ms_per_step": ms_dense,
                          "zha_best_ms": best, "zha_faster": best < ms_dense, **tag}), flush=True)
        wsf = Z.empty_workspace(g, 1, Z.ZHA_OP_FLAT, dev)
        ids = torch.empty(w.B, 1, w.Hq, Z.leaf_cap(g), dtype=torch.int32, device=dev)
        cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=dev)
        ms_flat = timed(lambda: Z.zha_flat_index(g, q, K, V, pos, p, ids, cnt, O, wsf, st))
        touched = float((cnt.double() * 64 + 1).mean().item()) / (w.T + 1)
        print(json.dumps({"sweep": "crossover", "T": T, "path": "flat", "ms_per_step": ms_flat,
                          "kv_touched_approx": touched, **tag}), flush=True)
        del K, V, wsd, wsf, ids, cnt
        torch.cuda.empty_cache()


def tile_unions(ids: np.ndarray, cnt: np.ndarray, pos: np.ndarray, Hkv: int, G: int) -> np.ndarray:
    """Chunks each query tile gathers: the union over its Qt = 128 // G queries x G heads
    of their leaf lists, plus chunk 0 and every query's own chunk (the tiles of
    zha_prefill_attn).  ids [B, nq, Hq, cap], cnt [B, nq, Hq], pos [B, nq].  Returns the
    entry count of every tile, in (sequence, KV head, tile) order."""
    B, nq, Hq, _ = ids.shape
    qt = 128 // G
    out = []
    for b in range(B):
        for hk in range(Hkv):
            for q0 in range(0, nq, qt):
                qs = range(q0, min(nq, q0 + qt))
                parts = [np.array([0]), np.asarray(pos[b, list(qs)]) // 64]
                for qi in qs:
                    for h in range(hk * G, (hk + 1) * G):
                        parts.append(ids[b, qi, h, :cnt[b, qi, h]])
                out.append(len(np.unique(np.concatenate(parts))))
    return np.asarray(out, np.int64)


def run_prefill(args):
    """Chunked-prefill attention: the workload's n_new appended causal queries, routed once
    (untimed), then attended by the query-tile tensor-core path (zha_prefill_attn, timed
    over --steps calls) and by the per-query gather path (zha_sparse_attn) on the same
    leaf lists.  One JSON line; the roofline is the tile kernel's tensor-pipe rate."""
    import hierarchical_sparse_attention_02_b200 as Z
    from hierarchical_sparse_attention_02_b200 import _lib
    Z.load_library()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = S.workload("prefill-append-256k")
    if args.batch is not None or args.n_new is not None:
        w = S.scaled(w, T=w.T, B=args.batch, n_new=args.n_new)
    p = args.p if args.p is not None else w.p[0]
    g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=w.depth, R=w.R)
    C, K, V = S.clustered_kv(w, dev)
    qref = S.reference_queries(w, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tree = Z.empty_tree(g, dev)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    kn, vn = S.new_tokens(w, C, w.n_new, dev)
    Z.zha_append(g, K, V, kn, vn, w.T, qref, tree, st)
    Q = S.queries(w, C, w.n_new, dev)
    del C
    nq = w.n_new
    pos = (w.T + torch.arange(nq, device=dev, dtype=torch.int64)).view(1, -1).repeat(w.B, 1).contiguous()
    ids = torch.empty(w.B, nq, w.Hq, Z.leaf_cap(g), dtype=torch.int32, device=dev)
    cnt = torch.empty(w.B, nq, w.Hq, dtype=torch.int32, device=dev)
    wr = Z.empty_workspace(g, nq, Z.ZHA_OP_ROUTE, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Z.zha_route(g, Q, pos, p, tree, ids, cnt, wr, st)
    torch.cuda.synchronize()
    e0.record(); Z.zha_route(g, Q, pos, p, tree, ids, cnt, wr, st); e1.record()
    torch.cuda.synchronize()
    route_ms = e0.elapsed_time(e1)
    del wr
    O1 = torch.empty(w.B, nq, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
    O2 = torch.empty_like(O1)
    wp = Z.empty_workspace(g, nq, Z.ZHA_OP_PREFILL, dev)
    wa = Z.empty_workspace(g, nq, Z.ZHA_OP_ATTN, dev)
    lib = _lib.load()

    def timed(fn, steps, warm):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        n_ev = steps
        a = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
        b = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
        for x in a + b:
            x.record()
        torch.cuda.synchronize()
        arr_s = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(x.cuda_event) for x in a])
        arr_e = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(x.cuda_event) for x in b])
        lib.zha_trace(_lib.ZHA_TRACE_ATTN, arr_s, arr_e, n_ev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            fn()
        t1.record()
        torch.cuda.synchronize()
        k = lib.zha_trace_count(_lib.ZHA_TRACE_ATTN)
        lib.zha_trace(_lib.ZHA_TRACE_ATTN, None, None, 0)
        if st.item() != 0:
            raise RuntimeError(f"device status {st.item()}")
        kern = sum(x.elapsed_time(y) for x, y in zip(a[:k], b[:k])) / max(1, k)
        return t0.elapsed_time(t1) / steps, kern

    clocks = ClockSampler(0)
    time.sleep(0.3)
    clocks.mark_start()
    tile_ms, tile_kern = timed(lambda: Z.zha_prefill_attn(g, Q, K, V, pos, ids, cnt, O2, wp, st),
                               args.steps, args.warmup)
    clocks.mark_end()
    clk = clocks.stop()
    q_ms, q_kern = timed(lambda: Z.zha_sparse_attn(g, Q, K, V, pos, ids, cnt, O1, wa, st),
                         max(1, min(args.steps, 3)), 1)
    diff = (O1.float() - O2.float()).abs()
    ent = tile_unions(ids.cpu().numpy(), cnt.cpu().numpy(), pos.cpu().numpy(), w.Hkv, w.G)
    flops_exec = float(ent.sum()) * 4.0 * 128 * 64 * 128          # S and P.V on 128 rows per chunk
    kept = cnt.cpu().numpy().astype(np.float64)
    useful = float((kept * 64).sum() + w.B * nq * w.Hq) * 4.0 * 128   # rows x their own keys (approx.)
    peaks = {"bf16_tflops": 1590.0, "kind": "fallback"}
    try:
        mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        peaks = {"bf16_tflops": float(mp["bf16_tflops"]), "kind": "measured (burst)"}
    except (OSError, ValueError, KeyError):
        pass
    achieved = flops_exec / (tile_kern * 1e-3) / 1e12
    qh = w.B * nq * w.Hq
    line = {
        "metric": "ZHA prefill attention query-heads/s", "value": qh / (tile_ms * 1e-3), "unit": "query-heads/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": tile_ms, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {**config_of(w, p), "path": "prefill", "n_new": nq, "tile_queries": 128 // w.G},
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_kind": peaks["kind"], "flops_per_launch": flops_exec, "kernel_ms": tile_kern,
                     "useful_flops_fraction": useful / flops_exec},
        "tiles": {"count": int(len(ent)), "entries_mean": float(ent.mean()), "entries_max": int(ent.max()),
                  "kv_bytes_per_launch": float(ent.sum()) * 2 * 64 * 128 * 2},
        "per_query_path": {"ms": q_ms, "kernel_ms": q_kern, "speedup_of_tiles": q_ms / tile_ms},
        "route_ms": route_ms,
        "max_abs_diff_vs_per_query_path": float(diff.max().item()),
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.model:
        peaks = {"hbm_gbs": hbm_peak()[0], "bf16_tflops": 1590.0}
        try:
            peaks["bf16_tflops"] = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"]
        except (OSError, ValueError, KeyError):
            pass
        for raw in open(args.model):
            raw = raw.strip()
            if raw.startswith("{") and '"frontier"' in raw and '"path": "zha"' in raw:
                print(json.dumps(paper_model(json.loads(raw), peaks)), flush=True)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.path == "prefill":
        run_prefill(args)
        return
    w = S.workload(args.workload)
    if args.batch is not None:
        w = S.scaled(w, T=w.T, B=args.batch)
    if args.segment > 0:
        import dataclasses
        w = dataclasses.replace(w, segment=args.segment, name=f"{w.name}+seg{args.segment}")
    p = args.p if args.p is not None else w.p[0]
    ws, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, w, p, ws, rank)
        barrier(ws)
        return

    import hierarchical_sparse_attention_02_b200 as Z
    from hierarchical_sparse_attention_02_b200 import _lib
    Z.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    wr = S.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank}) if rank else w
    g = Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=w.depth, R=w.R, d=w.d,
                   dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32, rope_pairs=args.rope)
    C, K, V = S.clustered_kv(wr, dev)
    qref = S.reference_queries(wr, dev)
    qref_plain = qref
    freq = None
    if args.rope:                     # the tree calls read the frequencies after the references
        freq = (10000.0 ** (-torch.arange(args.rope, dtype=torch.float64) / args.rope)).float()
        qref = Z.reference_block(qref, freq)
    k_new, v_new = S.new_tokens(wr, C, 1, dev)
    q = S.queries(wr, C, 1, dev)
    del C
    tree = Z.empty_tree(g, dev)
    wsb = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    cap = Z.leaf_cap(g)
    ids = torch.empty(w.B, 1, w.Hq, cap, dtype=torch.int32, device=dev)
    cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=dev)
    O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=dev)
    stream = torch.cuda.current_stream()

    # tree build (prefill of the summaries), timed once
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)          # warm
    torch.cuda.synchronize()
    e0.record(); Z.zha_build_tree(g, K, w.T, qref, tree, st); e1.record()
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)
    k_bytes = w.B * w.Hkv * w.T * w.d * (2 if w.dtype == "bf16" else 4)

    if args.path == "zha":
        def step():
            Z.zha_decode(g, q, k_new, v_new, K, V, w.T, qref, p, tree, ids, cnt, O, wsb, st)
    else:
        # baselines attend from the same position over the same cache (new token appended once)
        Z.zha_append(g, K, V, k_new, v_new, w.T, qref, tree, st)
        qpos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=dev)
        op = Z.ZHA_OP_DENSE if args.path == "dense" else Z.ZHA_OP_FLAT
        wsb = Z.empty_workspace(g, 1, op, dev)
        if args.path == "dense":
            def step():
                Z.zha_dense_decode(g, q, K, V, qpos, O, wsb, st)
        else:
            def step():
                Z.zha_flat_index(g, q, K, V, qpos, p, ids, cnt, O, wsb, st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if st.item() != 0:
        raise RuntimeError(f"device status {st.item()} after warm-up")

    Ksteps = args.steps
    n_ev = Ksteps * 8                 # a decode step launches the attention once per chunk (<= 8)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in starts + stops:          # torch creates the CUDA event at its first record
        e.record(stream)
    torch.cuda.synchronize()
    arr_s = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(e.cuda_event) for e in starts])
    arr_e = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(e.cuda_event) for e in stops])
    lib = _lib.load()
    clocks = ClockSampler(torch.cuda.current_device())
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    # the dominant kernel is traced live: the attention, or the chunk scores of the flat path
    dom = _lib.ZHA_TRACE_ROUTE_SCORE if args.path == "flat" and w.dtype == "bf16" else _lib.ZHA_TRACE_ATTN
    graph = None
    if args.graph:
        # the whole step captured once; the timed loop replays it (no host launches)
        graph = torch.cuda.CUDAGraph()
        n_g0 = Z.launch_count()
        with torch.cuda.graph(graph):
            step()
        graph_launches = Z.launch_count() - n_g0
        graph.replay()
        torch.cuda.synchronize()
    else:
        lib.zha_trace(dom, arr_s, arr_e, n_ev)
    n_launch0 = Z.launch_count()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    t_start.record(stream)
    for _ in range(Ksteps):
        if graph is not None:
            graph.replay()
        else:
            step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(ws)
    if graph is None:
        launches = Z.launch_count() - n_launch0
        traced = lib.zha_trace_count(dom)
        lib.zha_trace(dom, None, None, 0)
    ms_local = t_start.elapsed_time(t_end) / Ksteps
    if graph is None:
        dom_launches = traced / Ksteps                     # launches of the traced kernel per step
        dom_ms = sum(a.elapsed_time(b) for a, b in zip(starts[:traced], stops[:traced])) / max(1, traced)
    if st.item() != 0:
        raise RuntimeError(f"device status {st.item()} in the timed region")
    ms, value = whole_job_rate(w.B * w.Hq, ms_local, ws)
    stages = stage_breakdown(lib, step, stream, min(Ksteps, 20), ms_local)
    if graph is not None:
        # replays launch what the capture launched; the dominant kernel is timed on the
        # traced (uncaptured) steps of the stage breakdown
        launches = graph_launches * Ksteps
        dom_name_stage = "route_score" if dom == _lib.ZHA_TRACE_ROUTE_SCORE else "attention"
        per = stages.get(dom_name_stage + "_per_launch")
        dom_launches = float(len(per)) if per else 1.0
        dom_ms = stages[dom_name_stage] / dom_launches

    # end to end through the public API with host buffers
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
    hq, hk, hv, hO = pin(q), pin(k_new), pin(v_new), pin(O)
    hq.copy_(q); hk.copy_(k_new); hv.copy_(v_new)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new)

    def e2e_step():
        dq.copy_(hq, non_blocking=True); dk.copy_(hk, non_blocking=True); dv.copy_(hv, non_blocking=True)
        if args.path == "zha":
            Z.zha_decode(g, dq, dk, dv, K, V, w.T, qref, p, tree, ids, cnt, O, wsb, st)
        elif args.path == "dense":
            Z.zha_dense_decode(g, dq, K, V, qpos, O, wsb, st)
        else:
            Z.zha_flat_index(g, dq, K, V, qpos, p, ids, cnt, O, wsb, st)
        hO.copy_(O, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(Ksteps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / Ksteps, ws)
    barrier(ws)
    clk = clocks.stop()

    # workload statistics (untimed): index-set sizes, KV-group unions, frontiers
    es = 2 if w.dtype == "bf16" else 4
    T1 = w.T + 1
    vstart = (w.T // 64) * 64
    partial = w.T - vstart + 1
    ids_c, cnt_c = ids.cpu().numpy(), cnt.cpu().numpy()
    nvis = vstart // 64
    units = w.B * w.Hkv
    c1 = w.t_cap // 64
    cps = max(16, -(-units * (c1 + 2) // 4096))                     # the library's split size
    krange = 1024                                                     # chunk ids per union block
    per_head, union_rows, items = [], 0, 0
    for bb in range(w.B):
        for hkv in range(w.Hkv):
            if args.path == "dense":
                lists = [np.arange(nvis)] * w.G
            else:
                lists = [ids_c[bb, 0, h, :cnt_c[bb, 0, h]] for h in range(hkv * w.G, (hkv + 1) * w.G)]
            for lst in lists:
                has0 = len(lst) and lst[0] == 0
                per_head.append((len(lst) * 64 + (0 if has0 or nvis == 0 else 1) + partial) / T1)
            u = np.unique(np.concatenate(lists)) if lists else np.zeros(0, np.int64)
            sink = any(not (len(l) and l[0] == 0) for l in lists) and nvis >= 1
            union_rows += len(u) * 64 + (1 if sink else 0) + partial
            # work items: per block of `krange` ids, ceil(entries / cps)
            per_block = np.bincount(u // krange, minlength=nvis // krange + 1) if len(u) else np.zeros(1, np.int64)
            per_block = per_block.astype(np.int64)
            per_block[0] += 1 if sink else 0
            per_block = np.concatenate([per_block, np.zeros(nvis // krange + 1, np.int64)])
            per_block[nvis // krange] += 1                            # the query's own chunk
            items += int(np.sum(-(-per_block // cps)))
    gathered = union_rows * 2 * w.d * es
    partial_bytes = items * w.G * (w.d + 2) * 4          # o[d], m, l written per head and split
    attn_bytes = gathered + partial_bytes
    # flat path: every visible chunk's keys read once, a score and an id written per head
    flat_bytes = units * nvis * 64 * w.d * es + w.B * w.Hq * nvis * 12 if args.path == "flat" else 0
    peak, peak_kind = hbm_peak()
    if dom == _lib.ZHA_TRACE_ATTN:
        dom_name = "attn_tc_kernel" if w.dtype == "bf16" else "attn_split_kernel"
        per_launch = attn_bytes / max(1.0, dom_launches)
    else:
        dom_name = "flat_tc_kernel"
        per_launch = flat_bytes / max(1.0, dom_launches)
    achieved = per_launch / (dom_ms * 1e-3) / 1e9
    # per-level frontier sizes: one more (untimed) routing of the step's queries with the
    # level counts switched on; its leaf lists must equal the decode step's
    frontier = None
    if args.path == "zha":
        try:
            lcnt = torch.zeros(w.B, 1, w.Hq, w.depth, 2, dtype=torch.int32, device=dev)
            n_cap = {l: Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1)}
            lids = torch.zeros(w.B, 1, w.Hq, max(1, sum(n_cap.values())), dtype=torch.int32, device=dev)
            ids2, cnt2 = torch.empty_like(ids), torch.empty_like(cnt)
            qpos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=dev)
            Z.zha_route(g, q, qpos, p, tree, ids2, cnt2, wsb, st, lcnt, lids)
            torch.cuda.synchronize()
            lc_np = lcnt.cpu().numpy()
            nvis = {l: (64 * (w.T // 64)) // (64 * w.branch ** (l - 1)) for l in range(1, w.depth + 1)}
            unions = candidate_unions(lc_np, lids.cpu().numpy(), n_cap, nvis, w.G, w.branch)
            ids2_c, cnt2_c = ids2.cpu().numpy(), cnt2.cpu().numpy()
            same = bool(np.array_equal(cnt2_c, cnt_c)) and all(
                np.array_equal(ids2_c[bb, 0, h, :cnt_c[bb, 0, h]], ids_c[bb, 0, h, :cnt_c[bb, 0, h]])
                for bb in range(w.B) for h in range(w.Hq))
            levels = frontier_stats(lc_np)
            for f in levels:
                f["candidates_group_union"] = unions.get(f["level"])
            frontier = {"levels": levels, "route_matches_decode": same}
            del lcnt, lids, ids2, cnt2
        except Exception as e:   # statistics outside the timed region: report, do not hide
            frontier = {"error": repr(e)}
    cpu = None
    near = None
    parity = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # the decode step's own inputs of sequence 0 (the cache holds the new token at T)
        pool = OraclePool(w, p, K[0], V[0], q[0, 0], qref_plain,
                          inv_freq=freq.double().numpy() if freq is not None else None, workers=args.cpu_workers)
        try:
            r = oracle_sample(pool, args.cpu_seconds)
            cpu = {"value": r["value"], "unit": "query-heads/s", "cores": pool.n, "host_cpus": pool.cpus,
                   "kind": "oracle",
                   "sample": f"{r['heads']} query heads of sequence 0 of {w.name}, route + attention, fp64 "
                             f"numpy, {pool.n} worker processes x 1 thread, {r['wall_s']:.1f} s wall "
                             f"(trees built untimed, {pool.build_s:.1f} s)"}
            if args.path == "zha":
                near = {**near_cutoff_from_flags(r["flags"]), "sample": "the oracle's routes of the cpu_baseline sample"}
                Oc = O.float().cpu().numpy()
                leaves = {h: ids_c[0, 0, h, :cnt_c[0, 0, h]] for h in range(w.Hq)}
                outs = {h: Oc[0, 0, h] for h in range(w.Hq)}
                parity = {**pool.check(leaves, outs), "sample": "the heads of the cpu_baseline sample, "
                          "against the decode step's leaf lists and outputs"}
        finally:
            pool.close()
    line = {
        "metric": "ZHA decode query-heads/s", "value": value, "unit": "query-heads/s", "n_gpus": ws,
        "steps": Ksteps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {**config_of(w, p), "path": args.path, **({"rope_pairs": args.rope} if args.rope else {}),
                   **({"cuda_graph": True} if args.graph else {})},
        "roofline": {"bound": "hbm", "kernel": dom_name,
                     "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": (profiled_traffic(w, units / max(1.0, dom_launches))
                                 if args.path == "zha" and w.dtype == "bf16" else None),
                     "algorithmic_bytes_per_launch": per_launch, "kernel_ms": dom_ms,
                     "launches_per_step": dom_launches},
        "step_hbm_gbs": (attn_bytes + flat_bytes) / (ms * 1e-3) / 1e9,
        "kv_touched": {"mean": float(np.mean(per_head)), "p50": float(np.median(per_head)),
                       "p99": float(np.percentile(per_head, 99)),
                       "group_union": union_rows / (units * T1)},
        "stages_ms": stages,
        "frontier": frontier,
        "near_cutoff": near,
        "parity": parity,
        "tree_build": {"ms": build_ms, "gbs": k_bytes / (build_ms * 1e-3) / 1e9},
        "e2e": {"value": ws * w.B * w.Hq / (e2e_ms * 1e-3), "unit": "query-heads/s",
                "h2d_bytes_per_step": (q.numel() + k_new.numel() + v_new.numel()) * es,
                "d2h_bytes_per_step": O.numel() * es},
        "gpu_launches": launches,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
