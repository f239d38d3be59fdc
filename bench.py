"""Benchmark of the hybrid-attention forward on B200 (one process per GPU).

`python bench.py --gpus N --steps K --warmup W` times K steps of one workload (default: the CSA
prefill at 128k tokens, bf16) and rank 0 prints one JSON line. A step is one csa_forward call: the
compressor over kv and over the indexer key stream, the indexer score, top-k, and the sparse +
sliding attention with the sink and both RoPE rotations. With N > 1 (torchrun, NCCL) every rank
runs its own sequence (data parallel, no collective on the data path; weak scaling) and the time
is the maximum over ranks. `--impl reference` times the fp64 CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_attention_compressor_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FP32_LANES_PER_SM = 128
N_SM = 148


# ------------------------------------------------------------------------------------------------
# algorithmic work (only the causal, visible work)
# ------------------------------------------------------------------------------------------------
DATA = "synthetic (seeded generators; the shapes and distributions of the workload)"


def visible(wl, S=None):
    S = wl.S if S is None else S
    t = np.arange(S, dtype=np.int64)
    nwin = np.minimum(t + 1, wl.W)
    nvis = (t + 1) // wl.m if wl.m else np.zeros_like(t)
    return nwin, nvis


def work(wl) -> dict:
    """Per-step algorithmic FLOPs / bytes of each kernel (summed over B sequences)."""
    nwin, nvis = visible(wl)
    esz = 4 if wl.dtype == "f32" else 2
    out = {}
    if wl.kind == "csa":
        nsel = np.minimum(nvis, wl.k)
        out["attention"] = ("flops", float((nwin + nsel).sum()) * 4 * wl.H * wl.D * wl.B)
        out["indexer_score"] = ("flops", float(nvis.sum()) * 2 * wl.nI * wl.cI * wl.B)
        out["topk"] = ("bytes", float(nvis.sum() * 4 + wl.S * wl.k * 4) * wl.B)
        out["compress_index"] = ("bytes", float(wl.S * wl.cI + wl.N * wl.cI) * esz * wl.B)
    elif wl.kind == "hca":
        out["attention"] = ("flops", float((nwin + nvis).sum()) * 4 * wl.H * wl.D * wl.B)
    else:
        out["attention"] = ("flops", float(nwin.sum()) * 4 * wl.H * wl.D * wl.B)
    if wl.kind in ("csa", "hca"):
        out["compress"] = ("bytes", float(wl.S * wl.D + wl.N * wl.D) * esz * wl.B)
    out["rotate_kv"] = ("bytes", float(2 * wl.S * wl.D) * esz * wl.B)
    return out


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def wait_samples(self, n: int, keep_busy, limit_s: float = 5.0):
        """Keep the GPU busy with keep_busy() (untimed) until n samples have been read, so that
        a timed region shorter than the sampling period still has samples taken under the same
        load right before and after it."""
        t0 = time.time()
        while self.proc is not None and len(self.lines) < n and time.time() - t0 < limit_s:
            keep_busy()
            torch.cuda.synchronize()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "200 ms samples while step replays run back to back, the timed "
                          "region included"}


# ------------------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def rank_workload(wl: W.Workload, rank: int) -> W.Workload:
    """Data-parallel replica: every rank runs the same shapes on its own seeded sequence."""
    from dataclasses import replace
    return replace(wl, seed=wl.seed + 1000 * rank)


def max_over_ranks(x: float, device=None) -> float:
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def make_step(wl, g, dev):
    import sparse_attention_compressor_b200 as sac
    p = sac.make_params(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                        sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                        dtype=wl.dtype)
    kind = {"swa": sac.SAC_KIND_SWA, "hca": sac.SAC_KIND_HCA, "csa": sac.SAC_KIND_CSA}[wl.kind]
    ws = torch.empty(sac.sac_workspace_size(p, kind), dtype=torch.uint8, device=dev)
    o = torch.empty_like(g["q"])

    def step():
        if wl.kind == "csa":
            sac.csa_forward(p, g["q"], g["kv"], g["cmp_gate"], g["cmp_bias"], g["q_idx"],
                            g["w_idx"], g["k_idx"], g["idx_gate"], g["idx_bias"], g["sinks"], o,
                            None, None, None, ws)
        elif wl.kind == "hca":
            sac.hca_forward(p, g["q"], g["kv"], g["cmp_gate"], g["cmp_bias"], g["sinks"], o, None,
                            ws)
        else:
            sac.swa_forward(p, g["q"], g["kv"], g["sinks"], o, ws)
    return step, o


def capture(fn):
    """fn (which has already run eagerly) captured once into a CUDA graph; a step is then one
    replay, so the timed region holds no host launch gaps."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    return g


def kernel_times(fn, dev, flush: bool = False) -> dict:
    """Per-kernel device times of one step: fn captured into a second graph with the library's
    timing events around every launch and replayed once (the timed graph carries no events);
    with flush, L2 is flushed before that replay as timed_flushed() does before every step."""
    import sparse_attention_compressor_b200 as sac
    sac.sac_timing_begin()
    g = capture(fn)
    if flush:
        torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev).fill_(0)
        torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev).sum()
    g.replay()
    torch.cuda.synchronize(dev)
    out = sac.sac_timing_end()
    del g
    return out


def timed(step, steps, dev):
    barrier(dev)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize(dev)
    barrier(dev)
    return a.elapsed_time(b)


def timed_flushed(step, steps, dev):
    """Like timed(), but L2 is flushed before every step: a write of twice its size, then a read
    of another buffer of that size, so that the dirty lines of the write are evicted before the
    step starts (their write-back would otherwise be charged to the step). Each step is bracketed
    by its own events and only the steps are summed."""
    junk = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    junk_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    for a, b in evs:
        junk.fill_(0)
        junk_r.sum()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize(dev)
    barrier(dev)
    return sum(a.elapsed_time(b) for a, b in evs)


def tensor_kernels(wl) -> set:
    """Kernels that run on tcgen05 for this workload (bf16 layers with 64 heads of 512; the
    indexer with 64 heads of 128); the rest run on CUDA cores."""
    out = set()
    if wl.dtype == "bf16" and wl.H == 64 and wl.D == 512 and wl.R <= 64:
        out.add("attention")
    if wl.kind == "csa" and wl.dtype == "bf16" and wl.nI == 64 and wl.cI == 128:
        out.add("indexer_score")
    return out


# DRAM bytes (read + write) per launch of a kernel come from one ncu capture, recorded in
# profiles/ncu_traffic.json with the SHA-256 of the kernel's sources at capture time. A record
# whose sources have changed since is stale and the roofline reports traffic null.
CSRC = os.path.join(ROOT, "sparse_attention_compressor_b200", "csrc")
KERNEL_SOURCES = {
    "attention": ["attention_tc.cu", "tc_ptx.cuh", "sac_common.cuh"],
    "csa_decode_attention": ["attention_tc.cu", "tc_ptx.cuh", "sac_common.cuh"],
    "hca_decode_attention": ["attention_tc.cu", "tc_ptx.cuh", "sac_common.cuh"],
    # the prefill indexer; decode and chunked prefill run indexer_decode_tc.cu (below)
    "indexer_score": ["indexer_tc.cu", "tc_ptx.cuh", "sac_common.cuh"],
    "topk": ["topk.cu", "sac_common.cuh"],
    "compress": ["compress.cu", "pool_window.cuh", "tc_ptx.cuh", "sac_common.cuh"],
    "compress_index": ["compress.cu", "pool_window.cuh", "tc_ptx.cuh", "sac_common.cuh"],
    "rotate_kv": ["compress.cu", "pool_window.cuh", "tc_ptx.cuh", "sac_common.cuh"],
    "decode_append": ["decode_append.cu", "pool_window.cuh", "sac_common.cuh"],
    "o_proj": ["oproj.cu", "tc_ptx.cuh"],
}
# kernels whose source differs for the paged (decode / chunked-prefill) workloads
PAGED_SOURCES = {
    "indexer_score": ["indexer_decode_tc.cu", "tc_ptx.cuh", "sac_common.cuh"],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def source_hash(kernel: str, workload: str = "") -> str:
    import hashlib
    h = hashlib.sha256()
    paged = workload in W.WORKLOADS and W.WORKLOADS[workload].kind == "decode"
    files = PAGED_SOURCES.get(kernel) if paged and kernel in PAGED_SOURCES else \
        KERNEL_SOURCES.get(kernel, [])
    for f in files:
        path = os.path.join(CSRC, f)
        if os.path.exists(path):
            with open(path, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(workload: str, kernel: str):
    """(bytes per launch, record) of a current ncu record of the kernel on this workload, or
    (None, None) when there is none or its sources changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    with open(TRAFFIC_FILE) as f:
        recs = json.load(f)
    for r in recs:
        if r["workload"] == workload and r["kernel"] == kernel and \
                r["source_sha256"] == source_hash(kernel, workload):
            return float(r["dram_bytes_per_launch"]), r
    return None, None


def record_traffic(raw_csv: str, workload: str, kernel: str, name_regex: str, summary: str,
                   scale: float = 1.0, scaled_from: str = "") -> dict:
    """Add (or replace) the ncu traffic record of one kernel on one workload.

    raw_csv is `ncu -i <report> --page raw --csv` of a capture of that kernel; the record keeps
    the mean dram__bytes_read.sum + dram__bytes_write.sum over the captured launches whose name
    matches name_regex, times `scale` when the capture ran a smaller case than the workload (the
    ratio of units processed, stated in scaled_from), with the SHA-256 of the kernel's sources."""
    import csv
    import re
    to_bytes = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    with open(raw_csv) as f:
        rows = [r for r in csv.reader(f)]
    # ncu prints its own log lines before the table: the header row names the kernel column
    start = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    head = rows[start]
    ik = head.index("Kernel Name")
    per = []
    if "Metric Name" in head:
        # `--metrics ... --csv` launch list: one row per (launch ID, metric)
        iid, im = head.index("ID"), head.index("Metric Name")
        iu, iv = head.index("Metric Unit"), head.index("Metric Value")
        by_launch = {}
        for r in rows[start + 1:]:
            if len(r) != len(head) or not re.search(name_regex, r[ik]):
                continue
            if r[im] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
                by_launch.setdefault(r[iid], 0.0)
                by_launch[r[iid]] += float(r[iv].replace(",", "")) * to_bytes[r[iu]]
        per = list(by_launch.values())
    else:
        # raw page: one row per launch, one column per metric, units in the second row
        units, data = rows[start + 1], rows[start + 2:]
        for r in data:
            if len(r) != len(head) or not re.search(name_regex, r[ik]):
                continue
            tot = 0.0
            for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
                i = head.index(m)
                tot += float(r[i].replace(",", "")) * to_bytes[units[i]]
            per.append(tot)
    if not per:
        raise SystemExit(f"no launch of {name_regex!r} in {raw_csv}")
    rec = {"workload": workload, "kernel": kernel,
           "dram_bytes_per_launch": sum(per) / len(per) * scale,
           "launches_captured": len(per), "source_sha256": source_hash(kernel, workload),
           "summary": summary}
    if scaled_from:
        rec["scaled_from"] = scaled_from
    recs = []
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            recs = [r for r in json.load(f)
                    if not (r["workload"] == workload and r["kernel"] == kernel)]
    recs.append(rec)
    recs.sort(key=lambda r: (r["workload"], r["kernel"]))
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(recs, f, indent=1)
        f.write("\n")
    return rec


def roofline(wl, ktimes: dict, peaks: dict, steps: int, tensor_kernels: set) -> tuple:
    wk = work(wl)
    total = sum(v[1] for v in ktimes.values()) or 1.0
    rows = {}
    for name, (launches, ms) in ktimes.items():
        per_launch_ms = ms / max(launches, 1)
        launches_per_step = launches / steps
        entry = {"launches": launches, "ms_per_launch": per_launch_ms, "share": ms / total}
        if name in wk:
            kind, amount = wk[name]
            amount /= launches_per_step  # per launch
            if kind == "flops":
                achieved = amount / (per_launch_ms * 1e-3) / 1e12
                if name in tensor_kernels:
                    bound, peak = "tensor", peaks["bf16_tflops"]
                else:
                    bound = "alu"
                    peak = N_SM * FP32_LANES_PER_SM * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
                entry.update(bound=bound, achieved=achieved, peak=peak, unit="TFLOP/s",
                             frac=achieved / peak)
            else:
                achieved = amount / (per_launch_ms * 1e-3) / 1e9
                entry.update(bound="hbm", achieved=achieved, peak=peaks["hbm_gbs"], unit="GB/s",
                             frac=achieved / peaks["hbm_gbs"])
        rows[name] = entry
    dom = max(ktimes, key=lambda k: ktimes[k][1])
    return roof_of(wl.name, dom, rows[dom], peaks), rows


def roof_of(workload: str, kernel: str, d: dict, peaks: dict) -> dict:
    traffic, rec = ncu_traffic(workload, kernel)
    roof = {"kernel": kernel, "bound": d.get("bound"), "achieved": d.get("achieved"),
            "peak": d.get("peak"), "unit": d.get("unit"), "frac": d.get("frac"),
            "traffic": traffic, "peak_source": peaks["source"]}
    if rec is not None:
        roof["traffic_source"] = rec["summary"]
        if rec.get("scaled_from"):
            roof["traffic_note"] = rec["scaled_from"]
    return roof


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(wl, budget_s: float = 12.0, single_budget_s: float = 4.0) -> dict:
    """The fp64 oracle on a bounded sample of query rows of the same workload (rank 0, N=1):
    first on all host threads, then single-threaded. Rows are drawn uniformly, so rows / time
    estimates the tokens/s of the whole sequence (each row's work, indexer scores over its visible
    entries included, is independent given the pools); the estimate is marked extrapolated when
    the sample is smaller than the workload."""
    import oracle
    t0 = time.perf_counter()
    threads = oracle.max_threads()
    n = max(1, threads)
    x = W.prefill_inputs(wl, with_queries=False)
    rng = np.random.default_rng(0)
    total = wl.B * wl.S
    while True:
        rows = np.sort(rng.choice(total, size=min(n, total), replace=False))
        dt = oracle_rows(wl, x, rows)
        if dt > budget_s / 3 or n >= total or time.perf_counter() - t0 > budget_s:
            break
        n = int(n * min(8.0, max(2.0, (budget_s / 3) / max(dt, 1e-3))))
    out = {"value": len(rows) / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": f"{len(rows)} random query rows of {wl.name} (full path incl. compressor "
                     f"over all {wl.S} tokens), {dt:.2f} s on {threads} threads",
           "extrapolated": len(rows) < total}
    # single-threaded point on a smaller sample of the same rows
    oracle.set_threads(1)
    try:
        n1 = max(1, min(len(rows), int(len(rows) * single_budget_s / max(dt * threads, 1e-3))))
        rows1 = rows[:n1]
        dt1 = oracle_rows(wl, x, rows1)
        out["single_thread"] = {"value": len(rows1) / dt1, "unit": "tokens/s", "cores": 1,
                                "sample": f"{len(rows1)} of the same rows, {dt1:.2f} s",
                                "extrapolated": len(rows1) < total}
    finally:
        oracle.set_threads(threads)
    return out


def oracle_rows(wl, x, rows) -> float:
    import oracle
    p = oracle.OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L,
                            nI=wl.nI, cI=wl.cI, k=wl.k)
    rq = W.prefill_row_inputs(wl, rows)
    t = time.perf_counter()
    if wl.kind == "csa":
        oracle.csa_forward(p, rq["q"], x["kv"], x["cmp_gate"], x["cmp_bias"], rq["q_idx"],
                           rq["w_idx"], x["k_idx"], x["idx_gate"], x["idx_bias"], x["sinks"],
                           rows=rows)
    elif wl.kind == "hca":
        oracle.hca_forward(p, rq["q"], x["kv"], x["cmp_gate"], x["cmp_bias"], x["sinks"],
                           rows=rows)
    else:
        oracle.swa_forward(p, rq["q"], x["kv"], x["sinks"], rows=rows)
    return time.perf_counter() - t


def config_of(wl, world):
    cfg = {"workload": wl.name, "B": wl.B, "S": wl.S, "H": wl.H, "head_dim": wl.D,
           "rope_dim": wl.R, "rope_theta": wl.theta, "sliding_window": wl.W,
           "parallelism": f"dp{world}",
           "l2": "inputs larger than L2 (q alone %d MiB > 126 MiB), no flush" %
                 (wl.B * wl.S * wl.H * wl.D * (2 if wl.dtype == "bf16" else 4) // 2 ** 20),
           "launch": "one CUDA graph replay per step"}
    if wl.kind in ("csa", "hca"):
        cfg.update(m=wl.m, compressor_window=wl.L)
    if wl.kind == "csa":
        cfg.update(index_n_heads=wl.nI, index_head_dim=wl.cI, index_topk=wl.k)
    return cfg


def run_ours(args, wl0):
    import sparse_attention_compressor_b200 as sac
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    wl = rank_workload(wl0, rank)
    host = W.prefill_inputs(wl)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    g = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
    torch.cuda.synchronize(dev)
    step, o = make_step(wl, g, dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # one step captured as a CUDA graph
    graph = capture(step)
    graph.replay()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        clk.wait_samples(1, graph.replay)
        ms = timed(graph.replay, args.steps, dev)
        clk.wait_samples(len(clk.lines) + 1, graph.replay)
    ktimes = kernel_times(step, dev)
    ms = max_over_ranks(ms, dev)
    ms_step = ms / args.steps
    tokens = wl.B * wl.S * world
    value = tokens / (ms_step * 1e-3)

    # end to end: pinned host inputs -> device, the call, the output back to pinned host memory
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = o.numel() * o.element_size()

    def e2e_step():
        for k, v in pinned.items():
            g[k].copy_(v, non_blocking=True)
        step()
        o_host.copy_(o, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize(dev)
    e2e_graph = capture(e2e_step)
    e2e_ms = max_over_ranks(timed(e2e_graph.replay, args.steps, dev), dev) / args.steps

    peaks = measured_peaks()
    roof, krows = roofline(wl, ktimes, peaks, 1, tensor_kernels=tensor_kernels(wl))
    launches = sum(v[0] for v in ktimes.values()) * args.steps
    line = {
        "metric": f"{wl.kind.upper()} attention fwd tokens/s (prefill)", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": DATA,
        "config": config_of(wl, world), "clocks": clk.summary(),
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches, "roofline": roof, "kernels": krows,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------------------------------------
# query-sharded prefill: one sequence over N ranks (halo send / recv, pool all-gather)
# ------------------------------------------------------------------------------------------------
def run_sharded(args, wl):
    """One step = sharded_forward on every rank: the halo exchange, the local cache append, the
    NCCL all-gather of the pools and the rank's chunk of queries. Strong scaling: the sequence is
    fixed, each rank takes S/N of its queries."""
    import sparse_attention_compressor_b200 as sac
    from sparse_attention_compressor_b200 import sharded
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    kind = sac.SAC_KIND_CSA if wl.kind == "csa" else sac.SAC_KIND_HCA
    sp = sharded.plan(wl.S, world, rank, wl.m, wl.L, wl.W, page_size=64)
    x = {k: v.to(dev) for k, v in W.prefill_slice_inputs(wl, sp.s0, sp.s1).items()}
    p = sac.make_params(1, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                        sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                        dtype=wl.dtype)
    o = torch.empty_like(x["q"])
    ws = torch.empty(sac.sac_chunk_workspace_size(p, kind, 1, sp.n), dtype=torch.uint8,
                     device=dev)

    def step():
        sharded.sharded_forward(sp, kind, p, x, o, ws=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        clk.wait_samples(1, step)
        ms = timed(step, args.steps, dev)
        clk.wait_samples(len(clk.lines) + 1, step)
    ms = max_over_ranks(ms, dev) / args.steps
    line = {
        "metric": f"{wl.kind.upper()} attention fwd tokens/s (prefill)",
        "value": wl.S / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": wl.dtype, "data": DATA,
        "config": dict(config_of(wl, world), parallelism=f"seq{world}",
                       launch="eager launches per step (halo send / recv and pool all-gather on "
                              "NCCL, then the chunk kernels)"),
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------------------------------------
# decode: one step = the CSA layer and the HCA layer, each over its paged cache
# ------------------------------------------------------------------------------------------------
def decode_bytes(wl, d_csa, d_hca) -> dict:
    """Algorithmic HBM bytes per decode step (what must be read / written once)."""
    esz = 2
    out = {}
    ctx = d_csa["ctx_lens"].numpy().astype(np.int64)
    nv = ctx // wl.m
    win = np.minimum(ctx, wl.W)
    qb = wl.nseq * wl.H * wl.D * esz
    out["indexer_score"] = float((nv * wl.cI * esz).sum() + wl.nseq * wl.nI * (wl.cI * esz + 4)
                                 + (nv * 4).sum())
    out["topk"] = float((nv * 4).sum() + wl.nseq * wl.k * 4)
    out["csa_decode_attention"] = float(((np.minimum(nv, wl.k) + win) * wl.D * esz).sum() + 2 * qb)
    ctx_h = d_hca["ctx_lens"].numpy().astype(np.int64)
    out["hca_decode_attention"] = float(((ctx_h // d_hca["m"] + np.minimum(ctx_h, wl.W))
                                         * wl.D * esz).sum() + 2 * qb)
    # cache append: the new row read, written rotated to its page and un-rotated to the ring; a
    # closing window (ctx % m == 0) reads its L ring rows and writes one entry
    app = 0.0
    for d, m, L in ((d_csa, wl.m, wl.L), (d_hca, d_hca["m"], d_hca["m"])):
        closing = int((d["ctx_lens"].numpy() % m == 0).sum())
        app += wl.nseq * 3 * wl.D * esz + closing * (L + 1) * wl.D * esz
    out["decode_append"] = app
    closing = int((d_csa["ctx_lens"].numpy() % wl.m == 0).sum())
    out["decode_append_index"] = float(wl.nseq * 2 * wl.cI * esz + closing * (wl.L + 1) * wl.cI * esz)
    return out


def chunk_work(wl, d_csa, d_hca) -> dict:
    """Algorithmic work per chunked-prefill step: FLOPs of the contractions (indexer scores and
    attention, tensor-bound: every chunk row re-uses the same cached rows), bytes of the rest."""
    esz, n = 2, wl.chunk
    out = {}
    ctx = d_csa["ctx_lens"].numpy().astype(np.int64)
    t = (ctx[:, None] - n + np.arange(n)[None, :])  # [nseq, n] positions of the chunk rows
    nv = (t + 1) // wl.m
    win = np.minimum(t + 1, wl.W)
    out["indexer_score"] = ("flops", float((nv * 2 * wl.nI * wl.cI).sum()))
    out["topk"] = ("bytes", float((nv * 4).sum() + t.size * wl.k * 4))
    out["csa_chunk_attention"] = ("flops", float(((np.minimum(nv, wl.k) + win)
                                                  * 4 * wl.H * wl.D).sum()))
    ctx_h = d_hca["ctx_lens"].numpy().astype(np.int64)
    th = (ctx_h[:, None] - n + np.arange(n)[None, :])
    out["hca_chunk_attention"] = ("flops", float(((th + 1) // d_hca["m"] + np.minimum(th + 1, wl.W))
                                                 .sum() * 4 * wl.H * wl.D))
    # append: every chunk row read once and written rotated (plus the ring's last L rows); each
    # closing entry reads its L rows and writes one
    app = 0.0
    for d, m, L in ((d_csa, wl.m, wl.L), (d_hca, d_hca["m"], d_hca["m"])):
        c = d["ctx_lens"].numpy().astype(np.int64)
        closing = (c // m - (c - n) // m).sum()
        app += (2 * t.size + wl.nseq * min(L, n)) * wl.D * esz + closing * (L + 1) * wl.D * esz
    out["chunk_append"] = ("bytes", float(app))
    closing = (ctx // wl.m - (ctx - n) // wl.m).sum()
    out["chunk_append_index"] = ("bytes", float((t.size + wl.nseq * min(wl.L, n)) * wl.cI * esz
                                                + closing * (wl.L + 1) * wl.cI * esz))
    return out


def run_decode(args, wl0):
    import sparse_attention_compressor_b200 as sac
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    wl = rank_workload(wl0, rank)
    dc = W.decode_inputs(wl, "csa")
    dh = W.decode_inputs(wl, "hca")
    gc = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in dc.items()}
    gh = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in dh.items()}
    max_ctx = int(max(dc["ctx_lens"].max(), dh["ctx_lens"].max()))
    pc = sac.make_params(1, max_ctx, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                         sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                         dtype=wl.dtype)
    ph = sac.make_params(1, max_ctx, wl.H, wl.D, wl.R, wl.theta, m=dh["m"], win_len=dh["m"],
                         sliding_window=wl.W, dtype=wl.dtype)
    n = wl.chunk
    if n > 1:
        ws = torch.empty(sac.sac_chunk_workspace_size(pc, sac.SAC_KIND_CSA, wl.nseq, n),
                         dtype=torch.uint8, device=dev)
        ws_h = torch.empty(sac.sac_chunk_workspace_size(ph, sac.SAC_KIND_HCA, wl.nseq, n),
                           dtype=torch.uint8, device=dev)
    else:
        ws = torch.empty(sac.sac_decode_workspace_size(pc, sac.SAC_KIND_CSA, wl.nseq),
                         dtype=torch.uint8, device=dev)
        ws_h = torch.empty(sac.sac_decode_workspace_size(ph, sac.SAC_KIND_HCA, wl.nseq),
                           dtype=torch.uint8, device=dev)
    oc = torch.empty_like(gc["q"])
    oh = torch.empty_like(gh["q"])
    ps = wl.page_size

    def chunk_step():
        # each layer: append the chunk's tokens to its caches, then attend
        sac.prefill_chunk_append(pc, sac.SAC_KIND_CSA, wl.nseq, n, gc["ctx_lens"], gc["kv_new"],
                                 gc["kv_pages"], gc["kv_block_table"], ps,
                                 cmp_state=gc["cmp_state"], cmp_gate=gc["cmp_gate"],
                                 cmp_bias=gc["cmp_bias"], pool_pages=gc["pool_pages"],
                                 pool_block_table=gc["pool_block_table"],
                                 k_idx_new=gc["k_idx_new"], idx_state=gc["idx_state"],
                                 idx_gate=gc["idx_gate"], idx_bias=gc["idx_bias"],
                                 idx_pool_pages=gc["idx_pool_pages"])
        sac.csa_prefill_chunk(pc, wl.nseq, n, gc["q"], gc["kv_pages"], gc["kv_block_table"],
                              gc["ctx_lens"], ps, gc["pool_pages"], gc["idx_pool_pages"],
                              gc["pool_block_table"], gc["q_idx"], gc["w_idx"], gc["sinks"], oc,
                              None, ws)
        sac.prefill_chunk_append(ph, sac.SAC_KIND_HCA, wl.nseq, n, gh["ctx_lens"], gh["kv_new"],
                                 gh["kv_pages"], gh["kv_block_table"], ps,
                                 cmp_state=gh["cmp_state"], cmp_gate=gh["cmp_gate"],
                                 cmp_bias=gh["cmp_bias"], pool_pages=gh["pool_pages"],
                                 pool_block_table=gh["pool_block_table"])
        sac.hca_prefill_chunk(ph, wl.nseq, n, gh["q"], gh["kv_pages"], gh["kv_block_table"],
                              gh["ctx_lens"], ps, gh["pool_pages"], gh["pool_block_table"],
                              gh["sinks"], oh, ws_h)

    def decode_step():
        # each layer: append the new token to its caches, then attend
        sac.decode_append(pc, sac.SAC_KIND_CSA, wl.nseq, gc["ctx_lens"], gc["kv_new"],
                          gc["kv_pages"], gc["kv_block_table"], ps, cmp_state=gc["cmp_state"],
                          cmp_gate=gc["cmp_gate"], cmp_bias=gc["cmp_bias"],
                          pool_pages=gc["pool_pages"], pool_block_table=gc["pool_block_table"],
                          k_idx_new=gc["k_idx_new"], idx_state=gc["idx_state"],
                          idx_gate=gc["idx_gate"], idx_bias=gc["idx_bias"],
                          idx_pool_pages=gc["idx_pool_pages"])
        sac.csa_decode(pc, wl.nseq, gc["q"], gc["kv_pages"], gc["kv_block_table"], gc["ctx_lens"],
                       ps, gc["pool_pages"], gc["idx_pool_pages"], gc["pool_block_table"],
                       gc["q_idx"], gc["w_idx"], gc["sinks"], oc, None, ws)
        sac.decode_append(ph, sac.SAC_KIND_HCA, wl.nseq, gh["ctx_lens"], gh["kv_new"],
                          gh["kv_pages"], gh["kv_block_table"], ps, cmp_state=gh["cmp_state"],
                          cmp_gate=gh["cmp_gate"], cmp_bias=gh["cmp_bias"],
                          pool_pages=gh["pool_pages"], pool_block_table=gh["pool_block_table"])
        sac.hca_decode(ph, wl.nseq, gh["q"], gh["kv_pages"], gh["kv_block_table"], gh["ctx_lens"],
                       ps, gh["pool_pages"], gh["pool_block_table"], gh["sinks"], oh, ws_h)

    step = chunk_step if n > 1 else decode_step
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    graph = capture(step)
    graph.replay()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        clk.wait_samples(1, graph.replay)
        ms = timed_flushed(graph.replay, args.steps, dev)
        clk.wait_samples(len(clk.lines) + 1, graph.replay)
    ktimes = kernel_times(step, dev, flush=True)
    ms = max_over_ranks(ms, dev)
    us_step = 1e3 * ms / args.steps
    # end to end: the step's new-token inputs from pinned host memory, outputs back
    pin = {k: dc[k].pin_memory() for k in ("q", "q_idx", "w_idx", "kv_new", "k_idx_new")}
    pin["q_h"] = dh["q"].pin_memory()
    pin["kv_new_h"] = dh["kv_new"].pin_memory()
    oc_h = torch.empty(oc.shape, dtype=oc.dtype, pin_memory=True)
    oh_h = torch.empty(oh.shape, dtype=oh.dtype, pin_memory=True)

    def e2e_step():
        gc["q"].copy_(pin["q"], non_blocking=True)
        gc["q_idx"].copy_(pin["q_idx"], non_blocking=True)
        gc["w_idx"].copy_(pin["w_idx"], non_blocking=True)
        gc["kv_new"].copy_(pin["kv_new"], non_blocking=True)
        gc["k_idx_new"].copy_(pin["k_idx_new"], non_blocking=True)
        gh["q"].copy_(pin["q_h"], non_blocking=True)
        gh["kv_new"].copy_(pin["kv_new_h"], non_blocking=True)
        step()
        oc_h.copy_(oc, non_blocking=True)
        oh_h.copy_(oh, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize(dev)
    e2e_graph = capture(e2e_step)
    e2e_us = 1e3 * max_over_ranks(timed_flushed(e2e_graph.replay, args.steps, dev),
                                  dev) / args.steps
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = (oc.numel() + oh.numel()) * oc.element_size()
    peaks = measured_peaks()
    if n > 1:
        wb = chunk_work(wl, dc, dh)
    else:
        db = decode_bytes(wl, dc, dh)
        if "decode_append_index" not in ktimes:  # both CSA parts ran as one launch
            db["decode_append"] += db.pop("decode_append_index")
        wb = {k: ("bytes", v) for k, v in db.items()}
    krows = {}
    total = sum(v[1] for v in ktimes.values()) or 1.0
    for name, (launches, kms) in ktimes.items():
        per = kms / max(launches, 1)
        row = {"launches": launches, "ms_per_launch": per, "share": kms / total}
        if name in wb:
            kind, amount = wb[name]
            if kind == "bytes":
                ach = amount / launches / (per * 1e-3) / 1e9
                row.update(bound="hbm", achieved=ach, peak=peaks["hbm_gbs"], unit="GB/s",
                           frac=ach / peaks["hbm_gbs"])
            else:
                ach = amount / launches / (per * 1e-3) / 1e12
                row.update(bound="tensor", achieved=ach, peak=peaks["bf16_tflops"],
                           unit="TFLOP/s", frac=ach / peaks["bf16_tflops"])
        krows[name] = row
    dom = max(ktimes, key=lambda k: ktimes[k][1])
    d = krows[dom]
    cfg = {"workload": wl.name, "nseq": wl.nseq, "ctx": f"U[{wl.ctx_lo},{wl.ctx_hi}]",
           "page_size": wl.page_size, "H": wl.H, "head_dim": wl.D, "csa_m": wl.m,
           "hca_m": dh["m"], "index_topk": wl.k, "sliding_window": wl.W,
           "parallelism": f"dp{world}",
           "l2": "flushed before every step (252 MiB written, then another 252 MiB read)",
           "launch": "one CUDA graph replay per step (cache append + both layers)"}
    if n > 1:
        cfg["chunk"] = n
        tok_s = wl.nseq * n * world / (us_step * 1e-6)
        head = {"metric": f"chunked prefill tokens/s (CSA + HCA layer, {wl.nseq} sequences x {n}"
                          " tokens against a cached prefix)",
                "value": tok_s, "unit": "tokens/s", "higher_is_better": True}
        e2e = {"value": wl.nseq * n * world / (e2e_us * 1e-6), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    else:
        head = {"metric": "decode us/step (CSA + HCA layer, 64 sequences)", "value": us_step,
                "unit": "us/step", "higher_is_better": False}
        e2e = {"value": e2e_us, "unit": "us/step", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
    line = {
        "metric": head["metric"], "value": head["value"],
        "unit": head["unit"], "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us_step / 1e3, "higher_is_better": head["higher_is_better"],
        "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": DATA,
        "config": cfg,
        "clocks": clk.summary(),
        "e2e": e2e,
        "gpu_launches": sum(v[0] for v in ktimes.values()) * args.steps,
        "roofline": roof_of(wl.name, dom, d, peaks),
        "kernels": krows,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = inline_cpu_baseline(run_reference_paged, wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_oproj(args, wl0):
    """The grouped output projection alone: two GEMMs, timed like the prefill path."""
    import sparse_attention_compressor_b200 as sac
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    wl = rank_workload(wl0, rank)
    T, G, rk, hid = wl.B * wl.S, wl.o_groups, wl.o_rank, wl.hidden
    x = W.oproj_inputs(T, wl.H, wl.D, G, rk, hid, wl.seed)
    g = {k: v.to(dev).contiguous() for k, v in x.items()}
    p = sac.make_params(1, T, wl.H, wl.D, wl.R, wl.theta)
    ws = torch.empty(sac.sac_oproj_workspace_size(p, T, G, rk), dtype=torch.uint8, device=dev)
    out = torch.empty((T, hid), dtype=torch.bfloat16, device=dev)

    def step():
        sac.o_proj_forward(p, T, G, rk, hid, g["o"], g["w_a"], g["w_b"], out, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    graph = capture(step)
    graph.replay()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        clk.wait_samples(1, graph.replay)
        ms = timed_flushed(graph.replay, args.steps, dev)
        clk.wait_samples(len(clk.lines) + 1, graph.replay)
    ktimes = kernel_times(step, dev, flush=True)
    ms = max_over_ranks(ms, dev) / args.steps
    pin_o = x["o"].pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def e2e_step():
        g["o"].copy_(pin_o, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize(dev)
    e2e_graph = capture(e2e_step)
    e2e_ms = max_over_ranks(timed_flushed(e2e_graph.replay, args.steps, dev), dev) / args.steps
    peaks = measured_peaks()
    flops = 2.0 * T * (wl.H * wl.D * rk + G * rk * hid)
    launches, kms = ktimes.get("o_proj", (1, ms))
    ach = flops / (kms / max(launches, 1) * 1e-3) / 1e12
    line = {
        "metric": "grouped output projection tokens/s", "value": T * world / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": DATA,
        "config": {"workload": wl.name, "tokens": T, "H": wl.H, "head_dim": wl.D,
                   "o_groups": G, "o_lora_rank": rk, "hidden": hid, "parallelism": f"dp{world}",
                   "l2": "flushed before every step (252 MiB written, then another 252 MiB read)",
                   "launch": "one CUDA graph replay per step (two tcgen05 GEMM launches)"},
        "clocks": clk.summary(),
        "e2e": {"value": T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": pin_o.numel() * 2, "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": 2 * args.steps,
        "roofline": roof_of(wl.name, "o_proj", {"bound": "tensor", "achieved": ach,
                                                 "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                                 "frac": ach / peaks["bf16_tflops"]}, peaks),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = inline_cpu_baseline(run_reference_oproj, wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def _logical_rows(pages, bt, s, lo, hi):
    """Rows lo..hi-1 of sequence s of a paged cache (CPU tensors) as float64 numpy."""
    ps = pages.shape[1]
    idx = np.arange(lo, hi)
    pg = bt[s, idx // ps].numpy()
    return pages[torch.from_numpy(pg).long(), torch.from_numpy(idx % ps)].double().numpy()


def _oracle_paged_step(wl, d, layer, rows):
    """The oracle's attention of the listed (sequence, position) rows of one layer over the rows of
    the paged caches they read (copied once per sequence to a page-size-1 layout); seconds."""
    import oracle
    m = d["m"]
    seqs = sorted({s for s, _ in rows})
    slot = {s: i for i, s in enumerate(seqs)}
    ctx = d["ctx_lens"].numpy()
    kv_rows, pool_rows, ipool_rows = [], [], []
    maxc = int(max(ctx[s] for s in seqs))
    kbt = np.full((len(seqs), maxc), -1, dtype=np.int32)
    pbt = np.full((len(seqs), max(1, maxc // m)), -1, dtype=np.int32)
    nk = npl = 0
    for s in seqs:
        c, i = int(ctx[s]), slot[s]
        lo = max(0, min(t for ss, t in rows if ss == s) - wl.W + 1)
        kv_rows.append(_logical_rows(d["kv_pages"], d["kv_block_table"], s, lo, c))
        kbt[i, lo:c] = np.arange(nk, nk + c - lo)
        nk += c - lo
        nv = c // m
        if nv:
            pool_rows.append(_logical_rows(d["pool_pages"], d["pool_block_table"], s, 0, nv))
            if layer == "csa":
                ipool_rows.append(_logical_rows(d["idx_pool_pages"], d["pool_block_table"], s, 0,
                                                nv))
            pbt[i, :nv] = np.arange(npl, npl + nv)
            npl += nv
    p = oracle.OracleParams(1, maxc, wl.H, wl.D, wl.R, wl.theta, wl.W, m=m,
                            L=wl.L if layer == "csa" else m, nI=wl.nI if layer == "csa" else 0,
                            cI=wl.cI if layer == "csa" else 0, k=wl.k if layer == "csa" else 0)
    n = wl.chunk
    def tok(name, s, t):  # the per-token tensor row of (s, t)
        x = d[name]
        return x[s] if n == 1 else x[s, t - (int(ctx[s]) - n)]
    q = np.stack([tok("q", s, t).double().numpy() for s, t in rows])
    kw = {}
    if layer == "csa":
        kw = dict(q_idx=np.stack([tok("q_idx", s, t).double().numpy() for s, t in rows]),
                  w_idx=np.stack([tok("w_idx", s, t).double().numpy() for s, t in rows]),
                  idx_pool_pages=np.concatenate(ipool_rows)[:, None, :])
    sl = [slot[s] for s, _ in rows]
    t0 = time.perf_counter()
    oracle.decode(p, q, np.concatenate(kv_rows)[:, None, :], kbt[sl],
                  np.array([t + 1 for _, t in rows], dtype=np.int32), 1,
                  pool_pages=np.concatenate(pool_rows)[:, None, :], pool_block_table=pbt[sl],
                  sinks=d["sinks"].double().numpy(), **kw)
    return time.perf_counter() - t0


def run_reference_paged(args, wl):
    """The oracle on a bounded sample of a decode (or chunked-prefill) step: the attention of a
    few query rows of each layer, scaled to the step's rows by count."""
    import oracle
    oracle.build()
    world, _, _ = dist_env()
    dc, dh = W.decode_inputs(wl, "csa"), W.decode_inputs(wl, "hca")
    n = wl.chunk
    rng = np.random.default_rng(2)
    ctx_c, ctx_h = dc["ctx_lens"].numpy(), dh["ctx_lens"].numpy()
    per = 4  # sampled rows per layer and step
    def sample(ctx):
        ss = rng.choice(wl.nseq, size=per)
        return [(int(s), int(ctx[s]) - 1 - int(rng.integers(0, n))) for s in ss]
    times = []
    for i in range(args.warmup + args.steps):
        t = _oracle_paged_step(wl, dc, "csa", sample(ctx_c)) + \
            _oracle_paged_step(wl, dh, "hca", sample(ctx_h))
        if i >= args.warmup:
            times.append(t)
    rows_step = wl.nseq * n
    s_per_step = sum(times) / len(times) * rows_step / per
    threads = oracle.max_threads()
    sample_txt = (f"each step: {per} random query rows of each layer (CSA with its indexer and "
                  f"top-k, HCA) through the oracle's paged attention, scaled by count to the "
                  f"{rows_step} rows of a step")
    if n > 1:
        value, unit, hib = rows_step / s_per_step, "tokens/s", True
        metric = (f"chunked prefill tokens/s (CSA + HCA layer, {wl.nseq} sequences x {n} tokens "
                  "against a cached prefix)")
    else:
        value, unit, hib = s_per_step * 1e6, "us/step", False
        metric = "decode us/step (CSA + HCA layer, 64 sequences)"
    return metric, value, unit, hib, s_per_step * 1e3, threads, sample_txt


def run_reference_oproj(args, wl):
    """The oracle's grouped output projection of a bounded sample of token rows."""
    import oracle
    oracle.build()
    T = wl.B * wl.S
    x = W.oproj_inputs(T, wl.H, wl.D, wl.o_groups, wl.o_rank, wl.hidden, wl.seed)
    o, wa, wb = (x[k].double().numpy() for k in ("o", "w_a", "w_b"))
    rng = np.random.default_rng(3)
    per = 64
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(T, size=per, replace=False))
        t0 = time.perf_counter()
        oracle.o_proj(o, wa, wb, wl.o_groups, rows=rows, round_mid=True)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    s = sum(times) / len(times)
    return ("grouped output projection tokens/s", per / s, "tokens/s", True, s * 1e3,
            oracle.max_threads(), f"each step: {per} random token rows of {T}")


def inline_cpu_baseline(fn, wl) -> dict:
    """The oracle arm of a decode, chunked-prefill or projection workload on a small sample (one
    warm-up and two timed steps), as the bench line's cpu_baseline."""
    class _A:
        warmup, steps = 1, 2
    _, value, unit, _, _, threads, sample = fn(_A, wl)
    return {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model()}


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    if wl.kind in ("decode", "oproj"):
        fn = run_reference_paged if wl.kind == "decode" else run_reference_oproj
        metric, value, unit, hib, ms_step, threads, sample = fn(args, wl)
        line = {
            "impl": "reference", "metric": metric, "value": value, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": hib, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "parallelism": f"dp{world}"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    import oracle
    oracle.build()
    x = W.prefill_inputs(wl, with_queries=False)
    threads = oracle.max_threads()
    # rows per step: long sequences cost more per row (the indexer scores every visible entry)
    n = max(16, int(32 * threads * min(1.0, 32768 / wl.S)))
    rng = np.random.default_rng(1)
    samples = [np.sort(rng.choice(wl.B * wl.S, size=n, replace=False))
               for _ in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle_rows(wl, x, samples[i])
    t = [oracle_rows(wl, x, samples[args.warmup + i]) for i in range(args.steps)]
    ms_step = 1e3 * sum(t) / len(t)
    value = n / (ms_step * 1e-3)
    sample = (f"each step: {n} random query rows of {wl.name} through the full oracle path "
              f"(compressor over all {wl.S} tokens, indexer, top-k, attention)")
    line = {
        "impl": "reference", "metric": f"{wl.kind.upper()} attention fwd tokens/s (prefill)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def launch_ranks(n: int, argv: list) -> int:
    """Run this script on n local ranks (torch.distributed.run, rendezvous on 127.0.0.1) and return
    the launcher's exit status; rank 0 prints the JSON line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + argv
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="csa_128k_bf16", choices=list(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["dp", "seq"], default="dp",
                    help="dp: every rank its own sequence (weak scaling); seq: one sequence "
                         "split by queries over the ranks (CSA / HCA prefill, strong scaling)")
    ap.add_argument("--record-traffic", nargs=4, metavar=("RAW_CSV", "KERNEL", "REGEX", "SUMMARY"),
                    help="write the ncu traffic record of KERNEL on --workload from a raw-page "
                         "CSV of its capture (no GPU work)")
    ap.add_argument("--traffic-scale", type=float, default=1.0)
    ap.add_argument("--traffic-scaled-from", default="")
    args = ap.parse_args(argv)
    wl = W.WORKLOADS[args.workload]
    if args.record_traffic:
        raw, kern, rx, summ = args.record_traffic
        print(json.dumps(record_traffic(raw, args.workload, kern, rx, summ, args.traffic_scale,
                                        args.traffic_scaled_from)))
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: relaunch this command under torch.distributed.run
        sys.exit(launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv)))
    if args.impl == "reference":
        run_reference(args, wl)
    elif wl.kind == "decode":
        run_decode(args, wl)
    elif wl.kind == "oproj":
        run_oproj(args, wl)
    elif args.shard == "seq" and wl.kind in ("csa", "hca"):
        run_sharded(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
