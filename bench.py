#!/usr/bin/env python
"""Benchmark: GQA decode over a KV cache on B200.

One step = one decode step of the whole path for one batch of sequences: the
split-KV decode kernel (group mapping, page-table translation, K/V tile loads,
q.k scores, online softmax, p.V) and, where the decomposition needs one, the
combine kernel that merges the splits and normalises.  The inputs are resident
in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ragged]
    python bench.py --query-tokens 8 --workload llama70b   # a verification step: 8 query tokens per sequence
    python bench.py --impl reference ...                    # the float64 CPU oracle instead

Prints one JSON line (rank 0).  The headline is the workload named by
--workload (default: the ragged paged batch, the largest single-GPU
configuration); ``per_config`` holds the same measurement for every workload
(tiny, Llama-2-70B layer, ragged, long-context b=1 and b=4, the group-ratio
sweep G = 1, 2, 4, 8, 32) and two verification steps, taken in the same
process at the same step count.  Under torchrun every rank runs its own shard
of sequences of the same shape (weak scaling, no collective on the data path);
the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_bandwidth_b200 import accounting  # noqa: E402
from kv_cache_bandwidth_b200.workloads import WORKLOADS, draw_verify_q, make_inputs  # noqa: E402

METRIC = "GQA decode µs/step and KV-cache HBM GB/s as % of B200 peak (1 GPU)"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
# The workloads of per_config, and the verification steps measured beside them.
PER_CONFIG = ["tiny", "llama70b", "ragged", "long1", "long4", "sweep_g1", "sweep_g2", "sweep_g4", "sweep_g8",
              "sweep_g32"]
PER_CONFIG_VERIFY = [("llama70b", 8), ("llama70b", 16)]
# Copies of a cache that fits in L2 that the steps rotate over (at most): the
# other copies' bytes between two reads of one copy must exceed twice the L2.
MAX_ROTATE_COPIES = 16


# --------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The sources each profiled kernel is built from (its own header, the helpers
# it includes and the launch code); a committed ncu record stays valid while
# these hash the same.
KERNEL_SOURCES = {
    "gqa_decode_kernel": ("gqa_api.cu", "gqa_kernels.cuh", "ptx.cuh"),
    "gqa_combine_kernel": ("gqa_api.cu", "gqa_kernels.cuh", "ptx.cuh"),
    "gqa_verify_tc_kernel": ("gqa_api.cu", "gqa_kernels.cuh", "gqa_verify_tc.cuh", "ptx.cuh", "tc05.cuh"),
}


def kernel_source_hash(files=None) -> str:
    """sha256 (16 hex digits) over the named csrc files (default: all of them)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_bandwidth_b200", "csrc")
    for name in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_key(workload: str, n_query: int = 1) -> str:
    return workload if n_query == 1 else "%s_verify%d" % (workload, n_query)


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the decode kernel from a committed ncu capture,
    if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_hash") == kernel_source_hash(KERNEL_SOURCES.get(e.get("kernel_name"))):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def l2_plan(kv_bytes: int):
    """How steps of a workload are kept from reading L2-resident data:
    ("resident", 1) when the KV bytes exceed three times the L2 (each step
    streams the cache through L2 and evicts its own start long before the
    next step reads it again); ("rotate", n) when n <=
    MAX_ROTATE_COPIES copies of the cache, read in turn, put more than twice
    the L2 between two reads of one copy; else ("flush", 1): L2 is flushed
    before every step and each step is timed alone."""
    if kv_bytes > 3 * L2_BYTES:
        return "resident", 1
    n = 2 + (2 * L2_BYTES) // kv_bytes if kv_bytes else MAX_ROTATE_COPIES + 1
    if n <= MAX_ROTATE_COPIES:
        return "rotate", n
    return "flush", 1


def l2_desc(kv_bytes: int) -> str:
    how, n = l2_plan(kv_bytes)
    if how == "resident":
        return "inputs %.0f MiB > 3x the 126 MB L2, steps back to back (no flush)" % (kv_bytes / 2 ** 20)
    if how == "rotate":
        return ("steps back to back over %d copies of the %.0f MiB cache in turn (%.0f MiB of other copies "
                "between two reads of one copy > 2x L2)" % (n, kv_bytes / 2 ** 20, (n - 1) * kv_bytes / 2 ** 20))
    return "L2 flushed before every step (2x L2 written, then 2x L2 read), each step timed alone"


class ClockSampler:
    """Samples SM clocks and clock-event reasons during the timed region (NVML)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, interval_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.interval = interval_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for b, name in self.REASONS.items():
                if bits & b and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.interval)

    def __enter__(self):
        if self._nv is not None:
            self._stop.clear()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
            self._thread = None

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    from kv_cache_bandwidth_b200 import dist as gdist

    return x if world == 1 else gdist.max_over_ranks(x)


def config_dict(w, inp, n_query=1):
    """The workload a line measures (the same dict in both arms): its shape,
    layout, KV bytes, seed and how L2 is kept out of the timing.  How the
    library decomposes the step is reported beside it, under "plan"."""
    kv = accounting.kv_bytes_per_step(w.G, w.d, inp.seqlens.tolist())
    cfg = {
        "workload": w.name if n_query == 1 else "verification step, %d query tokens per sequence, over %s" % (
            n_query, w.name), "b": w.b, "H": w.H, "G": w.G, "d": w.d, "m": w.m,
        "layout": "paged P=%d" % w.page_size if w.paged else "contiguous [b,G,m,d]",
        "kv_bytes_per_step": kv, "seed": w.seed, "l2": l2_desc(kv),
    }
    if w.len_lo is not None:
        cfg["lengths"] = "uniform integers in [%d, %d] (seeded)" % (w.len_lo, w.len_hi)
    if w.peaky_frac > 0:
        cfg["peaky"] = "%.0f%% of key rows x8 per (sequence, group)" % (100 * w.peaky_frac)
    if n_query > 1:
        cfg["query_tokens"] = n_query
        cfg["rows_per_kv_group"] = n_query * w.r
        cfg["mask"] = "query token t of n sees cached positions < len - (n - 1 - t)"
    return cfg


def plan_dict(split_tokens, max_len, n_query=1, tc=False, entry="split", cluster=0):
    """The library's decomposition of a step (GPU arm only)."""
    if entry == "cluster":
        decomp = "gqa_decode: one block or cluster per (sequence, group)"
    elif cluster > 1:
        decomp = ("thread-block clusters of %d blocks per (sequence, group), merged through distributed shared "
                  "memory (one kernel)" % cluster)
    elif split_tokens == 0:
        decomp = "equal-work ranges over all (sequence, group) tiles (stream-K) + combine"
    else:
        n_splits = -(-max_len // split_tokens)
        decomp = "fixed splits of %d tokens (%d per sequence), %s" % (
            split_tokens, n_splits, "one block per (sequence, group), final rows" if n_splits == 1 else
            "merged in the decode kernel" if n_splits <= 8 else "combine kernel")
    d = {"split_tokens": split_tokens, "decomposition": decomp}
    if cluster > 1:
        d["cluster_blocks"] = cluster
    if n_query > 1:
        d["kernel"] = "gqa_verify_tc_kernel (tcgen05)" if tc else "gqa_decode_kernel (mma.sync)"
    return d


# --------------------------------------------------------------------------- oracle leg

def oracle_time(inp, target_s: float = 15.0, max_seq=None, q_verify=None):
    """Time the float64 oracle (as it stands, all host cores) on a bounded
    sample of whole sequences of the workload, about target_s of CPU time: a
    prefix of the sequences when the workload is larger, or the whole workload
    repeated when it is smaller.  q_verify (bf16 [b, n, H, d]): time the
    oracle's verification decode of those query tokens instead.
    Returns (GB/s, seconds, threads, description)."""
    import numpy as np

    import oracle

    w = inp.workload
    q = inp.q.cpu() if q_verify is None else q_verify.cpu()
    nq = 1 if q_verify is None else q.shape[1]
    kc, vc = inp.k_cache.cpu(), inp.v_cache.cpu()
    sl = inp.seqlens.cpu()
    pt = None if inp.page_table is None else inp.page_table.cpu()
    threads = oracle.max_threads()
    lens = sl.tolist()

    def run(n_seq):
        rows = np.arange(n_seq * nq * w.H, dtype=np.int64)
        t0 = time.perf_counter()
        if q_verify is None:
            oracle.gqa_decode(q, kc, vc, sl, pt, num_kv_heads=w.G, scale=w.scale, rows=rows)
        else:
            oracle.gqa_decode_verify(q, kc, vc, sl, pt, num_kv_heads=w.G, scale=w.scale, rows=rows)
        return time.perf_counter() - t0

    probe = run(1)
    per_seq = max(probe, 1e-6)
    n = max(1, min(w.b if max_seq is None else max_seq, int(target_s / per_seq)))
    dt = run(n) if n > 1 else probe
    reps = 1
    if dt < 0.5 * target_s:  # the sample is quick: repeat it until about target_s
        reps = 1 + int((target_s - dt) / max(dt, 1e-6))
        reps = min(reps, 10000)
        for _ in range(reps - 1):
            dt += run(n)
    kv = accounting.kv_bytes_per_step(w.G, w.d, lens[:n])
    desc = "%d of %d sequences (all %d heads%s each) of the workload, %.3g GB of KV, %d run(s)" % (
        n, w.b, w.H, "" if nq == 1 else " x %d query tokens" % nq, kv / 1e9, reps)
    return reps * kv / dt / 1e9, dt, threads, desc


def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, device="cpu")
    qv = draw_verify_q(w, args.query_tokens) if args.query_tokens > 1 else None
    kv_step = accounting.kv_bytes_per_step(w.G, w.d, inp.seqlens.tolist())
    # every step a bounded sample: a whole-sequence slice sized so the run ends in minutes
    budget = args.oracle_seconds if args.oracle_seconds > 0 else min(15.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_time(inp, target_s=budget, q_verify=qv)
    vals, times, desc, threads = [], [], "", 0
    for _ in range(args.steps):
        gbs, dt, threads, desc = oracle_time(inp, target_s=budget, q_verify=qv)
        vals.append(gbs)
        times.append(dt)
    value = statistics.median(vals)
    ms = kv_step / (value * 1e9) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, inp, args.query_tokens),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU leg

class L2Flush:
    """Empties L2 of the step's inputs: writes a buffer of twice the L2 size,
    then reads another of the same size, so that L2 holds only clean lines of
    data the step never touches (a write alone would leave ~126 MB of dirty
    lines for the timed step to write back)."""

    def __init__(self):
        n = 2 * L2_BYTES // 4
        self.w = torch.empty(n, dtype=torch.float32, device="cuda")
        self.r = torch.ones(n, dtype=torch.float32, device="cuda")
        self.sink = None

    def __call__(self):
        self.w.zero_()
        self.sink = self.r.sum()


class Case:
    """One workload instance on the GPU and the public call of one step.

    The KV cache is the decode state and stays resident; a cache that fits in
    L2 is held in several copies that successive steps read in turn (see
    l2_plan), so that back-to-back steps still stream from HBM."""

    def __init__(self, args, w, nq, rank, with_copies=True):
        from kv_cache_bandwidth_b200 import gqa

        self.gqa = gqa
        self.w = w = w.with_(seed=w.seed + 1000 * rank)  # each rank: its own shard of sequences
        self.nq = nq
        self.entry = args.entry
        self.inp = inp = make_inputs(w, device="cuda")
        self.q = inp.q if nq == 1 else draw_verify_q(w, nq, device="cuda")
        self.kv_step = accounting.kv_bytes_per_step(w.G, w.d, inp.seqlens.tolist())
        self.max_seqlen = int(inp.seqlens.max())
        self.dims = gqa.dims_for(inp.q, inp.k_cache, inp.page_table)
        # 0: the library's choice (equal-work ranges for a paged cache); > 0:
        # fixed splits of that many tokens; -1: the library's plan
        split = max(0, args.split_tokens)
        self.split = split
        if nq == 1:
            self.ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, self.max_seqlen, split)
        else:
            n = gqa.gqa_decode_verify_workspace_size(self.dims, nq, self.max_seqlen, split)
            self.ws = torch.empty(max(256, n), dtype=torch.uint8, device="cuda")
        self.cluster = 0
        self.tc = gqa.TC_AUTO_ROWS < nq * w.r <= (128 if w.d == 128 else 64)
        if split > 0:
            self.eff_split = split
        elif self.entry == "split":
            kind, self.eff_split, c = gqa.gqa_plan_decomposition_ex(self.dims, self.max_seqlen, nq)
            self.cluster = c if kind == gqa.PLAN_CLUSTERS else 0
        else:
            self.eff_split = gqa.gqa_plan_split_tokens(self.dims, self.max_seqlen)
        n_splits = -(-self.max_seqlen // self.eff_split) if self.eff_split > 0 else 0
        self.launches_per_step = 1 if (self.entry == "cluster" or self.cluster > 1 or
                                       0 < n_splits <= gqa.SERIAL_MERGE_MAX_SPLITS) else 2
        self.out = torch.empty(self.q.shape, dtype=torch.float32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.how, n_copies = l2_plan(self.kv_step)
        self.caches = [(inp.k_cache, inp.v_cache)]
        if with_copies:
            for _ in range(n_copies - 1):
                self.caches.append((inp.k_cache.clone(), inp.v_cache.clone()))
        self.flush = L2Flush() if self.how == "flush" else None
        self.i = 0

    def call(self, q, sl, pt, out, k, v, status=None, stream=None):
        gqa = self.gqa
        if self.nq > 1:
            gqa.gqa_decode_verify(q, k, v, sl, pt, split_tokens=self.split, max_seqlen=self.max_seqlen,
                                  workspace=self.ws, out=out, status=status, stream=stream)
        elif self.entry == "cluster":
            gqa.gqa_decode(q, k, v, sl, pt, out=out, status=status, stream=stream)
        else:
            gqa.gqa_decode_split(q, k, v, sl, pt, split_tokens=self.split, max_seqlen=self.max_seqlen,
                                 workspace=self.ws, out=out, status=status, stream=stream)

    def step(self):
        k, v = self.caches[self.i % len(self.caches)]
        self.i += 1
        self.call(self.q, self.inp.seqlens, self.inp.page_table, self.out, k, v, status=self.status)

    def decode_only(self):
        """The decode kernel alone (the step without its combine launch)."""
        k, v = self.caches[self.i % len(self.caches)]
        self.i += 1
        if self.nq > 1:  # no two-kernel entry point for verification: the whole step
            self.step()
            return
        self.gqa.gqa_split_partials(self.inp.q, k, v, self.inp.seqlens, self.inp.page_table,
                                    split_tokens=self.split, max_seqlen=self.max_seqlen, workspace=self.ws,
                                    out=self.out, status=self.status)

    def check_status(self):
        torch.cuda.synchronize()
        st = int(self.status.item())
        if st != 0:
            raise RuntimeError("%s: decode reported status %d" % (self.w.name, st))

    def time_steps(self, steps, world):
        """ms per step, max over ranks: back-to-back steps between two events
        (resident or rotating caches), or flush + one event pair per step."""
        stream = torch.cuda.current_stream()
        if self.how != "flush":
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(world)
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(steps):
                self.step()
            ev1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            total = ev0.elapsed_time(ev1)
        else:
            total = sum(self.time_flushed(steps, world, sync=False))
        return max_over_ranks(total, world) / steps

    def time_flushed(self, steps, world, sync=True, fn=None):
        """Per-step ms of `fn` (default: one step), each launch alone after an
        L2 flush, between its own event pair."""
        fn = fn or self.step
        flush = self.flush or L2Flush()
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        if sync:
            barrier(world)
        torch.cuda.synchronize()
        for a, b in evs:
            flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        if sync:
            barrier(world)
        return [a.elapsed_time(b) for a, b in evs]

    def kernel_ms(self, steps, world):
        """The dominant kernel (the decode kernel) alone: mean of isolated
        launches between CUDA events on its stream, L2 flushed first when the
        cache fits in it; for a one-launch step that is the step itself."""
        kern = self.step if self.launches_per_step == 1 else self.decode_only
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(max(steps, 10))]
        flush = None if self.how == "resident" else (self.flush or L2Flush())
        for a, b in evs:
            if flush is not None:
                flush()
            a.record(stream)
            kern()
            b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world)

    def kernel_name(self):
        tc_name = "gqa_verify_tc_kernel"
        if self.nq > 1:
            return "%s (verification, %d rows per KV group%s)" % (
                tc_name if self.tc else "gqa_decode_kernel", self.nq * self.w.r,
                "" if self.launches_per_step == 1 else "; decode + combine timed together")
        if self.tc:
            return "%s (%d rows per KV group)" % (tc_name, self.w.r)
        if self.entry == "split":
            if self.cluster > 1:
                return "gqa_decode_kernel (thread-block clusters of %d, merged in distributed shared memory)" % (
                    self.cluster)
            if self.eff_split == 0:
                return "gqa_decode_kernel (equal-work ranges)"
            return "gqa_decode_kernel (fixed splits%s)" % (", merged in-kernel" if self.launches_per_step == 1 else "")
        return "gqa_decode_kernel (gqa_decode)"

    def plan(self):
        return plan_dict(self.eff_split, self.max_seqlen, self.nq, self.tc, self.entry, self.cluster)

    def free(self):
        self.caches = []
        self.inp = None
        self.ws = None
        self.flush = None


def measure_point(args, name, nq, world, rank, hbm):
    """One per_config entry: the same step timing as the headline, the
    kernel alone, and for caches that fit in L2 the flush-then-event time."""
    case = Case(args, WORKLOADS[name], nq, rank)
    for _ in range(args.warmup):
        case.step()
    case.check_status()
    ms = case.time_steps(args.steps, world)
    kern = case.kernel_ms(args.steps, world)
    case.check_status()
    kv = case.kv_step
    d = {"us_per_step": ms * 1e3, "kv_bytes": kv, "gbs": world * kv / (ms * 1e-3) / 1e9,
         "frac": kv / (ms * 1e-3) / 1e9 / hbm, "kernel_us": kern * 1e3,
         "kernel_frac": kv / (kern * 1e-3) / 1e9 / hbm, "timing": case.how,
         "traffic": recorded_traffic(traffic_key(name, nq)), "plan": case.plan()["decomposition"]}
    if case.how == "rotate":
        flushed = max_over_ranks(statistics.median(case.time_flushed(max(args.steps, 10), world)), world)
        d["us_flushed"] = flushed * 1e3
        d["frac_flushed"] = kv / (flushed * 1e-3) / 1e9 / hbm
    case.free()
    del case
    torch.cuda.empty_cache()
    return d


def sweep_fit(per_config):
    """Does the step time of the group-ratio sweep follow its KV bytes?  A
    least-squares line t = fixed + bytes / bandwidth through the sweep points
    whose cache exceeds twice the L2 (their time is set by streaming the
    cache), and every sweep point's time over that line's value (1.0: on the
    line; above 1: a per-step cost beyond the line's fixed part)."""
    pts = {k: v for k, v in per_config.items() if k.startswith("sweep_g")}
    big = [(v["kv_bytes"], v["us_per_step"]) for v in pts.values() if v["kv_bytes"] > 2 * L2_BYTES]
    if len(big) < 2:
        return None
    n = len(big)
    mx = sum(x for x, _ in big) / n
    my = sum(y for _, y in big) / n
    sxx = sum((x - mx) ** 2 for x, _ in big)
    slope = sum((x - mx) * (y - my) for x, y in big) / sxx  # us per byte
    fixed = my - slope * mx
    return {"fixed_us": fixed, "marginal_gbs": 1e-3 / slope, "fit_points": n,
            "time_over_fit": {k: v["us_per_step"] / (fixed + slope * v["kv_bytes"]) for k, v in pts.items()}}


def main_gpu(args):
    world, rank, local = dist_setup()
    hbm, hbm_kind = peaks()
    nq = args.query_tokens
    case = Case(args, WORKLOADS[args.workload], nq, rank)
    w, inp = case.w, case.inp

    # ---- warm-up
    for _ in range(args.warmup):
        case.step()
    case.check_status()

    if args.profile_only:
        # for a profiler: the warm-up above and K plain steps, nothing else
        for _ in range(args.steps):
            case.step()
        case.check_status()
        if rank == 0:
            print(json.dumps({"profile_only": True, "workload": w.name, "steps": args.steps,
                              "warmup": args.warmup, "plan": case.plan()}), flush=True)
        return 0

    # ---- timed region: K steps, inputs resident in HBM
    clocks = ClockSampler(local)
    with clocks:
        ms_per_step = case.time_steps(args.steps, world)
    timed_samples = len(clocks.samples)
    case.check_status()
    value = world * case.kv_step / (ms_per_step * 1e-3) / 1e9

    # ---- dominant kernel alone (decode kernel), CUDA events on its stream
    kern_ms = case.kernel_ms(args.steps, world)
    achieved = case.kv_step / (kern_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": recorded_traffic(traffic_key(args.workload, nq)),
                "kernel": case.kernel_name(), "peak_kind": hbm_kind,
                "kernel_us": kern_ms * 1e3, "algorithmic_bytes_per_launch": case.kv_step}

    # ---- end to end through the public API with host buffers
    e2e = e2e_leg(args, case, world)
    plan = case.plan()
    launches = case.launches_per_step * args.steps
    cfg = config_dict(w, inp, nq)

    # ---- CPU baseline: the oracle on host cores (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs, dt, threads, desc = oracle_time(inp, target_s=args.oracle_seconds if args.oracle_seconds > 0 else 15.0,
                                             q_verify=None if nq == 1 else case.q)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": desc + "; %.1f s of CPU time" % dt}
    # ---- every workload, measured the same way in this process
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            per_config[name] = measure_point(args, name, 1, world, rank, hbm)
        for name, n in PER_CONFIG_VERIFY:
            per_config[traffic_key(name, n)] = measure_point(args, name, n, world, rank, hbm)

    # ---- last: the headline step repeated for >= 1 s, so that the clock
    # record has samples even when the timed region is a few milliseconds (at
    # the end, so that the heat it leaves behind touches no other measurement)
    with clocks:
        t_end = time.perf_counter() + max(1.0, args.clock_window)
        n_win = 0
        while time.perf_counter() < t_end:
            for _ in range(32):
                case.step()
            n_win += 32
            torch.cuda.synchronize()
    case.check_status()
    case.free()
    del case
    torch.cuda.empty_cache()

    if rank == 0:
        clk = clocks.summary()
        clk["timed_region_samples"] = timed_samples
        clk["window"] = "timed region + %d more steps over >= %.1f s" % (n_win, max(1.0, args.clock_window))
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "plan": plan,
            "frac_of_peak_hbm": value / world / hbm, "peak_hbm_gbs": hbm, "peak_kind": hbm_kind,
            "frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
            "entry": "gqa_decode_verify" if nq > 1 else "gqa_decode_split" if args.entry == "split" else "gqa_decode",
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk, "per_config": per_config,
            "sweep_fit": sweep_fit(per_config),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def e2e_leg(args, case, world):
    """Same metric through the public call with host buffers: each step copies the
    step's inputs (q, lengths, page table) from pinned host memory, runs the
    decode and reads the result back into pinned host memory.  The KV cache is
    the decode state and stays resident in HBM (copies of it read in turn when
    it fits in L2, as in the device-timed steps).

    Steps are pipelined the way a serving loop would run them: two sets of
    device input/output buffers, the copies on their own streams (the copy
    engines) and the decode on a compute stream, so step i+1's inputs travel
    and step i-1's result returns while step i decodes.  Events order every
    buffer reuse."""
    inp, q = case.inp, case.q
    h_q = q.cpu().pin_memory()
    h_sl = inp.seqlens.cpu().pin_memory()
    h_pt = None if inp.page_table is None else inp.page_table.cpu().pin_memory()
    h_out = [torch.empty(q.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    d_q = [torch.empty_like(q) for _ in range(2)]
    d_sl = [torch.empty_like(inp.seqlens) for _ in range(2)]
    d_pt = [None if h_pt is None else torch.empty_like(inp.page_table) for _ in range(2)]
    d_out = [torch.empty(q.shape, dtype=torch.float32, device="cuda") for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in comp_done + out_done:
        e.record(torch.cuda.current_stream())
    h2d = h_q.numel() * h_q.element_size() + h_sl.numel() * 4 + (0 if h_pt is None else h_pt.numel() * 4)
    d2h = h_out[0].numel() * 4

    def step(i):
        k = i % 2
        kc, vc = case.caches[i % len(case.caches)]
        with torch.cuda.stream(s_in):      # inputs of step i (buffer k is free once step i-2 decoded)
            s_in.wait_event(comp_done[k])
            d_q[k].copy_(h_q, non_blocking=True)
            d_sl[k].copy_(h_sl, non_blocking=True)
            if h_pt is not None:
                d_pt[k].copy_(h_pt, non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_comp):    # decode of step i (its output buffer is free once read back)
            s_comp.wait_event(in_done[k])
            s_comp.wait_event(out_done[k])
            case.call(d_q[k], d_sl[k], d_pt[k], d_out[k], kc, vc, stream=s_comp)
            comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):     # result of step i back to the host
            s_out.wait_event(comp_done[k])
            h_out[k].copy_(d_out[k], non_blocking=True)
            out_done[k].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    n = max(10, min(args.steps, 200))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(s_in)
    for i in range(n):
        step(i)
    s_in.wait_stream(s_out)
    ev1.record(s_in)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / n, world)
    return {"value": world * case.kv_step / (ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "note": "every step: q, lengths (and page table) H2D from pinned memory, decode, output D2H to "
                    "pinned memory; steps pipelined over copy and compute streams; KV cache resident"}


def main(argv=None):
    ap = argparse.ArgumentParser(description="GQA decode benchmark (B200)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="ragged")
    ap.add_argument("--entry", choices=["split", "cluster"], default="split")
    ap.add_argument("--split-tokens", type=int, default=-1,
                    help="-1: the library's plan; 0: the library's automatic choice at run time (the same); "
                         "> 0: fixed splits of that many tokens")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="measure the headline workload only")
    ap.add_argument("--profile-only", action="store_true",
                    help="run the warm-up and --steps plain steps of the workload and exit (for ncu); no timing")
    ap.add_argument("--clock-window", type=float, default=1.0,
                    help="seconds of repeated steps sampled for clocks after the timed region (>= 1)")
    ap.add_argument("--oracle-seconds", type=float, default=0.0,
                    help="CPU seconds of oracle work per timed sample (0: 15 s for cpu_baseline; the reference "
                         "arm spreads about two minutes over its steps)")
    ap.add_argument("--query-tokens", type=int, default=1,
                    help="query tokens per sequence (> 1: a verification step through gqa_decode_verify)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (use --impl reference for the CPU oracle)")
    return main_gpu(args)


if __name__ == "__main__":
    raise SystemExit(main())
