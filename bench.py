"""Benchmark of paged split-KV decode attention on B200.

One step = one decode-attention call (split kernel + combine kernel) over one
batch of synthetic decode queries against a paged bf16 KV cache, through the
C-ABI library.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b|long|ragged|gqa32|gqa80|tiny|...]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on the host cores

Metric: achieved HBM bandwidth over algorithmic bytes (KV bytes that must be read
+ q bytes + out bytes) per call, in GB/s, with the µs/call beside it.  Inputs
are resident in HBM before the timed region.  Two independent instances of the
workload (different seeds, each larger than L2 for the large workloads) are used
in turn, so every call reads KV that the previous call did not touch.

Several GPUs (one process each, under torchrun): every rank runs its own batch
of the same shape (independent decode problems, no collective on the data path);
the value is the bytes of all ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attention achieved HBM GB/s (algorithmic KV+q+out bytes per call / time)"
UNIT = "GB/s"
DEFAULT_STEPS = {"llama8b": 200, "long": 100, "ragged": 50, "tiny": 200, "llama8b_contig": 200,
                 "long_contig": 100, "gqa32": 200, "gqa80": 100}
DEFAULT_REFERENCE_STEPS = 20
# measured beside the headline decode workload, in the same run: the other configurations with a
# 70% target or a reported number, and the multi-query shapes of the tensor-core decode kernel
PER_CONFIG = ("long", "ragged", "gqa32", "gqa80")
CSRC = os.path.join(ROOT, "decode_attention_paged_split_b200", "csrc")
GEMV_METRIC = "decode projection GEMV achieved HBM GB/s (algorithmic W+x+y bytes per call / time)"
GEMV_WORKLOADS = [f"gemv_{layer}_m{m}" for layer in workloads.GEMV_SHAPES for m in (1, 3, 8)]
PREFILL_METRIC = "paged multi-query (prefill chunk) attention achieved TFLOP/s and HBM GB/s"
PREFILL_WORKLOADS = ["prefill_llama8b_chunk"]
SWEEP_WORKLOADS = ["sweep"]
SWEEP_METRIC = "paged decode attention us/call with a cold L2, head-dim / GQA sweep (B=4, L ~ U{1..1024})"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "split_kernel_traffic.json")
PREFILL_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "prefill_tc2_kernel_traffic.json")
GEMV_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_kernel_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=sorted(workloads.NAMED) + GEMV_WORKLOADS + PREFILL_WORKLOADS + SWEEP_WORKLOADS,
                   default="llama8b",
                   help="a decode-attention workload, or gemv_<layer>_m<M> for the decode projection")
    p.add_argument("--num-splits", type=int, default=0, help="0 = auto (the default launch configuration)")
    p.add_argument("--no-host-lens", action="store_true",
                   help="decode: do not pass the host copy of the lengths as the planning hint")
    p.add_argument("--prefill-kernel", choices=["auto", "mma_sync", "tcgen05"], default="auto",
                   help="kernel of the prefill workload (auto = what attn_paged_prefill picks)")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    p.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi clocks")
    p.add_argument("--no-per-config", action="store_true",
                   help="decode: do not also measure the long-context and ragged configurations")
    p.add_argument("--instances", type=int, default=2,
                   help="independent copies of the workload used in turn (1 keeps the device footprint small "
                        "for profiling; every large workload is bigger than L2 on its own)")
    p.add_argument("--min-seconds", type=float, default=2.0,
                   help="repeat the timed K-step region until about this long (at least 3 repetitions)")
    a = p.parse_args(argv)
    a.steps_given = a.steps is not None
    if a.steps is None:
        a.steps = (DEFAULT_REFERENCE_STEPS if a.impl == "reference" else DEFAULT_STEPS.get(a.workload, 2000))
    if a.instances < 1:
        p.error("--instances must be >= 1")
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


# ---------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def init_group(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- inputs
def make_instances(name: str, rank: int, count: int = 2):
    """`count` instances of the named workload with the same structure (lengths, page
    table) and independent values; the seed of the values differs per rank and instance."""
    gen = workloads.NAMED[name]
    base = {"tiny": 1234, "llama8b": 8, "long": 131072, "ragged": 4262, "llama8b_contig": 8,
            "long_contig": 131072, "gqa32": 32, "gqa80": 80, "hd32": 77, "hd64": 77, "hd256": 77}[name]
    return [gen(seed=base, value_seed=base + 1000003 * rank + i) for i in range(count)]


def _align(n: int, a: int) -> int:
    return (n + a - 1) // a * a


class Resident:
    """A workload resident on the device: KV cache, a packed [q | page_table | seq_lens]
    buffer (so the end-to-end leg moves a step's inputs in one copy), out, workspace and
    the prepared library call."""

    def __init__(self, w, device, num_splits, apd, host_hint=True):
        self.w = w
        self.k = w.k_cache.contiguous().to(device)
        self.v = w.v_cache.contiguous().to(device)
        qb, pb, sb = w.q.numel() * 2, w.page_table.numel() * 4, w.seq_lens.numel() * 4
        self.offsets = (0, _align(qb, 256), _align(qb, 256) + _align(pb, 256))
        self.packed_bytes = self.offsets[2] + sb
        host = torch.zeros(self.packed_bytes, dtype=torch.uint8)
        self._views(host)[0].copy_(w.q)
        self._views(host)[1].copy_(w.page_table)
        self._views(host)[2].copy_(w.seq_lens)
        self.host_packed = host.pin_memory()
        self.dev_packed = self.host_packed.to(device)
        self.q, self.page_table, self.seq_lens = self._views(self.dev_packed)
        self.out = torch.empty_like(self.q)
        self.host_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.num_splits = num_splits
        self.ws = apd.alloc_workspace(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, num_splits,
                                      device=device)
        self.contig = w.meta.get("kv_policy") == "contig"
        # a serving loop knows its lengths on the host: they go along as the planning hint
        self.host_lens = w.seq_lens.clone() if host_hint else None
        self.call = apd.DecodeCall(self.q, self.k, self.v, None if self.contig else self.page_table, self.seq_lens,
                                   self.out, w.scale, num_splits, self.ws, host_seq_lens=self.host_lens)
        self.bytes = w.algorithmic_bytes()

    def _views(self, buf):
        w = self.w
        o = self.offsets
        q = buf[o[0]:o[0] + w.q.numel() * 2].view(torch.bfloat16).view(w.q.shape)
        pt = buf[o[1]:o[1] + w.page_table.numel() * 4].view(torch.int32).view(w.page_table.shape)
        sl = buf[o[2]:o[2] + w.seq_lens.numel() * 4].view(torch.int32).view(w.seq_lens.shape)
        return q, pt, sl


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, enabled: bool = True):
        self.proc = None
        self.path = None
        if not enabled:
            return
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        import tempfile

        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, r in rows:
            for n, v in zip(names[1:], r[1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- measurement legs
DECODE_KERNEL_SOURCES = ("apd_kernels.cuh", "apd_ptx.cuh")  # the split and combine kernels' device code
# the tensor-core multi-query decode kernel (plan mode 3) and the pieces it is built from
DECODE_TC_KERNEL_SOURCES = ("apd_decode_tc.cuh", "apd_kernels.cuh", "apd_prefill_tc.cuh", "apd_ptx.cuh")
PLAN_MODE_NAMES = {0: "balanced + combine", 1: "fixed splits", 2: "one CTA per unit, single kernel",
                   3: "tensor-core multi-query"}


def decode_kernel_of(plan) -> tuple:
    """The dominant kernel of a decode plan and the headers its device code comes from."""
    if plan.mode == 3:
        return "decode_mq_tc_kernel", DECODE_TC_KERNEL_SOURCES
    if plan.mode in (1, 2):
        return "unit_kernel", DECODE_KERNEL_SOURCES
    return "split_kernel", DECODE_KERNEL_SOURCES


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed, so that editing a comment
    does not change the hash of the code."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha(sources=DECODE_KERNEL_SOURCES) -> str:
    """Hash of the decode kernels' device code (the headers they are compiled from, comments
    and whitespace ignored); the host-side API file and the other kernels' headers are not
    included."""
    h = hashlib.sha256()
    for name in sorted(sources):
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


PREFILL_KERNEL_SOURCES = ("apd_kernels.cuh", "apd_prefill.cuh", "apd_prefill_tc.cuh", "apd_ptx.cuh")
GEMV_KERNEL_SOURCES = ("apd_gemv.cuh", "apd_kernels.cuh", "apd_ptx.cuh")


def committed_traffic(workload: str, path=None, sources=DECODE_KERNEL_SOURCES):
    """dram read+write bytes per launch of the dominant kernel from a committed ncu capture
    (default: the decode split kernel), or None when no capture of this workload is
    recorded or the kernel's device code changed since.  The file holds one record or a
    list of records (one per workload)."""
    try:
        with open(path or TRAFFIC_FILE) as f:
            recs = json.load(f)
    except (OSError, ValueError):
        return None
    sha = kernel_source_sha(sources)
    for t in recs if isinstance(recs, list) else [recs]:
        if t.get("kernel_source_sha") == sha and t.get("workload") == workload:
            return t.get("dram_bytes_per_launch")
    return None


def time_steps(insts, stream, steps, split_events=False):
    """Eager calls rotating over the instances; returns (elapsed_s, mean split-kernel s or None)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    per = []
    if split_events:
        per = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start.record(stream)
    for i in range(steps):
        inst = insts[i % len(insts)]
        if split_events:
            b, m = per[i]
            b.record(stream)
            inst.call(stream, split_done_event=m)
        else:
            inst.call(stream)
    end.record(stream)
    end.synchronize()
    elapsed = start.elapsed_time(end) / 1e3
    split = None
    if split_events:
        split = sum(b.elapsed_time(m) for b, m in per) / 1e3 / steps
    return elapsed, split


GRAPH_CHUNK = 100


def graph_split_times(insts, stream, replays):
    """Split-kernel duration inside CUDA-graph replays: a graph of GRAPH_CHUNK calls (rotating
    over the instances) with an external event recorded before each call and the call's
    split_done_event right after its split kernel (both become event-record nodes), replayed
    `replays` times.  The event between the kernels turns off the programmatic overlap of
    those two launches, so this is the kernel's own start-to-end time.  Returns the mean in s."""
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(GRAPH_CHUNK)]
    for b, m in ev:  # create the events before capture
        b.record(stream)
        m.record(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i, (b, m) in enumerate(ev):
                b.record(stream)
                insts[i % len(insts)].call(stream, split_done_event=m)
    g.replay()
    torch.cuda.synchronize()
    tot, n = 0.0, 0
    for _ in range(replays):
        g.replay()
        torch.cuda.synchronize()
        tot += sum(b.elapsed_time(m) for b, m in ev) / 1e3
        n += len(ev)
    del g
    return tot / n


class GraphSteps:
    """Exactly `steps` consecutive calls `call(i, stream)` (i = 0 .. steps-1; the calls repeat
    with `period`, e.g. instances used in turn) captured as CUDA graphs of up to GRAPH_CHUNK
    calls, with event-record nodes before the first call and after the last: the interval
    between them is the calls' time on the device, without the host's launch of the graphs.
    Longer runs chain a first graph (with the start event), a middle graph replayed as often
    as needed and a last graph (with the end event)."""

    def __init__(self, call, stream, steps, period=1):
        self.start = torch.cuda.Event(enable_timing=True, external=True)
        self.end = torch.cuda.Event(enable_timing=True, external=True)
        self.start.record(stream)  # create the events before capture
        self.end.record(stream)
        torch.cuda.synchronize()
        # a graph that is replayed more than once holds a whole number of periods
        chunk = max(period, GRAPH_CHUNK - GRAPH_CHUNK % period)
        if steps <= chunk:
            self.plan = [(self._capture(call, stream, steps, True, True), 1)]
        else:
            mid_reps, last = divmod(steps - chunk, chunk)
            if last == 0:
                mid_reps, last = mid_reps - 1, chunk
            self.plan = [(self._capture(call, stream, chunk, True, False), 1)]
            if mid_reps:
                self.plan.append((self._capture(call, stream, chunk, False, False), mid_reps))
            self.plan.append((self._capture(call, stream, last, False, True), 1))
        self.steps = steps

    def _capture(self, call, stream, count, with_start, with_end):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                if with_start:
                    self.start.record(stream)
                for i in range(count):
                    call(i, stream)
                if with_end:
                    self.end.record(stream)
        return g

    def run(self, stream):
        with torch.cuda.stream(stream):
            for g, reps in self.plan:
                for _ in range(reps):
                    g.replay()
        self.end.synchronize()
        return self.start.elapsed_time(self.end) / 1e3

    def release(self):
        self.plan = []


def timed_reps(run, dist, device, min_seconds: float, max_reps: int = 20000):
    """Repetitions of one timed region (`run()` returns its device seconds), each bracketed by
    a barrier and a device synchronisation: one untimed, then as many as last about
    min_seconds (at least 3; the same count on every rank).  Returns the per-repetition
    seconds, each the max over ranks."""
    run()
    t1 = run()
    reps = max(3, min(max_reps, math.ceil(min_seconds / max(t1, 1e-9))))
    reps = int(max_over_ranks(float(reps), dist, device))
    times = []
    for _ in range(reps):
        barrier(dist, device)
        if device.type == "cuda":
            torch.cuda.synchronize(device)
        times.append(run())
    if dist is not None:
        t = torch.tensor(times, dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        times = t.cpu().tolist()
    return times


def timing_summary(times, steps):
    med = statistics.median(times)
    return {"reps": len(times), "steps_per_rep": steps, "median_us_per_call": med / steps * 1e6,
            "min_us_per_call": min(times) / steps * 1e6, "max_us_per_call": max(times) / steps * 1e6,
            "timed_s": sum(times),
            "stat": "median over repetitions of the K-call region (each the max over ranks)"}


def e2e_steps(insts, stream, steps):
    """End to end through the public API with host buffers.  Per step: one pinned-host
    -> device copy of the packed [q | page_table | seq_lens] inputs, the call, and one
    device -> pinned-host copy of out.  Copies run on two copy streams so that step
    i+1's inputs and step i-1's output move while step i computes; events keep every
    buffer's reuse ordered (instance j is used by steps j, j+2, ...).
    Returns (elapsed_s, h2d bytes, d2h bytes) per step."""
    dev = insts[0].q.device
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(insts)
    computed = [torch.cuda.Event() for _ in range(n)]
    out_copied = [torch.cuda.Event() for _ in range(n)]
    in_ready = [torch.cuda.Event() for _ in range(n)]
    used = [False] * n
    h2d = insts[0].packed_bytes
    d2h = insts[0].out.nbytes
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    for i in range(steps):
        j = i % n
        inst = insts[j]
        with torch.cuda.stream(h2d_s):
            if used[j]:
                h2d_s.wait_event(computed[j])  # the previous call on these buffers has read its inputs
            inst.dev_packed.copy_(inst.host_packed, non_blocking=True)
            in_ready[j].record(h2d_s)
        stream.wait_event(in_ready[j])
        if used[j]:
            stream.wait_event(out_copied[j])  # the previous output of these buffers has left the device
        inst.call(stream)
        computed[j].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(computed[j])
            inst.host_out.copy_(inst.out, non_blocking=True)
            out_copied[j].record(d2h_s)
        used[j] = True
    stream.wait_stream(d2h_s)
    stream.wait_stream(h2d_s)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3, h2d, d2h


def oracle_baseline(w, min_seconds: float = 10.0, max_calls: int = 50, single_core_seconds: float = 5.0):
    """The fp64 CPU oracle on the whole workload, as it stands: on all host threads (OpenMP
    over query rows), repeated until about min_seconds, then on one thread for about
    single_core_seconds."""
    import oracle

    def timed(nthreads, seconds, cap):
        calls, t0 = 0, time.perf_counter()
        while True:
            oracle.paged_decode(w, nthreads=nthreads)
            calls += 1
            el = time.perf_counter() - t0
            if el >= seconds or calls >= cap:
                return calls, el

    oracle.paged_decode(w)  # loads the library and faults in the pages once
    threads = oracle.max_threads()
    calls, el = timed(0, min_seconds, max_calls)
    calls1, el1 = timed(1, single_core_seconds, max_calls)
    rows = w.batch * w.num_q_heads
    return {"value": w.algorithmic_bytes() * calls / el / 1e9, "unit": UNIT, "cores": threads,
            "kind": "oracle", "nproc": os.cpu_count(), "omp_threads": threads,
            "sample": f"the whole {w.name} workload (all {rows} query rows), {calls} calls, {el:.1f} s, fp64, "
                      f"OpenMP over rows on {threads} threads",
            "single_core": {"value": w.algorithmic_bytes() * calls1 / el1 / 1e9, "unit": UNIT, "cores": 1,
                            "sample": f"the whole workload, {calls1} calls, {el1:.1f} s, one thread"}}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------- arms
def run_reference(a):
    """The reference arm: the fp64 CPU oracle on all host threads, each step the whole
    workload (the cpu_baseline leg's sample), or an equal share of its query rows when K
    whole calls would not end within a few minutes."""
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    import oracle

    w = make_instances(a.workload, 0, 1)[0]
    B, Hq = w.batch, w.num_q_heads
    total_bytes = w.algorithmic_bytes()
    oracle.paged_decode(w)  # loads the library and faults in the pages once
    t0 = time.perf_counter()
    oracle.paged_decode(w)
    t_whole = time.perf_counter() - t0
    budget = 150.0  # seconds for the warm-up and timed steps together
    rows_all = [(b, h) for b in range(B) for h in range(Hq)]
    per_row = w.seq_lens.to(torch.float64)
    row_weight = [float(per_row[b]) for b, _ in rows_all]
    total_weight = max(sum(row_weight), 1.0)
    if t_whole * (a.steps + a.warmup) <= budget:
        nrows = len(rows_all)
        sample = f"each step: the whole {w.name} workload (all {nrows} query rows)"
    else:
        nrows = max(1, int(len(rows_all) * budget / (t_whole * (a.steps + a.warmup))))
        sample = (f"each step: {nrows} of the {len(rows_all)} query rows of {w.name} (a window rotating over "
                  f"them; bytes counted in proportion to the rows' tokens)")

    def step(i):
        if nrows == len(rows_all):
            oracle.paged_decode(w)
            return float(total_bytes)
        lo = (i * nrows) % len(rows_all)
        idx = [(lo + j) % len(rows_all) for j in range(nrows)]
        oracle.paged_decode_rows(w, [rows_all[j] for j in idx])
        return total_bytes * sum(row_weight[j] for j in idx) / total_weight

    for i in range(a.warmup):
        step(i)
    t0 = time.perf_counter()
    done = 0.0
    for i in range(a.steps):
        done += step(a.warmup + i)
    el = time.perf_counter() - t0
    value = done / el / 1e9
    cores = oracle.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": el / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, a),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "nproc": os.cpu_count(),
                         "omp_threads": cores, "sample": f"{sample}, fp64 CPU oracle on {cores} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, a):
    n = getattr(a, "instances", 2)
    return {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "page_size": w.page_size, "kv_tokens": w.kv_tokens(),
            "num_splits": a.num_splits, "layout": w.layout, "kv_policy": w.meta.get("kv_policy", "paged"),
            "l2": (f"{n} independent instances used in turn (each call reads KV the previous call did not touch); "
                   "large workloads are each larger than L2") if n > 1 else
                  "one instance (large workloads are larger than L2 on their own)",
            "algorithmic_bytes_per_call": w.algorithmic_bytes(),
            "host_seq_lens_hint": not getattr(a, "no_host_lens", False),
            "launch": f"CUDA graphs of up to {GRAPH_CHUNK} consecutive calls with event-record nodes around "
                      f"the K calls; the K-call region repeated for about {getattr(a, 'min_seconds', 2.0):g} s"}


def measure_decode(a, name, apd, device, dist, rank, local, min_seconds, want_clocks, extras=False):
    """Times `a.steps` consecutive calls of a decode workload (graph replays, repeated, see
    timed_reps) on this rank's instances.  Returns a dict of the numbers, and the instances
    when `extras` (for the headline's eager, end-to-end and oracle legs)."""
    insts = [Resident(w, device, a.num_splits, apd, host_hint=not a.no_host_lens)
             for w in make_instances(name, rank, a.instances)]
    w0 = insts[0].w
    max_len = w0.k_cache.shape[1] if insts[0].contig else w0.page_table.shape[1] * w0.page_size
    plan = apd.query_plan(w0.batch, w0.num_q_heads, w0.num_kv_heads, w0.head_dim, a.num_splits,
                          host_seq_lens=insts[0].host_lens, max_seq_len=max_len)
    launches_per_step = 1 + (1 if plan.combine_ctas > 0 else 0)
    kname, ksources = decode_kernel_of(plan)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)

    time_steps(insts, stream, a.warmup)  # warm-up (eager)
    graphs = GraphSteps(lambda i, st: insts[i % len(insts)].call(st), stream, a.steps, period=len(insts))
    clocks = ClockSampler(local, enabled=want_clocks)
    times = timed_reps(lambda: graphs.run(stream), dist, device, min_seconds)
    clock_info = clocks.stop()
    graphs.release()
    t_med = statistics.median(times)
    bytes_rank = sum(insts[i % len(insts)].bytes for i in range(a.steps))
    bytes_all = sum_over_ranks(float(bytes_rank), dist, device)
    if launches_per_step == 1:
        # The call is this one kernel: its average launch duration is the timed region over
        # the launches in it.
        split_s = t_med / a.steps
        kernel_timing = ("the call is this one kernel: the median K-call region (event-record nodes around "
                         "the graph-replayed calls) over the K launches in it")
    else:
        barrier(dist, device)
        torch.cuda.synchronize(device)
        try:
            split_s = graph_split_times(insts, stream, replays=10)
        except RuntimeError as err:  # event-record nodes unavailable: fall back to eager event pairs
            print(f"graph split timing unavailable ({err}); using eager event pairs", file=sys.stderr)
            _, split_s = time_steps(insts, stream, a.steps, split_events=True)
        split_s = max_over_ranks(split_s, dist, device)
        kernel_timing = (f"CUDA events recorded around each {kname} launch inside replays of a "
                         f"{GRAPH_CHUNK}-call graph (event-record nodes)")
    peak, peak_src = peaks()
    mean_bytes = bytes_rank / a.steps
    achieved = mean_bytes / split_s / 1e9
    res = {
        "workload": w0.name, "us_per_call": t_med / a.steps * 1e6, "value": bytes_all / t_med / 1e9,
        "timing": timing_summary(times, a.steps),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                     "traffic": committed_traffic(name, sources=ksources), "peak_source": peak_src, "kernel": kname,
                     "kernel_us": split_s * 1e6, "kernel_timing": kernel_timing,
                     "call_frac_of_peak": bytes_all / t_med / 1e9 / max(1, (dist.get_world_size() if dist else 1))
                     / peak},
        "gpu_launches": launches_per_step * a.steps * len(times),
        "clocks": clock_info,
        "plan": {"mode": plan.mode,
                 "mode_name": PLAN_MODE_NAMES.get(plan.mode, str(plan.mode)),
                 "workers": plan.num_workers, "ctas": plan.grid_ctas, "warps_per_cta": plan.warps_per_cta,
                 "stages": plan.stages, "smem": plan.smem_bytes, "shared_kv_ring": bool(plan.shared_kv_ring),
                 "combine_ctas": plan.combine_ctas},
        "config": config_of(w0, a),
    }
    if extras:
        res.update(_insts=insts, _stream=stream, _t_med=t_med, _bytes_all=bytes_all)
    else:
        del insts
    return res


def run_ours(a):
    world, rank, local = dist_env()
    if a.gpus != world and world > 1:
        print(f"--gpus {a.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2
    if a.gpus > 1 and world == 1:
        print("--gpus N>1 needs torchrun (one process per GPU)", file=sys.stderr)
        return 2
    if not torch.cuda.is_available():
        print("no CUDA device", file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group(world, "nccl")
    import decode_attention_paged_split_b200 as apd

    want_clocks = not a.no_clocks and rank == 0
    head = measure_decode(a, a.workload, apd, device, dist, rank, local, a.min_seconds, want_clocks, extras=True)
    insts, stream, t_med, bytes_all = head["_insts"], head["_stream"], head["_t_med"], head["_bytes_all"]

    # the same steps launched eagerly from Python, for reference
    barrier(dist, device)
    torch.cuda.synchronize(device)
    eager_el, _ = time_steps(insts, stream, a.steps)
    eager_max = max_over_ranks(eager_el, dist, device)

    # end to end through host buffers
    e2e = None
    if not a.no_e2e:
        time_steps(insts, stream, 3)
        barrier(dist, device)
        torch.cuda.synchronize(device)
        e_el, h2d, d2h = e2e_steps(insts, stream, a.steps)
        torch.cuda.synchronize(device)
        e_max = max_over_ranks(e_el, dist, device)
        e2e = {"value": bytes_all / e_max / 1e9, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_max / a.steps * 1e3,
               "how": "per step, eager through the public Python API: one pinned-host->device copy of the "
                      "packed q|page_table|seq_lens, the call, one device->pinned-host copy of out; copies on "
                      "two copy streams overlap the neighbouring steps' compute"}
    w0 = insts[0].w
    del insts, head["_insts"]
    torch.cuda.empty_cache()

    # the other configurations with a target or a reported number, in the same run
    per_config = {}
    if a.workload == "llama8b" and not a.no_per_config:
        for name in PER_CONFIG:
            r = measure_decode(a, name, apd, device, dist, rank, local, max(0.5, a.min_seconds / 2), want_clocks)
            per_config[r["workload"]] = {k2: r[k2] for k2 in ("us_per_call", "value", "timing", "roofline", "clocks",
                                                             "plan", "gpu_launches")}
            per_config[r["workload"]]["unit"] = UNIT
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = oracle_baseline(w0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": t_med / a.steps * 1e3, "us_per_call": head["us_per_call"],
            "eager_us_per_call": eager_max / a.steps * 1e6,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": head["config"], "timing": head["timing"],
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "plan": head["plan"],
        }
        if per_config:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- decode projection (GEMV)
def gemv_spec(name: str):
    layer, m = name[len("gemv_"):].rsplit("_m", 1)
    return layer, int(m)


def run_gemv(a):
    """The decode projection y = x W^T on one GPU: CUDA-graph replays of the call,
    rotating over enough weight copies that every call reads weights from HBM."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        print("no CUDA device", file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group(world, "nccl")
    import decode_attention_paged_split_b200 as apd

    layer, M = gemv_spec(a.workload)
    N, K = workloads.GEMV_SHAPES[layer]
    case = workloads.gemv_named(layer, M, value_seed=7 + 1000003 * rank)
    copies = max(2, -(-400_000_000 // (N * K * 2)))
    x = case.x.to(device)
    ws = torch.zeros(apd.gemv_workspace_size(M, N, K), dtype=torch.uint8, device=device)
    ys = [torch.empty(M, N, dtype=torch.bfloat16, device=device) for _ in range(copies)]
    wdev = case.w.to(device)
    weights = [wdev] + [wdev.clone() for _ in range(copies - 1)]
    stream = torch.cuda.Stream(device)
    per_call = case.algorithmic_bytes()

    def call(i, st):
        apd.gemv(x, weights[i % copies], ys[i % copies], ws, stream=st)

    for i in range(a.warmup):
        call(i, stream)
    torch.cuda.synchronize(device)
    graphs = GraphSteps(call, stream, a.steps, period=copies)
    clocks = ClockSampler(local, enabled=not a.no_clocks and rank == 0)
    times = timed_reps(lambda: graphs.run(stream), dist, device, a.min_seconds)
    clock_info = clocks.stop()
    graphs.release()
    t_max = statistics.median(times)
    bytes_all = sum_over_ranks(float(per_call * a.steps), dist, device)
    value = bytes_all / t_max / 1e9

    e2e = None
    if not a.no_e2e:
        # per step: x in (pinned host -> device), the call, y out (device -> pinned host); the copies run on
        # two copy streams so they overlap the neighbouring steps' compute; buffers rotate over the copies
        hx = case.x.pin_memory()
        hys = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(copies)]
        xs = [x] + [x.clone() for _ in range(copies - 1)]
        h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
        computed = [torch.cuda.Event() for _ in range(copies)]
        copied = [torch.cuda.Event() for _ in range(copies)]
        ready = [torch.cuda.Event() for _ in range(copies)]
        used = [False] * copies
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d_s.wait_stream(stream)
        d2h_s.wait_stream(stream)
        for i in range(a.steps):
            j = i % copies
            with torch.cuda.stream(h2d_s):
                if used[j]:
                    h2d_s.wait_event(computed[j])
                xs[j].copy_(hx, non_blocking=True)
                ready[j].record(h2d_s)
            stream.wait_event(ready[j])
            if used[j]:
                stream.wait_event(copied[j])
            apd.gemv(xs[j], weights[j], ys[j], ws, stream=stream)
            computed[j].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(computed[j])
                hys[j].copy_(ys[j], non_blocking=True)
                copied[j].record(d2h_s)
            used[j] = True
        stream.wait_stream(d2h_s)
        stream.wait_stream(h2d_s)
        e1.record(stream)
        e1.synchronize()
        e_max = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device)
        e2e = {"value": bytes_all / e_max / 1e9, "unit": UNIT, "h2d_bytes_per_step": x.nbytes,
               "d2h_bytes_per_step": ys[0].nbytes, "ms_per_step": e_max / a.steps * 1e3,
               "how": "per step, eager through the public Python API: pinned-host->device copy of x, the call, "
                      "device->pinned-host copy of y (weights resident); copies on two copy streams overlap the "
                      "neighbouring steps' compute"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import oracle

        oracle.gemv(case.x, case.w)
        t0, calls = time.perf_counter(), 0
        while time.perf_counter() - t0 < 10.0 and calls < 200:
            oracle.gemv(case.x, case.w)
            calls += 1
        el_cpu = time.perf_counter() - t0
        cpu = {"value": per_call * calls / el_cpu / 1e9, "unit": UNIT, "cores": oracle.max_threads(),
               "kind": "oracle", "sample": f"the whole {case.name} product, {calls} calls, {el_cpu:.1f} s, fp64"}

    if rank == 0:
        peak, peak_src = peaks()
        gplan = apd.gemv_query_plan(M, N, K)
        us = t_max / a.steps * 1e6
        line = {
            "metric": GEMV_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": us / 1e3, "us_per_call": us, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": case.name, "M": M, "N": N, "K": K, "algorithmic_bytes_per_call": per_call,
                       "l2": f"{copies} weight copies used in turn ({copies * N * K * 2 / 1e6:.0f} MB > L2)",
                       "launch": f"CUDA graphs of up to {GRAPH_CHUNK} consecutive calls with event-record nodes "
                                 f"around the K calls; the K-call region repeated for about {a.min_seconds:g} s"},
            "roofline": {"bound": "hbm", "achieved": per_call / (t_max / a.steps) / 1e9, "peak": peak, "unit": UNIT,
                         "frac": per_call / (t_max / a.steps) / 1e9 / peak,
                         "traffic": committed_traffic(case.name, GEMV_TRAFFIC_FILE, GEMV_KERNEL_SOURCES),
                         "peak_source": peak_src,
                         "kernel": "gemv_kernel + gemv_sum_kernel (whole call)" if gplan["sum_ctas"]
                         else "gemv_kernel (the whole call)"},
            "timing": timing_summary(times, a.steps),
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": (2 if gplan["sum_ctas"] else 1) * a.steps * len(times),
            "clocks": clock_info, "plan": gplan,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- multi-query (prefill chunk)
def peak_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, ValueError, KeyError):
        return 1590.0, "fallback"


class PrefillInst:
    """One prefill-chunk instance on the device.  q, page_table and seq_lens are views into
    one packed device buffer (with a pinned host twin) so the end-to-end leg moves the
    step's inputs in one copy; the KV cache stays resident."""

    def __init__(self, w, device, kernel):
        import decode_attention_paged_split_b200 as apd

        self.apd, self.w, self.kernel = apd, w, kernel
        qb, ptb, slb = w.q.numel() * 2, w.page_table.numel() * 4, w.seq_lens.numel() * 4
        off_pt = (qb + 15) // 16 * 16
        off_sl = (off_pt + ptb + 15) // 16 * 16
        self.packed_bytes = off_sl + slb

        def views(buf):
            return (buf[:qb].view(torch.bfloat16).view(w.q.shape),
                    buf[off_pt:off_pt + ptb].view(torch.int32).view(w.page_table.shape),
                    buf[off_sl:off_sl + slb].view(torch.int32))

        self.host_packed = torch.empty(self.packed_bytes, dtype=torch.uint8, pin_memory=True)
        for dst, src in zip(views(self.host_packed), (w.q, w.page_table, w.seq_lens)):
            dst.copy_(src)
        self.dev_packed = self.host_packed.to(device)
        self.q, self.pt, self.sl = views(self.dev_packed)
        self.k, self.v = w.k_cache.contiguous().to(device), w.v_cache.contiguous().to(device)
        self.out = torch.empty_like(self.q)
        self.host_out = torch.empty(self.out.shape, dtype=self.out.dtype, pin_memory=True)

    def call(self, stream):
        self.apd.attn_paged_prefill(self.q, self.k, self.v, self.pt, self.sl, self.w.scale, self.w.causal_offset,
                                    None, self.out, stream=stream, kernel=self.kernel)


def prefill_kernel_name(choice):
    """The kernel the prefill workload (D = 128, 512 query rows per kv head) runs for a
    --prefill-kernel choice."""
    import decode_attention_paged_split_b200 as apd

    if choice == "auto":
        choice = apd.prefill_auto_kernel(128)
    return "prefill_tc2_kernel" if choice == "tcgen05" else "prefill_kernel"


def run_prefill(a):
    """The prefill chunk on one GPU: CUDA-graph replays of the call over two cache
    instances used in turn (each larger than L2)."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        print("no CUDA device", file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group(world, "nccl")
    import decode_attention_paged_split_b200 as apd

    ws = [workloads.prefill_llama8b_chunk(seed=8 + 1000003 * rank + i) for i in range(2)]
    insts = [PrefillInst(w, device, a.prefill_kernel) for w in ws]
    w0 = ws[0]
    per_bytes, per_flops = w0.algorithmic_bytes(), w0.algorithmic_flops()
    stream = torch.cuda.Stream(device)

    def call(i):
        insts[i % 2].call(stream)

    for i in range(a.warmup):
        call(i)
    torch.cuda.synchronize(device)
    graphs = GraphSteps(lambda i, st: call(i), stream, a.steps, period=2)
    clocks = ClockSampler(local, enabled=not a.no_clocks and rank == 0)
    times = timed_reps(lambda: graphs.run(stream), dist, device, a.min_seconds)
    clock_info = clocks.stop()
    graphs.release()
    t_max = statistics.median(times)
    bytes_all = sum_over_ranks(float(per_bytes * a.steps), dist, device)
    flops_all = sum_over_ranks(float(per_flops * a.steps), dist, device)

    # end to end through host buffers (PCIe-bound: the chunk's q and out are 16.8 MB each)
    e2e = None
    if not a.no_e2e:
        e2e_n = max(4, min(a.steps, 200))
        barrier(dist, device)
        torch.cuda.synchronize(device)
        e2e_el, h2d, d2h = e2e_steps(insts, stream, e2e_n)
        e2e_max = max_over_ranks(e2e_el, dist, device)
        e2e_flops = sum_over_ranks(float(per_flops * e2e_n), dist, device)
        e2e = {"value": e2e_flops / e2e_max / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_max / e2e_n * 1e3, "steps": e2e_n,
               "how": "per step, eager through the public Python API: one pinned-host->device copy of the packed "
                      "q|page_table|seq_lens, the call, one device->pinned-host copy of out; copies on two copy "
                      "streams overlap the neighbouring steps' compute"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import oracle

        sample = workloads.prefill_llama8b_chunk(batch=1, seq_lens=[4096])
        t0 = time.perf_counter()
        oracle.paged_prefill(sample)
        el_cpu = time.perf_counter() - t0
        cpu = {"value": sample.algorithmic_flops() / el_cpu / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
               "kind": "oracle", "sample": f"sequence 0 only (1 of 16) of the chunk, fp64, {el_cpu:.1f} s"}

    if rank == 0:
        us = t_max / a.steps * 1e6
        tpeak, tsrc = peak_tflops()
        hpeak, hsrc = peaks()
        tf = per_flops / (t_max / a.steps) / 1e12
        gbs = per_bytes / (t_max / a.steps) / 1e9
        line = {
            "metric": PREFILL_METRIC, "value": flops_all / t_max / 1e12, "unit": "TFLOP/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": us / 1e3, "us_per_call": us, "hbm_gbs": gbs,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w0.name, "batch": w0.batch, "q_len": w0.q_len, "num_q_heads": 32,
                       "num_kv_heads": 8, "head_dim": 128, "seq_len": 4096, "causal_offset": w0.causal_offset,
                       "algorithmic_bytes_per_call": per_bytes, "algorithmic_flops_per_call": per_flops,
                       "l2": "two cache instances used in turn, each larger than L2",
                       "launch": f"CUDA graphs of up to {GRAPH_CHUNK} consecutive calls with event-record nodes "
                                 f"around the K calls; the K-call region repeated for about {a.min_seconds:g} s"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": tpeak, "unit": "TFLOP/s", "frac": tf / tpeak,
                         "traffic": (committed_traffic(w0.name, PREFILL_TRAFFIC_FILE, PREFILL_KERNEL_SOURCES)
                                     if prefill_kernel_name(a.prefill_kernel) == "prefill_tc2_kernel" else None),
                         "peak_source": tsrc, "kernel": prefill_kernel_name(a.prefill_kernel),
                         "hbm_achieved_gbs": gbs, "hbm_frac": gbs / hpeak},
            "timing": timing_summary(times, a.steps),
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": a.steps * len(times), "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_sweep(a):
    """The head-dim / GQA sweep: every (D, heads, num_splits) case of the configuration, one
    call at a time with the L2 flushed before each (a 512 MB write), timed with CUDA events
    around the call.  The cases' footprints (2-17 MB) would otherwise stay in L2."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        print("no CUDA device", file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group(world, "nccl")
    import decode_attention_paged_split_b200 as apd

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)
    samples = max(5, min(a.steps, 200))
    clocks = ClockSampler(local, enabled=not a.no_clocks and rank == 0)
    cases, total_us, total_bytes = [], 0.0, 0
    for d, hq, hkv, s in workloads.sweep_cases():
        w = workloads.sweep_case(d, hq, hkv, s, seed=2024 + 1000003 * rank)
        q, k_, v_ = w.q.to(device), w.k_cache.contiguous().to(device), w.v_cache.contiguous().to(device)
        pt, sl = w.page_table.to(device), w.seq_lens.to(device)
        out = torch.empty_like(q)
        ws = apd.alloc_workspace(w.batch, hq, hkv, d, s, device=device)
        call = apd.DecodeCall(q, k_, v_, pt, sl, out, w.scale, s, ws)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(samples)]
        with torch.cuda.stream(stream):
            for i in range(a.warmup):
                call(stream)
            for i, (e0, e1) in enumerate(ev):
                flush.fill_(i & 0xFF)
                e0.record(stream)
                call(stream)
                e1.record(stream)
            warm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(samples)]
            for e0, e1 in warm:
                e0.record(stream)
                call(stream)
                e1.record(stream)
        stream.synchronize()
        cold = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in ev)
        hot = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in warm)
        cold = max_over_ranks(cold, dist, device)
        b = w.algorithmic_bytes()
        pl = apd.query_plan(w.batch, hq, hkv, d, s)
        cases.append({"case": w.name, "head_dim": d, "num_q_heads": hq, "num_kv_heads": hkv, "num_splits": s,
                      "kv_tokens": w.kv_tokens(), "algorithmic_bytes": b, "cold_l2_us": cold, "warm_l2_us": hot,
                      "cold_gbs": b / cold / 1e3, "launches": 1 + (1 if pl.combine_ctas > 0 else 0)})
        total_us += cold
        total_bytes += b
    clock_info = clocks.stop()
    if rank == 0:
        peak, peak_src = peaks()
        line = {"metric": SWEEP_METRIC, "value": total_us, "unit": "us (sum over the 16 cases)", "n_gpus": world,
                "steps": samples, "warmup": a.warmup, "ms_per_step": total_us / 1e3, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "sweep_b4_d32-256_h8x8-32x8_s1-4",
                           "l2": "512 MB written before each timed call (cold L2); warm_l2_us: the same call "
                                 "repeated without the flush",
                           "timing": f"CUDA events around each call, median of {samples}"},
                "roofline": {"bound": "hbm", "achieved": total_bytes / total_us / 1e3, "peak": peak, "unit": UNIT,
                             "frac": total_bytes / total_us / 1e3 / peak, "traffic": None,
                             "peak_source": peak_src,
                             "note": "latency-bound: 2-17 MB per call is a few microseconds at the HBM rate"},
                "cases": cases, "clocks": clock_info,
                "gpu_launches": sum(c["launches"] for c in cases) * (samples * 2 + a.warmup)}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    a = parse_args(argv)
    if a.workload == "sweep" and a.impl != "reference":
        return run_sweep(a)
    if a.impl == "reference":
        if a.workload.startswith(("gemv_", "prefill_")) or a.workload == "sweep":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the decode-attention "
                                                                  "workloads; use the gemv workloads' cpu_baseline"}))
            return 0
        return run_reference(a)
    if a.workload.startswith("gemv_"):
        return run_gemv(a)
    if a.workload.startswith("prefill_"):
        return run_prefill(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
