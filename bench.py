#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long32k]
                    [--impl ours|reference]

One step = one decode step of the workload through every piece of the path:
the host allocator's slots and tables (a1), the copy-on-write block copy when
the step has one (a2), the KV append of the new tokens (a3, written by the
decode kernel itself when the step appends one token per decoded sequence:
pa_append_decode), the paged decode main kernel (a4) and the split reduce
(a5); the grid takes the sequences longest first.  Default workload: the
long-context batch (8 sequences x 32768 tokens, 64/8 heads, head_dim 128,
bf16 KV, block size 16, 512-token splits); each step appends one token per
sequence and decodes; the last planned step decodes exactly 32768 tokens.

* ``value``: KV bytes read by the decode per step (sum over sequences of
  L_s * Hkv * D * 2 * 2 bytes) / device step time, with the step's inputs
  (queries, new K/V rows, slots, tables, lengths) already in HBM, timed with
  CUDA events over K steps (K cycles through up to 64 distinct planned steps;
  re-running a planned step rewrites the same slots with the same bytes, so
  every pass does identical work).  The KV cache (1.07 GB) is larger than
  L2, so no flush is needed between steps.
* ``e2e``: the same metric through the public API with host buffers: the
  allocator runs live, inputs are copied from pinned host memory and every
  step's output is copied back to pinned host memory (steps of a repeated
  layout replayed from CUDA graphs, their copies on copy streams of their
  own).  The host reads step i's output while the GPU runs step i+1 (two
  output buffers), so the GPU always has the next step queued;
  ``--sync-e2e`` waits for each step before launching the next.
* ``roofline``: the main decode kernel's algorithmic bytes per launch over
  its own CUDA-event time (events recorded by the library around that launch
  on the launching stream, L2 flushed by a 256 MB read before each of 32
  launches), against the measured HBM copy bandwidth.
* ``configs`` (N = 1): the Llama-8B-shaped, beam and continuous-mix (block
  16) workloads, each with its step time, main-kernel time and end to end.
* ``cpu_baseline``: the fp64 oracle on the host cores on a bounded sample of
  the same workload.
* ``prefill`` (N = 1): the chunked-prefill kernel on 8 x (4096 context +
  1024-token chunk), its TFLOP/s against the measured bf16 tensor peak, timed
  apart from the decode steps.

``--study prefix|swap|blocksize|prefill`` prints one side study instead.

``--impl reference`` times the oracle alone (the CPU arm).  With N > 1 GPUs
(torchrun) every rank runs its own batch (a different seed) with no
collective on the data path; times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

NOMINAL_HBM_GBS = 8000.0
# pa_decode's default merges split partials with a reduce kernel whenever a
# sequence has more than one split
FUSED_MERGE_MAX_SPLITS = 1
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------- distributed
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    group = None
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
        group = dist.group.WORLD
    return ws, rank, local, group


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(elapsed_s: float, units: float, ws: int, device=None):
    """(max elapsed over ranks, sum of units over ranks)."""
    if ws <= 1:
        return elapsed_s, units
    import torch.distributed as dist
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def rank_seed(base: int, rank: int) -> int:
    return base + 1000 * rank


# ----------------------------------------------------------------- workloads
def make_workload(name: str, n_steps: int, seed: int, batch: int = 0):
    if name == "long32k":
        return workloads.long_context(seed=seed, steps=n_steps, batch=batch or 8), 2048
    if name == "llama8b":
        return workloads.llama(seed=seed, steps=n_steps), 4096 // 16 + 1 + (n_steps + 15) // 16
    if name.startswith("mix"):
        bs = int(name[len("mix_bs"):]) if name.startswith("mix_bs") else 16
        return workloads.mix(seed=seed, block_size=bs, steps=n_steps), (8192 + n_steps) // bs + 2
    if name == "beam":
        return workloads.beam(seed=seed, steps=n_steps), (2050 + n_steps) // 16 + 2
    raise SystemExit(f"unknown workload {name}")


SEEDS = {"long32k": 2, "llama8b": 1, "beam": 3}

DESCR = {
    "long32k": "long context: B 8, Hq 64 / Hkv 8, D 128, bf16 KV, block 16, seq_len 32768, "
               "split 512 + reduce, 32768-block pool in a seeded permutation",
    "llama8b": "Llama-8B-shaped decode: B 32, Hq 32 / Hkv 8, D 128, bf16 KV, block 16, "
               "seq_len U[512, 4096], 16384-block pool in a seeded permutation",
    "beam": "prefix sharing / beam search: 4 prompts x 4 beams, 2050-token shared prefix, "
            "32/8 heads, D 128, fp16 KV, block 16",
    "mix_bs16": "continuous-batching mix: 256 sequences, seq_len log-U[16, 8192], 32/8 heads, "
                "D 128, bf16 KV, block 16, 10% finish and 128-token admissions per step",
}


def kv_bytes(lens, hkv, d, e) -> int:
    return int(np.asarray(lens, dtype=np.int64).sum()) * hkv * d * 2 * e


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.gpu = gpu_index
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = []
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[2]), float(parts[3]), parts[5:]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        lo, hi = (self.t0 or 0) - 1, (self.t1 or 1e18) + 1
        win = [r for r in rows if lo <= r[0] <= hi] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in win:
            for n, v in zip(names, r[3][1:]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median([r[1] for r in win])),
                "sm_max_mhz": float(max(r[2] for r in win)),
                "reasons": sorted(reasons), "samples": len(win)}


# ----------------------------------------------------------------- peaks
def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, torch copy read+write)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


# the main decode kernel of each variant: its name and its sources
DECODE_KERNELS = {1: ("decode_simt_kernel", "decode_simt.cu"),
                  2: ("decode_tc_kernel", "decode_tc.cu"),
                  3: ("decode_hw_kernel", "decode_hw.cu")}
COMMON_SOURCES = ("decode_common.cuh", "common.cuh", "launch.h")


def decode_source_hash(variant: int) -> str:
    """First 16 hex digits of the sha256 of a decode kernel's sources."""
    h = hashlib.sha256()
    for name in (DECODE_KERNELS[variant][1],) + COMMON_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_347_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload: str, variant: int, alg_bytes_per_launch: float):
    """DRAM bytes (read + write) per launch of the main decode kernel, from
    the committed ncu summary, if it was taken on the kernel's sources as they
    are now (else None).  A summary taken on a smaller case of the workload
    is scaled to a full launch by the ratio of algorithmic bytes, which
    holds while traffic grows in proportion to the tokens read."""
    name = DECODE_KERNELS[variant][0]
    path = os.path.join(ROOT, "profiles", f"{name}_{workload}.json")
    try:
        with open(path) as f:
            prof = json.load(f)
        h = decode_source_hash(variant)
    except (OSError, ValueError):
        return None
    if prof.get("kernel_src_sha256_16") != h:
        return None
    dram = float(prof["dram_bytes_per_launch"])
    alg = float(prof.get("algorithmic_bytes_per_launch") or 0)
    if alg > 0:
        dram *= alg_bytes_per_launch / alg
    return int(round(dram))


# ----------------------------------------------------------------- CPU oracle
class OracleSampler:
    """The fp64 oracle on sequence 0 of the workload's shape (same seed):
    state built once, then timed head by head.  A (sequence, head) pair is
    credited 1/G of its KV head's bytes, so a whole sequence counts its KV
    bytes once, as the device metric does."""

    def __init__(self, wl_name: str, seed: int):
        from oracle.run import OracleRun
        from oracle import attn
        self.attn = attn
        if wl_name == "long32k":
            wl = workloads.long_context(seed=seed, steps=1, batch=1)
        else:
            wl, _ = make_workload(wl_name, 1, seed)
        sh = self.sh = wl.shape
        self.orc = OracleRun(sh)
        steps = list(wl.steps)
        for st in steps[:-1]:
            self.orc.step(st, decode=False)
        self.last = steps[-1]
        res = self.orc.step(self.last, decode=False)
        self.bt, self.lens = res["block_tables"][:1], res["seq_lens"][:1]
        self.L = int(self.lens[0])
        self.G = sh.num_heads // sh.num_kv_heads
        self.threads = attn.max_threads()
        self.h = 0

    def run(self, budget_s: float, min_pairs: int = 1, threads: int = 0):
        sh = self.sh
        n = threads or self.threads
        done_bytes, done_pairs, spent = 0.0, 0, 0.0
        while spent < budget_s or done_pairs < min_pairs:
            chunk = [(0, (self.h + i) % sh.num_heads) for i in range(n)]
            t = time.perf_counter()
            self.attn.paged_decode(self.last.q[:1], self.orc.k_cache, self.orc.v_cache, self.bt,
                                   self.lens, sh.scale, sel=chunk, n_threads=n)
            spent += time.perf_counter() - t
            done_pairs += len(chunk)
            done_bytes += len(chunk) * self.L * sh.head_dim * 2 * sh.elem_bytes / self.G
            self.h += len(chunk)
        return done_bytes, spent, done_pairs


# ----------------------------------------------------------------- main arm
class Planned:
    """One workload made ready for timing: its runner with the prefill
    applied, every decode step planned by the host allocator (timed apart)
    and its inputs staged in HBM."""

    def __init__(self, name: str, n_plan: int, seed: int, dev, batch: int = 0,
                 partition: int = -1):
        from paged_kv_cache_347_b200.runner import PagedKVRunner
        self.name = name
        wl, self.width = make_workload(name, n_plan, seed, batch)
        self.sh = sh = wl.shape
        self.runner = PagedKVRunner.for_shape(sh, self.width, device=str(dev),
                                              partition_size=partition)
        steps = list(wl.steps)
        self.prefill, dec = steps[0], steps[1:]
        self.runner.run(self.prefill)                      # untimed prefill
        torch.cuda.synchronize()
        ast = self.runner.alloc.stats()
        self.alloc_info = {"block_size": sh.block_size, "used_blocks": ast["used_blocks"],
                           "reserved_slots": ast["reserved_slots"],
                           "logical_tokens": ast["logical_tokens"],
                           "tail_waste_frac": round(1 - ast["logical_tokens"]
                                                    / max(1, ast["reserved_slots"]), 5)}
        t = time.perf_counter()
        self.plans = [self.runner.plan(st.ops) for st in dec]
        self.plan_py_us = (time.perf_counter() - t) / len(dec) * 1e6
        self.alloc_us = self._step_plan_us(sh, steps)
        for acts in self.plans:
            self.runner.upload(acts)
        self.dev_in = [(st.k_new.to(dev), st.v_new.to(dev), st.q.to(dev)) for st in dec]
        self.b = dec[0].q.shape[0]
        self.out = torch.empty((self.b, sh.num_heads, sh.head_dim), dtype=torch.float32,
                               device=dev)
        self.decodes = [[a for a in acts if a.kind == "decode"][0] for acts in self.plans]
        self.step_bytes = [kv_bytes(d.lens, sh.num_kv_heads, sh.head_dim, sh.elem_bytes)
                           for d in self.decodes]
        # kernels each step launches: the copy-on-write copy, the append
        # (unless the decode writes the step's new tokens itself), the main
        # decode and, when the longest sequence has more splits than the
        # library merges inside the main kernel, the reduce
        self.launches_per = []
        for acts in self.plans:
            n = 0
            for a in acts:
                if a.kind == "write":
                    n += (1 if len(a.pairs) else 0) + (1 if a.nrows and not a.fused else 0)
                else:
                    n += 1 + (1 if math.ceil(a.max_len / (a.partition or 512))
                              > FUSED_MERGE_MAX_SPLITS else 0)
            self.launches_per.append(n)

    def _step_plan_us(self, sh, steps) -> float:
        """Host time per decode step of pa_step_plan (the runtime's one call:
        the step's events applied, slots, table rows, lengths and the
        longest-first order written into a staging buffer), on a replica of
        the allocator fed the same events; the events are encoded beforehand,
        as a runtime keeps them."""
        from paged_kv_cache_347_b200 import pagedattn as pa
        from paged_kv_cache_347_b200.runner import PagedKVRunner
        alloc = pa.BlockAllocator(sh.num_blocks, sh.block_size, sh.free_order)
        encs = [PagedKVRunner.encode_ops(st.ops) for st in steps]
        if any(e is None for e in encs):
            return float("nan")
        stage = np.zeros(1 << 20, np.uint8)

        def plan(e):
            nonlocal stage
            lay = alloc.step_layout(e.events, e.decode_ids.size, self.width)
            if lay.bytes > stage.nbytes:
                stage = np.zeros(lay.bytes, np.uint8)
            alloc.step_plan(e.events, e.decode_ids, self.width, stage)

        plan(encs[0])                                     # the prefill
        t = time.perf_counter()
        for e in encs[1:]:
            alloc.step_plan(e.events, e.decode_ids, self.width, stage)
        return (time.perf_counter() - t) / max(1, len(encs) - 1) * 1e6

    def step(self, i: int) -> None:
        j = i % len(self.plans)
        k, v, q = self.dev_in[j]
        self.runner.execute(self.plans[j], k, v, q, out=self.out)

    def alg_bytes(self, j: int) -> int:
        """Algorithmic bytes of step j's main decode launch: K/V of every
        token, the queries, the table entries and the lengths."""
        sh, d = self.sh, self.decodes[j]
        nb = int(sum(-(-int(x) // sh.block_size) for x in d.lens))
        return (self.step_bytes[j] + self.b * sh.num_heads * sh.head_dim * sh.elem_bytes
                + nb * 4 + self.b * 4)

    def partitions(self):
        return sorted({d.partition or 512 for d in self.decodes})

    def close(self):
        self.runner = self.plans = self.dev_in = None
        torch.cuda.empty_cache()


_FLUSH = {}


L2_BYTES = 126 * 1000 * 1000  # B200 L2 (126 MB)


def flush_l2(dev) -> None:
    """Reads 256 MB (twice the 126 MB L2) so that the next kernel finds none
    of its data in L2.  A read leaves clean lines, which the next kernel
    evicts for free; a write would leave ~126 MB of dirty lines for it to
    write back to HBM in its own time."""
    buf = _FLUSH.get(dev)
    if buf is None:
        buf = _FLUSH[dev] = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        _FLUSH[(dev, "sink")] = torch.empty(1, dtype=torch.float32, device=dev)
    torch.sum(buf, dim=0, keepdim=True, out=_FLUSH[(dev, "sink")])


def time_main_kernel(pl: Planned, n: int, dev) -> dict:
    """The main decode kernel alone, over n launches (cycling through the
    planned steps' decodes), each between CUDA events that the library
    records on the launching stream around that kernel, with L2 flushed
    before every launch (outside the events)."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    r, sh = pl.runner, pl.sh
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    alg = []
    for i in range(n + 2):
        j = i % len(pl.plans)
        d, q = pl.decodes[j], pl.dev_in[j][2]
        flush_l2(dev)
        if i >= 2:
            pa.set_profile_events(*evs[i - 2])
        pa.pa_decode(pl.out, q, r.k_cache, r.v_cache, d.dev["tables"], d.dev["lens"], r.scale,
                     max_seq_len=d.max_len, partition_size=d.partition, variant=d.variant,
                     heads_per_cta=d.hpc, seq_order=d.dev.get("order"))
        if i >= 2:
            pa.set_profile_events(None, None)
            alg.append(pl.alg_bytes(j))
    torch.cuda.synchronize()
    us = [b.elapsed_time(e) * 1e3 for b, e in evs]
    return {"us": us, "alg": alg}


def roofline_of(main: dict, peak: float, peak_src: str, traffic,
                kernel: str = "decode_tc_kernel") -> dict:
    us = np.asarray(main["us"])
    per_launch = float(np.mean(main["alg"]))
    # bytes over time launch by launch, averaged: the launches differ in size
    achieved = float(np.sum(main["alg"]) / np.sum(us) / 1e3)
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": f"pa_decode main ({kernel})", "peak_source": peak_src,
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "main_us_per_launch": round(float(us.mean()), 2),
            "main_us_median": round(float(np.median(us)), 2),
            "timed_launches": int(us.size),
            "main_us_p10_median_p90": [round(float(np.percentile(us, q)), 2)
                                       for q in (10, 50, 90)],
            "l2": "flushed before every timed launch",
            "algorithmic_bytes_per_launch": int(per_launch)}


def run_ours(args, ws, rank, local):
    from paged_kv_cache_347_b200 import pagedattn as pa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    seed = rank_seed(SEEDS.get(args.workload, 4), rank)
    n_plan = min(args.steps + args.warmup, 64)
    pl = Planned(args.workload, n_plan, seed, dev, args.batch, args.partition)
    sh, plans, b = pl.sh, pl.plans, pl.b

    # warm-up (the first W planned steps, then cycling)
    for i in range(args.warmup):
        pl.step(i)
    torch.cuda.synchronize()

    # The K timed steps as one CUDA graph, captured and replayed once
    # untimed: the device then runs them back to back, however fast the
    # host issues launches (a host that is late with the first step would
    # otherwise leave the device idle inside the timed region).  Replaying
    # the steps again repeats the same appends into the same slots and the
    # same decodes, so the timed replay does exactly the K steps' work.
    total_bytes = 0
    launches = 0
    for i in range(args.steps):
        total_bytes += pl.step_bytes[(args.warmup + i) % len(plans)]
        launches += pl.launches_per[(args.warmup + i) % len(plans)]
    timed = torch.cuda.CUDAGraph()
    keep = []  # every split workspace a captured step writes stays allocated
    with torch.cuda.graph(timed, capture_error_mode="thread_local"):
        for i in range(args.steps):
            pl.step(args.warmup + i)
            keep.append(pa.cached_workspace(dev))
    timed.replay()
    torch.cuda.synchronize()

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                          if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit()
                          else local)
    clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    clocks.mark("t0")
    # nothing but the steps between the two events: an event between two
    # kernels would stop the second launching as a programmatic dependent
    t_start.record()
    timed.replay()
    t_end.record()
    torch.cuda.synchronize()
    del timed, keep
    # the main kernel alone, after the steps (its own launches, not counted
    # in gpu_launches); still inside the clock record
    main = time_main_kernel(pl, max(16, args.main_launches), dev)
    clocks.mark("t1")
    barrier(ws)
    clk = clocks.stop()
    elapsed = t_start.elapsed_time(t_end) / 1e3
    errs = pa.device_errors(clear=True)
    if errs:
        raise SystemExit(f"device errors during the bench: {errs}")

    elapsed_max, bytes_all = aggregate(elapsed, float(total_bytes), ws, dev)
    value = bytes_all / elapsed_max / 1e9
    ms_per_step = elapsed_max / args.steps * 1e3

    peak, peak_src = hbm_peak()
    variant = pl.decodes[-1].variant or (1 if sh.dtype == "f32" else 2)
    traffic = traffic_from_profile(args.workload, variant, float(np.mean(main["alg"])))
    roof = roofline_of(main, peak, peak_src, traffic, DECODE_KERNELS[variant][0])

    # end to end through the public API with host buffers
    e2e = run_e2e(args, sh, pl.width, seed, pl.prefill, dev, ws)
    seq_len = int(max(int(max(d.lens)) for d in pl.decodes))
    res = {
        "metric": "paged decode attention: KV-read GB/s (% of B200 HBM peak), us/step",
        "value": round(value, 1), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "tokens_per_s": round(b * ws / (ms_per_step / 1e3), 1),
        "frac_of_peak": round(value / peak, 4), "frac_of_nominal_8tbs": round(value / NOMINAL_HBM_GBS, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), numpy PCG64, rounded to bf16)",
        "config": {"workload": f"{args.workload}: {DESCR.get(args.workload, args.workload)}",
                   "global_batch": b * ws, "seq_len": seq_len,
                   "parallelism": f"dp{ws} (independent batches, no collective)",
                   "l2": "inputs larger than L2 (KV cache 1.07 GB per step), no flush",
                   "planned_steps": len(plans), "host_alloc_us_per_step": round(pl.alloc_us, 2),
                   "host_alloc_note": "pa_step_plan per decode step (events applied, slots, "
                                      "table rows, lengths, order written)",
                   "host_plan_op_by_op_us_per_step": round(pl.plan_py_us, 2),
                   "partition_tokens": pl.partitions(),
                   "partition_policy": {-1: "per step, pa_decode_choose",
                                        0: "library default"}.get(args.partition, "fixed"),
                   "kernels": sorted({DECODE_KERNELS[d.variant or 2][0] for d in pl.decodes}),
                   "dispatch": "longest first; one-token appends fused into the decode",
                   "timed_region": "the K steps replayed from one CUDA graph (captured, and "
                                   "replayed once, before the timed replay)",
                   "allocator_after_prefill": pl.alloc_info},
        "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    pl.close()
    if rank == 0 and ws == 1 and not args.no_configs:
        res["configs"] = {name: measure_config(name, args, dev, peak)
                          for name in CONFIG_LINES}
    if rank == 0 and ws == 1 and not args.no_prefill:
        # the chunked-prefill kernel (tensor-core bound), timed apart from the
        # decode steps above
        mma_sync, tc, persistent, p16 = prefill_rows(4096, 1024)
        peak_tf, peak_tf_src = _bf16_peak_tflops()
        res["prefill"] = {
            "workload": "chunked prefill: 8 x (4096 context + 1024-token chunk), 32/8 heads, "
                        "D 128, bf16 KV, block 16",
            "kernel": "pa_prefill (prefill_umma_kernel, tcgen05)", "ms": tc["ms"],
            "roofline": {"bound": "tensor", "achieved": tc["tflops"], "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": tc["frac_of_bf16_peak"],
                         "flops_per_launch": tc["flops_per_launch"], "peak_source": peak_tf_src},
            "mma_sync_kernel_ms": mma_sync["ms"], "persistent_kernel_ms": persistent["ms"],
            "max_abs_diff_vs_mma_sync": tc["max_abs_diff_vs_mma_sync"],
            "one_fp16_p": {
                "variant": 4, "ms": p16["ms"], "tflops": p16["tflops"],
                "frac": p16["frac_of_bf16_peak"],
                "max_abs_diff_vs_mma_sync": p16["max_abs_diff_vs_mma_sync"],
                "note": "opt-in: each weight rounded once to fp16 (within 2^-11, against "
                        "2^-14 for the default's high part + remainder), half the P.V "
                        "products; the bf16 V stages converted to fp16 in shared memory"}}
        # the same workload with an f16 cache, where the one-fp16-P form needs
        # no conversion of V
        t2, t4 = prefill_rows(4096, 1024, dtype="f16",
                              variants=((2, "tcgen05"), (4, "tcgen05, one fp16 P")))
        res["prefill"]["f16_cache"] = {
            "tcgen05_ms": t2["ms"], "one_fp16_p_ms": t4["ms"], "one_fp16_p_tflops": t4["tflops"],
            "one_fp16_p_frac": t4["frac_of_bf16_peak"],
            "max_abs_diff_one_fp16_p_vs_tcgen05": t4["max_abs_diff_vs_tcgen05"]}
    if rank == 0 and ws == 1 and not args.no_cpu:
        smp = OracleSampler(args.workload, seed)
        nb, secs, pairs = smp.run(args.cpu_budget)
        res["cpu_baseline"] = {"value": round(nb / secs / 1e9, 4), "unit": "GB/s",
                               "cores": smp.threads, "kind": "oracle",
                               "sample": f"sequence 0 of the workload's shape ({smp.L} tokens), "
                                         f"{pairs} (sequence, head) pairs, fp64 C loop, "
                                         f"{secs:.1f} s"}
        res["cpu_baseline"]["single_thread"] = single_thread_oracle(seed)
    return res


def single_thread_oracle(seed: int) -> dict:
    """The oracle on one host thread: the Llama-8B-shaped workload's sequence
    0 (GB/s over a ~3 s sample) and the tiny workload's whole decode step (us
    per step, repeated for ~1 s)."""
    from oracle.run import OracleRun
    from oracle import attn
    smp = OracleSampler("llama8b", SEEDS.get("llama8b", seed))
    nb, secs, pairs = smp.run(3.0, threads=1)
    wl = workloads.tiny()
    orc = OracleRun(wl.shape)
    steps = list(wl.steps)
    res = orc.step(steps[0], decode=False)
    n, t = 0, time.perf_counter()
    while time.perf_counter() - t < 1.0:
        attn.paged_decode(steps[0].q, orc.k_cache, orc.v_cache, res["block_tables"],
                          res["seq_lens"], wl.shape.scale, n_threads=1)
        n += 1
    tiny_us = (time.perf_counter() - t) / n * 1e6
    return {"llama8b_GBs": round(nb / secs / 1e9, 4),
            "llama8b_sample": f"sequence 0 ({smp.L} tokens), {pairs} (sequence, head) pairs, "
                              f"{secs:.1f} s",
            "tiny_us_per_decode": round(tiny_us, 2), "threads": 1}


# The other configurations, measured on the default N = 1 run next to the
# headline workload: (planned decode steps, timed steps, e2e steps).
CONFIG_LINES = {"llama8b": (24, 24, 24), "beam": (24, 24, 24), "mix_bs16": (32, 32, 32)}


def measure_config(name: str, args, dev, peak: float) -> dict:
    """One configuration: device step time, the main kernel alone over 16+
    launches, and end to end through the public API.  A workload whose every
    step reads more K/V than L2 holds is timed as one loop of steps between
    two CUDA events, as the headline line is (an event between two steps
    would stop the next launching as a programmatic dependent); otherwise
    each step sits between its own events with L2 flushed before it."""
    n_plan, n_steps, n_e2e = CONFIG_LINES[name]
    seed = SEEDS.get(name, 4)
    pl = Planned(name, n_plan + 3, seed, dev, 0, args.partition)
    for i in range(3):
        pl.step(i)
    torch.cuda.synchronize()
    kv = sum(pl.step_bytes[(3 + i) % len(pl.plans)] for i in range(n_steps))
    # distinct K/V bytes the steps touch: the pool's blocks in use
    sh = pl.sh
    used = pl.runner.alloc.stats()["used_blocks"] * (2 * sh.num_kv_heads * sh.block_size
                                                      * sh.head_dim * sh.elem_bytes)
    looped = used > L2_BYTES
    if looped:
        b_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush_l2(dev)
        b_.record()
        for i in range(n_steps):
            pl.step(3 + i)
        e_.record()
        torch.cuda.synchronize()
        step_us = [b_.elapsed_time(e_) * 1e3 / n_steps]
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_steps)]
        for i in range(n_steps):
            flush_l2(dev)
            evs[i][0].record()
            pl.step(3 + i)
            evs[i][1].record()
        torch.cuda.synchronize()
        step_us = [b_.elapsed_time(e_) * 1e3 for b_, e_ in evs]
    main = time_main_kernel(pl, 16, dev)
    variant = pl.decodes[-1].variant or 2
    roof = roofline_of(main, peak, "", None, DECODE_KERNELS[variant][0])
    sh = pl.sh
    e2e_args = argparse.Namespace(**vars(args))
    e2e_args.workload, e2e_args.steps, e2e_args.e2e_steps, e2e_args.batch = name, n_e2e, n_e2e, 0
    e2e_args.warmup = 3
    e2e = run_e2e(e2e_args, sh, pl.width, seed, pl.prefill, dev, 1)
    mean_step = float(np.mean(step_us))
    out = {"workload": DESCR.get(name, name), "steps": n_steps,
           "us_per_step": round(mean_step, 2),
           "kv_GBs_step": round(kv / (mean_step * 1e-6 * n_steps) / 1e9, 1),
           "main_us": roof["main_us_per_launch"], "main_GBs": roof["achieved"],
           "kernels": sorted({DECODE_KERNELS[d.variant or 2][0] for d in pl.decodes}),
           "main_frac_of_peak": roof["frac"], "main_timed_launches": roof["timed_launches"],
           "partition_tokens": pl.partitions(),
           "tokens_per_s": round(pl.b / (mean_step * 1e-6), 1),
           "e2e_us_per_step": e2e["us_per_step"], "e2e": e2e,
           "host_alloc_us_per_step": round(pl.alloc_us, 2),
           "step_timing": ("one loop of steps between two events" if looped
                           else "each step between its own events"),
           "kv_blocks_in_use_MB": round(used / 1e6, 1),
           "l2": ("steps: the K/V blocks in use outsize L2, flushed once before the loop; "
                  "main kernel: flushed before every launch" if looped
                  else "flushed before every timed step and launch")}
    if name == "beam":
        out["note"] = ("16 beams' unique K/V (51 MB) fits in L2: GB/s are logical bytes "
                       "(each beam's reads), not HBM traffic; the first decode step, with "
                       "its 12 copy-on-write copies, is a warm-up step")
    pl.close()
    return out


def _chunks(enc, max_new: int):
    """A step's events cut into pieces of at most max_new appended tokens
    (a long append split across pieces; appends stay in order, so the rows
    of each piece are the next slice of the step's K/V rows).  Yields
    (events, first row, end row)."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    cur, rows, r0 = [], 0, 0
    for code, x, y in enc.events.tolist():
        if code != pa.EV_APPEND:
            cur.append((code, x, y))
            continue
        while y > 0:
            take = min(y, max_new - rows)
            cur.append((code, x, take))
            rows += take
            y -= take
            if rows == max_new:
                yield np.asarray(cur, np.int64).reshape(-1, 3), r0, r0 + rows
                cur, r0, rows = [], r0 + rows, 0
    if cur:
        yield np.asarray(cur, np.int64).reshape(-1, 3), r0, r0 + rows


def _decode_lens(sh, encs, width):
    """Each step's decode lengths, from the same events replayed on a host
    replica of the allocator (for the byte count of the metric)."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    alloc = pa.BlockAllocator(sh.num_blocks, sh.block_size, sh.free_order)
    stage = np.zeros(1 << 16, np.uint8)
    out = []
    for enc in encs:
        lay = alloc.step_layout(enc.events, enc.decode_ids.size, width)
        if lay.bytes > stage.nbytes:
            stage = np.zeros(lay.bytes, np.uint8)
        lay = alloc.step_plan(enc.events, enc.decode_ids, width, stage)
        b = enc.decode_ids.size
        out.append(stage[lay.off_lens:lay.off_lens + 4 * b].view(np.int32).copy())
    return out


def run_e2e_runtime(args, sh, width, seed, dev, ws):
    """Live steps through the native runtime (pa_runtime: one library call
    per step -- the allocator's events, the decode's choice, the copies in,
    the kernels from a CUDA graph, the output's copy back), inputs in
    page-locked host memory, every output read one step behind."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    n = max(1, min(args.steps, args.e2e_steps))
    w = min(args.warmup, 3)
    wl, _ = make_workload(args.workload, n + w, seed, args.batch)
    steps = list(wl.steps)
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[sh.dtype]
    dims = (sh.num_blocks, sh.num_kv_heads, sh.block_size, sh.head_dim)
    kc = torch.zeros(dims, dtype=dt, device=dev)
    vc = torch.zeros_like(kc)
    # a step's host inputs: its events as arrays (the form a runtime keeps
    # them in), new K/V rows and queries in page-locked memory
    encs = [PagedKVRunner.encode_ops(st.ops) for st in steps]
    lens = _decode_lens(sh, encs, width)
    b = steps[1].q.shape[0]
    max_new = max(16384, max(st.k_new.shape[0] for st in steps[1:]))
    rt = pa.Runtime(kc, vc, sh.num_heads, width, b, max_new, sh.scale, sh.free_order)
    k0, v0 = steps[0].k_new.pin_memory(), steps[0].v_new.pin_memory()
    none = np.empty(0, np.int64)
    for ev, r0, r1 in _chunks(encs[0], max_new):      # the prefill, untimed
        rt.wait_event(rt.step(ev, none, k0[r0:r1], v0[r0:r1], None, None))
    rt.wait()
    host = [(encs[i], steps[i].k_new.pin_memory(), steps[i].v_new.pin_memory(),
             steps[i].q.pin_memory()) for i in range(1, len(steps))]
    outs = [torch.empty((b, sh.num_heads, sh.head_dim), dtype=torch.float32).pin_memory()
            for _ in range(2)]

    def loop(first, count):
        pending = []
        for i in range(first, first + count):
            enc, k, v, q = host[i]
            pending.append(rt.step(enc.events, enc.decode_ids, k, v, q, outs[i & 1]))
            if len(pending) > 1:
                rt.wait_event(pending.pop(0))
        for ev in pending:
            rt.wait_event(ev)

    loop(0, w)
    st0 = rt.stats()
    barrier(ws)
    t = time.perf_counter()
    loop(w, n)
    el = time.perf_counter() - t
    st1 = rt.stats()
    kv = sum(kv_bytes(lens[1 + i], sh.num_kv_heads, sh.head_dim, sh.elem_bytes)
             for i in range(w, w + n))
    h2d = sum(host[i][1].nbytes + host[i][2].nbytes + host[i][3].nbytes
              for i in range(w, w + n)) / n
    el, total = aggregate(el, float(kv), ws, dev)
    return {"value": round(total / el / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(outs[0].nbytes),
            "steps": n, "us_per_step": round(el / n * 1e6, 2),
            "graph_replayed_steps": st1["replays"] - st0["replays"],
            "path": "pa_runtime (one library call per step)",
            "h2d_note": "new K/V rows and queries counted; the step's arrays (slots, table "
                        "rows, lengths, order) cross in the same copy stream",
            "outputs_read": "one step behind the launches"}


def run_e2e(args, sh, width, seed, prefill, dev, ws):
    if not args.e2e_python:
        return run_e2e_runtime(args, sh, width, seed, dev, ws)
    return run_e2e_python(args, sh, width, seed, prefill, dev, ws)


def run_e2e_python(args, sh, width, seed, prefill, dev, ws):
    """Live steps through the Python runner (PagedKVRunner prepare / stage_graph
    / replay_graph, or launch when a step has no graph form): host allocator,
    inputs copied from pinned host memory, every output copied back to pinned
    host memory and waited for, one step behind the launches unless
    ``--sync-e2e``."""
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    n = max(1, min(args.steps, args.e2e_steps))
    w = min(args.warmup, 3)
    wl, _ = make_workload(args.workload, n + w, seed, args.batch)
    steps = list(wl.steps)
    r = PagedKVRunner.for_shape(sh, width, device=str(dev), partition_size=args.partition)
    r.run(steps[0])
    torch.cuda.synchronize()
    # a step's host inputs: its events as arrays (pa_step_plan's form; ops it
    # does not take stay a list), new K/V rows and queries in page-locked memory
    host = [(r.encode_ops(st.ops) or st.ops, st.k_new.pin_memory(), st.v_new.pin_memory(),
             st.q.pin_memory()) for st in steps[1:]]
    b = steps[1].q.shape[0]
    # eager steps alternate between two output buffers, as the graphs of the
    # two staging slots do, so that step i+1 never overwrites the output of
    # step i before the host has it
    out_host = [torch.empty((b, sh.num_heads, sh.head_dim), dtype=torch.float32).pin_memory()
                for _ in range(2)]
    acc = {"h2d": 0, "d2h": 0, "kv": 0, "replays": 0}
    graphs = not args.no_graph
    lag = 0 if args.sync_e2e else 1

    def done(ev, res, counted):
        ev.synchronize()  # this step's output is in host memory
        if counted:
            d = [a for a in res["acts"] if a.kind == "decode"][0]
            acc["h2d"] += res["h2d"]
            acc["d2h"] += res["d2h"]
            acc["kv"] += kv_bytes(d.lens, sh.num_kv_heads, sh.head_dim, sh.elem_bytes)

    # Step i+1's allocator work and the copy of its inputs into page-locked
    # staging buffers run on the host while the GPU runs step i.  Staging
    # slot and output buffer of step i+1 are those of step i-1, whose output
    # is waited for first.
    def loop(first, count):
        if count <= 0:
            return
        pending = []
        prep = r.prepare(host[first][0])
        gr = r.stage_graph(prep, *host[first][1:]) if graphs else None
        for i in range(first, first + count):
            if gr is not None:
                res = r.replay_graph(gr, prep)
                acc["replays"] += first >= w
            else:
                res = r.launch(prep, *host[i][1:], out_host[i & 1])
            ev = res.get("ready")  # a graph step's output copy runs on its own stream
            if ev is None:
                ev = torch.cuda.Event()
                ev.record()
            pending.append((ev, res, first >= w))
            while len(pending) > lag:
                done(*pending.pop(0))
            if i + 1 < first + count:
                prep = r.prepare(host[i + 1][0])
                gr = r.stage_graph(prep, *host[i + 1][1:]) if graphs else None
        while pending:
            done(*pending.pop(0))

    loop(0, w)
    barrier(ws)
    t = time.perf_counter()
    loop(w, n)
    el = time.perf_counter() - t
    el, total = aggregate(el, float(acc["kv"]), ws, dev)
    return {"value": round(total / el / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": int(acc["h2d"] / n), "d2h_bytes_per_step": int(acc["d2h"] / n),
            "steps": n, "us_per_step": round(el / n * 1e6, 2),
            "graph_replayed_steps": acc["replays"],
            "outputs_read": "one step behind the launches" if lag else "each step before the next"}


def run_reference(args, ws, rank):
    """The oracle as it stands on the host cores, on a bounded sample per step."""
    if rank != 0:
        return None
    seed = SEEDS.get(args.workload, 4)
    smp = OracleSampler(args.workload, seed)
    # calibrate, then size each step so the whole run takes about two minutes
    _, secs1, pairs1 = smp.run(0.0)
    per_step_budget = max(secs1, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        smp.run(per_step_budget)
    nb_all = secs_all = 0.0
    pairs_all = 0
    for _ in range(args.steps):
        nb, secs, pairs = smp.run(per_step_budget)
        nb_all += nb
        secs_all += secs
        pairs_all += pairs
    v = nb_all / secs_all / 1e9
    return {
        "impl": "reference",
        "metric": "paged decode attention: KV-read GB/s (% of B200 HBM peak), us/step",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs_all / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), numpy PCG64, rounded to bf16)",
        "config": {"workload": f"{args.workload}: {DESCR.get(args.workload, args.workload)}",
                   "global_batch": 8, "seq_len": smp.L,
                   "parallelism": f"host cores (OpenMP, {smp.threads} threads)"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": smp.threads,
                         "kind": "oracle",
                         "sample": f"per step {pairs_all / args.steps:.0f} (sequence 0, head) "
                                   f"pairs of {smp.L} tokens, fp64 C loop"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ----------------------------------------------------------------- studies
def _events_ms(fn, reps=20):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    torch.cuda.synchronize()
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


def study_prefix(args):
    """Prefix caching on vs off for requests sharing a system prompt: K/V rows
    written at admission, admission time (allocator + append kernel), hits,
    and the causal attention the admission's prefill then needs (pa_prefill
    over the tokens each request must compute: its own suffix after the
    cached prompt, or every token without the cache)."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    res = {"study": "prefix_cache", "requests": 64, "prompt_tokens": 2048}
    for mode in ("on", "off"):
        wl = workloads.prefix_share(requests=64, prompt=2048, suffix_lo=16, suffix_hi=256,
                                    steps=1, num_blocks=16384)
        steps = list(wl.steps)
        admit = steps[0]
        if mode == "off":   # same tokens, no index: plain add + append of every token
            ops = []
            for op in admit.ops:
                ops += [("add", op[1]), ("append", op[1], len(op[2]))]
            admit = workloads.Step(ops, admit.k_new, admit.v_new, None, tag="admit")
        r = PagedKVRunner.for_shape(wl.shape, 160)
        k, v = admit.k_new.cuda(), admit.v_new.cuda()
        t = time.perf_counter()
        acts = r.plan(admit.ops)
        host_us = (time.perf_counter() - t) * 1e6
        r.upload(acts)
        rows = int(sum(int((a.slots >= 0).sum()) for a in acts if a.kind == "write"))
        ms = _events_ms(lambda: r.execute(acts, k, v, None), reps=10)
        st = r.alloc.stats()
        # tokens each request computes: those whose rows were written (a
        # cached token's row is skipped, slot -1, and its attention is done)
        ids = [op[1] for op in steps[0].ops]
        lens_all = [len(op[2]) for op in steps[0].ops]
        slots = np.concatenate([a.slots for a in acts if a.kind == "write"])
        own, o = [], 0
        for n in lens_all:
            own.append(int((slots[o:o + n] >= 0).sum()))
            o += n
        tables, lens = r.alloc.block_tables(ids, 160)
        cu = np.concatenate([[0], np.cumsum(own)]).astype(np.int32)
        g = torch.Generator(device="cuda").manual_seed(3)
        q = torch.randn(int(cu[-1]), 32, 128, generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty(int(cu[-1]), 32, 128, dtype=torch.float32, device="cuda")
        tab_d, len_d, cu_d = (torch.from_numpy(x).cuda() for x in (tables, lens, cu))
        pms = _events_ms(lambda: pa.pa_prefill(out, q, r.k_cache, r.v_cache, tab_d, len_d, cu_d,
                                                 r.scale, max_q_len=max(own),
                                                 max_seq_len=160 * 16), reps=10)
        flops = 4.0 * 128 * 32 * sum(sum(L - n + i + 1 for i in range(n))
                                      for L, n in zip(lens_all, own))
        res[mode] = {"rows_written": rows, "kv_bytes_written": rows * 8 * 128 * 2 * 2,
                     "append_kernel_us": round(ms * 1e3, 2), "allocator_us": round(host_us, 1),
                     "used_blocks": st["used_blocks"], "prefix_hit_blocks": st["prefix_hit_blocks"],
                     "prefix_query_blocks": st["prefix_query_blocks"],
                     "prefill_tokens": int(cu[-1]), "prefill_ms": round(pms, 3),
                     "prefill_tflops": round(flops / pms / 1e9, 1), "prefill_flops": flops}
        del r
        torch.cuda.empty_cache()
    res["device_errors"] = pa.device_errors()
    return res


def study_swap(args):
    """pa_swap_blocks bandwidth between HBM and pinned host memory for one
    32768-token sequence (2048 blocks of 8 heads x 16 x 128 bf16, K and V)."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, Hkv, bs, D, n = 4096, 8, 16, 128, 2048
    dk = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    dv = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    hk = torch.empty(n, Hkv, bs, D, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty(n, Hkv, bs, D, dtype=torch.bfloat16).pin_memory()
    r = np.random.default_rng(0)
    out_p = torch.from_numpy(np.stack([r.permutation(NB)[:n], np.arange(n)], 1)).cuda()
    in_p = torch.from_numpy(np.stack([np.arange(n), r.permutation(NB)[:n]], 1)).cuda()
    nbytes = n * Hkv * bs * D * 2 * 2
    out_ms = _events_ms(lambda: pa.pa_swap_blocks(hk, hv, dk, dv, out_p), reps=10)
    in_ms = _events_ms(lambda: pa.pa_swap_blocks(dk, dv, hk, hv, in_p), reps=10)
    errs = pa.device_errors()
    return {"study": "swap", "bytes": nbytes, "blocks": n,
            "swap_out_ms": round(out_ms, 3), "swap_out_GBs": round(nbytes / out_ms / 1e6, 1),
            "swap_in_ms": round(in_ms, 3), "swap_in_GBs": round(nbytes / in_ms / 1e6, 1),
            "device_errors": errs}


def study_blocksize(args):
    """Block-size trade-off on the continuous-batching mix: decode kernel
    bandwidth and the tail waste of partially filled last blocks."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    out = {"study": "block_size", "rows": []}
    for bs in (4, 8, 16, 32, 64):
        wl = workloads.mix(block_size=bs, steps=1)
        steps = list(wl.steps)
        r = PagedKVRunner.for_shape(wl.shape, 8256 // bs + 2)
        r.run(steps[0])
        acts = r.plan(steps[1].ops)
        r.upload(acts)
        dev = [t.cuda() for t in (steps[1].k_new, steps[1].v_new, steps[1].q)]
        d = [a for a in acts if a.kind == "decode"][0]
        o = torch.empty(dev[2].shape, dtype=torch.float32, device="cuda")
        r.execute(acts, *dev)
        # pa_decode's plain launch (variant 2, batch order, 512-token splits),
        # and the runner's choice (kernel, split, longest first)
        ms = _events_ms(lambda: pa.pa_decode(o, dev[2], r.k_cache, r.v_cache, d.dev["tables"],
                                             d.dev["lens"], r.scale, max_seq_len=d.max_len),
                        reps=20)
        ms_c = _events_ms(lambda: pa.pa_decode(o, dev[2], r.k_cache, r.v_cache, d.dev["tables"],
                                               d.dev["lens"], r.scale, max_seq_len=d.max_len,
                                               partition_size=d.partition, variant=d.variant,
                                               heads_per_cta=d.hpc,
                                               seq_order=d.dev.get("order")), reps=20)
        kvb = kv_bytes(d.lens, 8, 128, 2)
        st = r.alloc.stats()
        out["rows"].append({"block_size": bs, "decode_us": round(ms * 1e3, 2),
                            "kv_GBs": round(kvb / ms / 1e6, 1),
                            "chosen_decode_us": round(ms_c * 1e3, 2),
                            "chosen_kv_GBs": round(kvb / ms_c / 1e6, 1),
                            "chosen": {"kernel": DECODE_KERNELS[d.variant or 2][0],
                                       "partition": d.partition, "heads_per_cta": d.hpc},
                            "kernel": "tensor-core, " + ("cp.async" if bs < 8 else "TMA"),
                            "reserved_slots": st["reserved_slots"],
                            "logical_tokens": st["logical_tokens"],
                            "tail_waste_frac": round(1 - st["logical_tokens"] / st["reserved_slots"], 5),
                            "table_entries": st["table_entries"]})
        del r
        torch.cuda.empty_cache()
    return out


def _bf16_peak_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback 1.59 PFLOP/s"


def prefill_rows(ctx: int, chunk: int, batch: int = 8, dtype: str = "bf16",
                 variants=((1, "mma.sync"), (2, "tcgen05"), (3, "tcgen05 persistent"),
                           (4, "tcgen05, one fp16 P"))):
    """The prefill kernels (mma.sync, tcgen05, tcgen05 persistent, tcgen05 with
    one fp16 P) on one chunked-prefill workload (32/8 heads, D 128, bf16, bs 16): CUDA-event ms
    over 20 launches each, the definition's FLOPs (4 * D * Hq per (row,
    attended key)) and the kernels' full-size agreement."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    wl = workloads.chunked_prefill(batch=batch, ctx_lo=ctx, ctx_hi=ctx, chunk_lo=chunk,
                                   chunk_hi=chunk, dtype=dtype,
                                   num_blocks=batch * (ctx + chunk) // 16 + 64)
    steps = list(wl.steps)
    r = PagedKVRunner.for_shape(wl.shape, (ctx + chunk) // 16 + 2)
    r.run(steps[0])
    st = steps[1]
    acts = r.plan(st.ops)
    r.upload(acts)
    dev = [t.cuda() for t in (st.k_new, st.v_new, st.q)]
    r.execute(acts, *dev)
    a = [x for x in acts if x.kind == "prefill"][0]
    o = torch.empty((int(a.cu[-1]), 32, 128), dtype=torch.float32, device="cuda")
    flops = 4.0 * 128 * 32 * sum(ctx + i + 1 for i in range(chunk)) * batch
    peak, _ = _bf16_peak_tflops()
    rows = []
    first = None
    for variant, kernel in variants:
        ms = _events_ms(lambda: pa.pa_prefill(o, dev[2], r.k_cache, r.v_cache, a.dev["tables"],
                                              a.dev["lens"], a.dev["cu"], r.scale,
                                              max_q_len=a.max_q, max_seq_len=a.max_len,
                                              variant=variant), reps=20)
        tf = flops / (ms * 1e-3) / 1e12
        row = {"kernel": kernel, "context": ctx, "chunk": chunk, "batch": batch,
               "dtype": dtype, "ms": round(ms, 3), "tflops": round(tf, 1),
               "frac_of_bf16_peak": round(tf / peak, 4), "peak_tflops": peak,
               "flops_per_launch": flops}
        if first is None:
            first, first_kernel = o.clone(), kernel
        else:  # the kernels compute the same rows at full size
            row[f"max_abs_diff_vs_{first_kernel.replace('.', '_').replace(' ', '_')}"] = \
                float((o - first).abs().max())
        rows.append(row)
    del r
    torch.cuda.empty_cache()
    return rows


def study_prefill(args):
    """Chunked prefill, every kernel: 8 sequences x (4096 context + 1024
    chunk), (0 + 4096), (16384 + 512); 32/8 heads, D 128, bf16, bs 16."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    res = {"study": "prefill", "rows": []}
    for ctx, chunk in ((4096, 1024), (0, 4096), (16384, 512)):
        res["rows"] += prefill_rows(ctx, chunk)
    res["device_errors"] = pa.device_errors()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="long32k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--sync-e2e", action="store_true",
                    help="e2e: wait for each step's output before launching the next")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the chunked-prefill line added to the N = 1 bench output")
    ap.add_argument("--e2e-python", action="store_true",
                    help="e2e through the Python runner instead of the native runtime")
    ap.add_argument("--no-graph", action="store_true",
                    help="e2e: launch every step eagerly instead of replaying CUDA graphs")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--study", default="", choices=["", "prefix", "swap", "blocksize", "prefill"],
                    help="print one of the side studies instead of the bench line")
    ap.add_argument("--partition", type=int, default=-1,
                    help="split length in tokens: -1 chosen per step from the lengths "
                         "(pa_decode_partition_for), 0 the library default (512), or a "
                         "multiple of 64 in [64, 1024]")
    ap.add_argument("--main-launches", type=int, default=32,
                    help="launches of the main decode kernel timed alone after the steps")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations' lines (Llama-8B-shaped, beam, mix)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (small cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.study:
        fn = {"prefix": study_prefix, "swap": study_swap, "blocksize": study_blocksize,
              "prefill": study_prefill}[args.study]
        print(json.dumps(fn(args)), flush=True)
        return
    ws, rank, local, _ = dist_setup()
    try:
        if args.impl == "reference":
            res = run_reference(args, ws, rank)
        else:
            res = run_ours(args, ws, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
