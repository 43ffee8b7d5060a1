"""Benchmark of the sparse-MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload c5] [--no-per-config] [--calls N]

(--calls N: only N plain decode calls of the workload, for profilers.)

One step = one sparse_mla_decode call (the split kernel, plus the combine
kernel when the plan merges splits that way) over one batch of the workload,
inputs resident in HBM.  The headline workload is c5 (B=128, top-2048, paged
fp8 cache): the largest configuration, on one GPU.

Timing.  Workloads whose cache is larger than L2 (c3, c5, DeepSeek-V4 pages,
multi-token) run their K steps back to back under one pair of CUDA events on
the launching stream, rotating through nb batches that share the cache but
draw their own queries and index lists (inputs.reindexed), nb chosen so that
the rows gathered by one rotation exceed twice the L2 size: each step finds
its rows out of L2.  Workloads whose whole cache fits in L2 (c1, c2, c4)
cannot leave L2 that way: before every step L2 is flushed (a write of 2x L2,
then a read of another 2x L2 buffer, so that no dirty flush lines are left
to be written back inside the timed call), untimed, and each step is timed
with its own event pair.  config.l2 says which.  With N > 1 (torchrun) every
rank runs the workload on its own batch of sequences (the op shards over
batch with no exchange step; rank r draws its batch with inputs.shard_seed):
weak scaling, value = bytes of all ranks over the max-over-ranks time.  Rank
0 prints one JSON line.

Keys beyond the base contract:
  roofline     the split kernel (the whole step when it does not split) vs
               the measured HBM copy peak; traffic from the committed ncu
               summary of the same kernel sources, else null
  cpu_baseline the fp64 oracle timed on host cores on a bounded sample
  e2e          the same metric through sparse_mla_decode_host: q / indices
               (and page table) copied host -> device from pinned memory and
               out / lse back inside the timed region of every step,
               pipelined over four streams (serial: one stream)
  per_config   every workload (c1-c5, DeepSeek-V4 pages, multi-token, the
               indexer step): us per step timed as above, plus a cold single
               call after a flush, and the fraction of roofline
  clocks       SM clock / throttle reasons sampled during the timed region
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mla_decode_05_b200 import inputs  # noqa: E402

METRIC = "sparse-MLA decode µs/call and gathered-KV HBM GB/s (% of roofline) vs batch"
HEADLINE = "c5"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------- clocks
_REASON_BITS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}


def _nvml_sampler(conn, busid: str, period_s: float):
    """Runs in a spawned process: samples the SM clock and the clock event
    reasons of one GPU through NVML until told to stop."""
    import time as _t
    import pynvml
    pynvml.nvmlInit()
    h = pynvml.nvmlDeviceGetHandleByPciBusId(busid)
    reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
        pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
    maxsm = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    samples = []
    conn.send("ready")
    while not conn.poll(0):
        samples.append((_t.time(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), int(reasons(h))))
        _t.sleep(period_s)
    conn.recv()
    conn.send((maxsm, samples))


class ClockSampler:
    """Samples clocks in a separate process (no GIL contention with the timed
    loop); summary() keeps the samples taken inside [t0, t1]."""

    def __init__(self, device):
        self.proc = None
        self.conn = None
        try:
            import multiprocessing as mp
            pr = torch.cuda.get_device_properties(device)
            busid = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            ctx = mp.get_context("spawn")
            self.conn, child = ctx.Pipe()
            self.proc = ctx.Process(target=_nvml_sampler, args=(child, busid, 0.001), daemon=True)
            self.proc.start()
            if not self.conn.poll(60) or self.conn.recv() != "ready":
                raise RuntimeError("sampler did not start")
        except Exception as e:  # no NVML: report clocks as unavailable
            self.error = str(e)
            self.proc = None

    def summary(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML sampler unavailable: " + getattr(self, "error", "")}
        self.conn.send("stop")
        maxsm, samples = self.conn.recv()
        self.proc.join(timeout=10)
        inside = [x for x in samples if t0 <= x[0] <= t1]
        if not inside:  # the region was shorter than one sample: take the nearest
            inside = sorted(samples, key=lambda x: min(abs(x[0] - t0), abs(x[0] - t1)))[:1]
        reasons = sorted({name for _, _, r in inside for bit, name in _REASON_BITS.items() if r & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside) if inside else None, "sm_max_mhz": maxsm,
                "reasons": reasons, "samples": len(inside)}


# --------------------------------------------------------------- helpers
KERNEL_SOURCES = [os.path.join(ROOT, "sparse_mla_decode_05_b200", "csrc", "sparse_mla.cu"),
                  os.path.join(ROOT, "sparse_mla_decode_05_b200", "csrc", "indexer.cuh"),
                  os.path.join(ROOT, "include", "sparse_mla.h")]


def kernel_source_hash() -> str:
    """sha256 over every source compiled into the kernels, in a fixed order."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        h.update(open(p, "rb").read())
    return h.hexdigest()


def kernel_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the split kernel on
    `workload`, from the committed ncu summary
    profiles/smla_split_kernel_<workload>_dram.md; None when there is none or
    it was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"smla_split_kernel_{workload}_dram.md")
    try:
        text = open(path).read()
        src = kernel_source_hash()
    except OSError:
        return None
    m_sha = re.search(r"kernel sources sha256: `?([0-9a-f]{64})", text)
    m_b = re.search(r"dram bytes per launch: `?(\d+)", text)
    if not (m_sha and m_b) or m_sha.group(1) != src:
        return None
    return int(m_b.group(1))


def reduce_over_ranks(x: float, op: str, device) -> float:
    """max or sum of a host float over all ranks of the default process group
    (the value itself without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def roofline_us(ab, fl, peak_gbs, peak_tflops):
    return max(ab / (peak_gbs * 1e3), fl / (peak_tflops * 1e6))


def cache_bytes(w: inputs.Workload) -> int:
    n = w.kv.numel() * w.kv.element_size()
    return n + (0 if w.kv_row_scale is None else w.kv_row_scale.numel() * 4)


class Flusher:
    """Evicts L2 between timed steps: a write of 2x L2 (the flush), then a
    read of another 2x L2 buffer, which writes the flush's dirty lines back
    before the timed call instead of during it."""

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.l2 = l2
        self.w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        self.r = torch.ones(2 * l2 // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.r.sum(dtype=torch.int32)


class Batches:
    """nb batches of one workload on the device, sharing the cache (pool, row
    scales, page tables), each with its own q / index lists and plan."""

    def __init__(self, w: inputs.Workload, dev, nb: int, seed0: int):
        from sparse_mla_decode_05_b200 import api
        self.w = w
        self.kv = w.kv.to(dev)
        self.rsc = None if w.kv_row_scale is None else w.kv_row_scale.to(dev)
        self.pt = None if w.page_table is None else w.page_table.to(dev)
        self.ws = [w] + [inputs.reindexed(w, seed0 + k) for k in range(1, nb)]
        self.plans = [api.DecodePlan(x.q.to(dev), self.kv, x.indices.to(dev), w.scale, kv_row_scale=self.rsc,
                                     page_table=self.pt, page_size=w.page_size) for x in self.ws]
        p0 = self.plans[0]
        self.nsplit, self.clustered, self.streamk = p0.nsplit, p0.clustered, p0.streamk
        self.launches_per_step = 1 + (1 if p0.nsplit > 1 and not p0.clustered else 0)
        self.alg_bytes = float(np.mean([inputs.algorithmic_bytes(x) for x in self.ws]))
        self.alg_flops = float(np.mean([inputs.algorithmic_flops(x) for x in self.ws]))

    def __len__(self):
        return len(self.plans)


def rotation_count(w: inputs.Workload, l2: int):
    """Batches to rotate so that one rotation gathers more than 2x L2 of rows,
    or None when the cache itself fits in 2x L2 (rotation cannot evict it)."""
    if cache_bytes(w) <= 2 * l2:
        return None
    return int(min(64, max(2, math.ceil(2 * l2 / inputs.algorithmic_bytes(w)))))


def time_back_to_back(fn_i, nb, steps, warmup, flusher, stream):
    """ms per step of steps back-to-back calls fn_i(i % nb), one event pair."""
    for i in range(warmup):
        fn_i(i % nb)
    flusher()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn_i(i % nb)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def time_flushed(fn_i, nb, steps, warmup, flusher, stream):
    """Per-step ms of fn_i(i % nb), L2 flushed before each step (untimed)."""
    for i in range(warmup):
        flusher()
        fn_i(i % nb)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        flusher()
        a.record(stream)
        fn_i(i % nb)
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_workload(bt: Batches, steps, warmup, flusher, stream):
    """(ms per step, l2 note): back to back over the rotation when the cache
    exceeds 2x L2, else flushed per step (mean)."""
    run = lambda i: bt.plans[i].run()
    if rotation_count(bt.w, flusher.l2) is not None:
        ms = time_back_to_back(run, len(bt), steps, warmup, flusher, stream)
        return ms, (f"inputs larger than L2: {len(bt)} batches over one {cache_bytes(bt.w) / 1e9:.2f} GB cache "
                    f"rotate, steps back to back")
    ts = time_flushed(run, len(bt), steps, warmup, flusher, stream)
    return float(np.mean(ts)), "flushed before every timed step (2x L2 write, then 2x L2 read; untimed)"


def cold_call_us(bt: Batches, reps, flusher, stream):
    """Median / p10 / p90 of one call after a flush (latency of a lone call)."""
    ts = time_flushed(lambda i: bt.plans[i].run(), len(bt), reps, 3, flusher, stream)
    return float(np.median(ts)) * 1e3, float(np.percentile(ts, 10)) * 1e3, float(np.percentile(ts, 90)) * 1e3


def oracle_time(w: inputs.Workload, budget_s: float = 15.0):
    """fp64 oracle on the host: returns (seconds per full-workload step
    estimated from a bounded sample, sample description, threads)."""
    from oracle import sparse_mla_ref as ref
    B = w.batch
    args = dict(d_v=w.d_v, kv_format=w.kv_format,
                kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.numpy(), page_size=w.page_size)
    qb, kv, idx = w.np_q_bits(), w.np_kv(), w.indices.numpy()
    pt = None if w.page_table is None else w.page_table.numpy()
    done, t_used, reps = 0, 0.0, 0
    t0 = time.perf_counter()
    while t_used < budget_s and reps < 1000:
        for b in range(B):
            if w.tokens > 1:
                ref.sparse_mla_decode_multi_token(qb[b:b + 1], kv, idx[b:b + 1], w.scale,
                                                  page_table=None if pt is None else pt[b:b + 1], **args)
            else:
                ref.sparse_mla_decode(qb, kv, idx, w.scale, seqs=[b], page_table=pt, **args)
            done += 1
            t_used = time.perf_counter() - t0
            if t_used >= budget_s:
                break
        reps += 1
    per_seq = t_used / max(done, 1)
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    return per_seq * B, f"{done} sequences of {w.name} (whole workload = {B} sequences), {t_used:.1f} s", threads


def describe(name):
    return {**inputs.CONFIG_DESCRIPTIONS, **inputs.EXTRA_DESCRIPTIONS}[name]


# --------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=list(inputs.CONFIG_NAMES + inputs.EXTRA_NAMES))
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--oracle-budget", type=float, default=15.0)
    ap.add_argument("--calls", type=int, default=0,
                    help="only make this many plain decode calls of the workload and exit (for profilers)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peak_gbs, peak_tf, peak_tf_sus, peak_src = load_peaks()
    w = inputs.make_config(args.workload, seed=inputs.shard_seed(args.workload, rank))
    config = {"workload": f"{args.workload}: {describe(args.workload)}", "batch": w.batch,
              "tokens_per_seq": w.tokens, "topk": w.topk, "heads": 64, "d_qk": int(w.q.shape[-1]), "d_v": 512,
              "kv_dtype": w.kv_format, "paged": w.page_size > 0,
              "parallelism": f"batch shards x{world} (weak, no collective)" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return
        sec_per_step, sample, threads = oracle_time(w, budget_s=min(args.oracle_budget, 20.0))
        val = inputs.algorithmic_bytes(w) / sec_per_step / 1e9
        config["l2"] = "not applicable (host oracle)"
        line = {"metric": METRIC, "value": val, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if args.calls > 0:
        # a plain run for profilers: the workload's decode, args.calls times
        from sparse_mla_decode_05_b200 import api
        dev = torch.device("cuda", local)
        plan = api.DecodePlan(w.q.to(dev), w.kv.to(dev), w.indices.to(dev), w.scale,
                              kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.to(dev),
                              page_table=None if w.page_table is None else w.page_table.to(dev),
                              page_size=w.page_size)
        for _ in range(args.calls):
            plan.run()
        torch.cuda.synchronize()
        assert api.device_error() == 0, "device error word set"
        print(json.dumps({"calls": args.calls, "workload": args.workload, "nsplit": plan.nsplit}))
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    from sparse_mla_decode_05_b200 import api

    flusher = Flusher(dev)
    l2 = flusher.l2
    nb = rotation_count(w, l2) or 1
    bt = Batches(w, dev, nb, seed0=1000 * 31 + 100_000 * rank)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    # --- headline: device-resident inputs, whole call, K timed steps
    clk = ClockSampler(dev)
    barrier()
    t_wall0 = time.perf_counter()
    t_clk0 = time.time()
    ms, l2_note = time_workload(bt, args.steps, args.warmup, flusher, stream)
    barrier()
    t_clk1 = time.time()
    t_wall = time.perf_counter() - t_wall0
    clocks = clk.summary(t_clk0, t_clk1)
    config["l2"] = l2_note
    ms = reduce_over_ranks(ms, "max", dev)
    job_bytes = reduce_over_ranks(bt.alg_bytes, "sum", dev)
    value = job_bytes / (ms * 1e-3) / 1e9

    # --- dominant kernel: the split kernel (the whole step without a combine)
    if bt.launches_per_step == 1:
        sp_ms = ms
    else:
        run_split = lambda i: bt.plans[i].run_split()
        if rotation_count(w, l2) is not None:
            sp_ms = time_back_to_back(run_split, len(bt), max(10, args.steps // 2), 3, flusher, stream)
        else:
            sp_ms = float(np.mean(time_flushed(run_split, len(bt), max(10, args.steps // 2), 3, flusher, stream)))
    achieved = bt.alg_bytes / (sp_ms * 1e-3) / 1e9
    rl_us = roofline_us(bt.alg_bytes, bt.alg_flops, peak_gbs, peak_tf)
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak_gbs, "unit": "GB/s", "frac": achieved / peak_gbs,
            "traffic": kernel_traffic(args.workload), "algorithmic_bytes": bt.alg_bytes,
            "kernel": "smla_split_kernel", "peak_source": f"{peak_src} (copy)",
            "split_kernel_us": sp_ms * 1e3, "nsplit": bt.nsplit,
            "split_reduction": ("stream-K (rows shared by up to 3 CTAs, merged by the last)" if bt.streamk else
                                "cluster (on chip)" if bt.clustered else
                                ("partials + combine" if bt.nsplit > 1 else "none")),
            "roofline_us": rl_us, "frac_of_step_roofline": rl_us / (ms * 1e3),
            "frac_vs_nominal_8TBps": achieved / 8000.0,
            "note": "achieved = algorithmic bytes per launch / mean launch time over the timed region"}

    # --- end to end through the host-buffer call (sparse_mla_decode_host):
    #     every step copies its q and index lists (+ page table) host ->
    #     device from pinned memory, decodes, and copies out + lse back.
    #     Pipelined over four streams (the value): the rotation's batches, a
    #     batch per step in turn, its own staging; serial: one stream.
    def host_plan(wb):
        return api.HostDecodePlan(wb.q.pin_memory(), bt.kv, wb.indices.pin_memory(), wb.scale,
                                  kv_row_scale=bt.rsc,
                                  page_table_host=None if wb.page_table is None else wb.page_table.pin_memory(),
                                  page_size=wb.page_size)

    n_streams = 4
    hb = max(n_streams, len(bt))
    hb += (-hb) % n_streams                               # each plan stays on one stream
    hws = [bt.ws[k % len(bt)] if k < len(bt) else inputs.reindexed(w, 777 + k) for k in range(hb)]
    hplans = [host_plan(x) for x in hws]
    h2d = w.q.numel() * 2 + w.indices.numel() * 4 + (0 if w.page_table is None else w.page_table.numel() * 4)
    d2h = hplans[0].out_host.numel() * 2 + hplans[0].lse_host.numel() * 4
    streams = [torch.cuda.Stream(dev) for _ in range(n_streams)]

    def pipelined(k_steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(streams[0])
        for s in streams[1:]:
            s.wait_event(t0)
        for i in range(k_steps):
            hplans[i % hb].run(streams[i % n_streams])
        for s in streams[1:]:
            j = torch.cuda.Event()
            j.record(s)
            streams[0].wait_event(j)
        t1.record(streams[0])
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    pipelined(2 * hb)                                     # warm-up
    k_pipe = max(4 * hb, args.steps)
    pipe_ms = reduce_over_ranks(pipelined(k_pipe) / k_pipe, "max", dev)
    ser = time_flushed(lambda i: hplans[i % hb].run(), hb, max(10, args.steps // 4), 3, flusher, stream)
    ser_ms = reduce_over_ranks(float(np.mean(ser)), "max", dev)
    e2e = {"value": job_bytes / (pipe_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": pipe_ms, "call": "sparse_mla_decode_host",
           "pipelined": {"streams": n_streams, "distinct_batches": hb, "steps": k_pipe},
           "serial": {"value": job_bytes / (ser_ms * 1e-3) / 1e9, "ms_per_step": ser_ms,
                      "l2": "flushed before every step (untimed)"}}
    del hplans, hws
    torch.cuda.empty_cache()
    assert api.device_error() == 0, "device error word set"

    # --- cold single call and 8 calls in one CUDA graph (a serving loop
    #     over layers; programmatic dependent launch lets each call's
    #     prologue overlap the previous call's tail), L2 flushed before each
    cold = cold_call_us(bt, 30, flusher, stream)
    b2b = None
    if rank == 0 and world == 1 and not args.no_per_config:
        calls = 8
        graph_plans = [bt.plans[k % len(bt)] for k in range(calls)]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for p in graph_plans:
                p.run(torch.cuda.current_stream(dev).cuda_stream)
        gt = time_flushed(lambda i: graph.replay(), 1, 30, 3, flusher, stream)
        b2b = {"calls": calls, "us_per_call": float(np.median(gt)) * 1e3 / calls,
               "note": f"{calls} calls in one CUDA graph, L2 flushed before each replay"}
        del graph
        torch.cuda.empty_cache()
        assert api.device_error() == 0, "device error word set"

    # --- every workload at 1 GPU (rank 0 only)
    per_config = None
    if rank == 0 and world == 1 and not args.no_per_config:
        per_config = []
        for name in inputs.CONFIG_NAMES + inputs.EXTRA_NAMES:
            if name == args.workload:
                bc = bt
            else:
                wc = inputs.make_config(name)
                bc = Batches(wc, dev, rotation_count(wc, l2) or 1, seed0=1000 * 47)
            k = 30 if rotation_count(bc.w, l2) is None else max(40, 4 * len(bc))
            mc, note = time_workload(bc, k, 3, flusher, stream)
            med, p10, p90 = cold_call_us(bc, 20, flusher, stream)
            ab, fl = bc.alg_bytes, bc.alg_flops
            rl = roofline_us(ab, fl, peak_gbs, peak_tf)
            per_config.append({"workload": name, "batch": bc.w.batch, "tokens_per_seq": bc.w.tokens,
                               "topk": bc.w.topk, "nsplit": bc.nsplit, "clustered": bc.clustered,
                               "streamk": bc.streamk,
                               "us_per_step": mc * 1e3, "gbs": ab / (mc * 1e-3) / 1e9, "roofline_us": rl,
                               "frac_roofline": rl / (mc * 1e3), "timing": note,
                               "cold_call_us": med, "cold_p10_us": p10, "cold_p90_us": p90,
                               "alg_bytes": ab, "alg_flops": fl})
            if bc is not bt:
                del bc
                torch.cuda.empty_cache()
        # the indexer step that produces the index lists (scores + top-k);
        # its 67 MB key cache fits in L2: flushed per step
        wi = inputs.make_indexer_config()
        ip = api.IndexerPlan(wi.q.to(dev), wi.w.to(dev), wi.k.to(dev), wi.page_table.to(dev),
                             wi.ctx_len.to(dev), wi.topk, max_ctx=wi.max_ctx)
        tms = time_flushed(lambda i: ip.run(), 1, 30, 3, flusher, stream)
        med = float(np.median(tms)) * 1e3
        ab = inputs.indexer_algorithmic_bytes(wi)
        fl = 2 * wi.q.shape[1] * wi.q.shape[2] * int(wi.ctx_len.sum())
        rl = max(ab / (peak_gbs * 1e3), fl / (peak_tf * 1e6))
        per_config.append({"workload": "indexer", "description": inputs.INDEXER_DESCRIPTION, "batch": wi.batch,
                           "topk": wi.topk, "max_ctx": wi.max_ctx, "us_per_step": med,
                           "p10_us": float(np.percentile(tms, 10)) * 1e3,
                           "p90_us": float(np.percentile(tms, 90)) * 1e3,
                           "gbs": ab / (med * 1e-6) / 1e9, "roofline_us": rl, "frac_roofline": rl / med,
                           "timing": "flushed before every timed step",
                           "scores_kernel_us": float(np.median(time_flushed(lambda i: ip.run_scores(), 1, 15, 3, flusher, stream))) * 1e3,
                           "topk_kernel_us": float(np.median(time_flushed(lambda i: ip.run_topk(), 1, 15, 3, flusher, stream))) * 1e3,
                           "alg_bytes": ab, "alg_flops": fl})
        del ip
        torch.cuda.empty_cache()
        assert api.device_error() == 0, "device error word set"

    # --- CPU baseline: the oracle on host cores, bounded sample
    cpu = None
    if rank == 0 and world == 1:
        sec, sample, threads = oracle_time(w, budget_s=args.oracle_budget)
        cpu = {"value": inputs.algorithmic_bytes(w) / sec / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": sample}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": bt.launches_per_step * args.steps, "clocks": clocks,
                "cold_call_us": {"median": cold[0], "p10": cold[1], "p90": cold[2]}, "back_to_back": b2b,
                "wall_s_timed_region": t_wall, "per_config": per_config}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
