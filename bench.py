"""Benchmark of the sparse-MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload c2] [--no-per-config]

One step = one sparse_mla_decode call (split kernel + combine when the plan
splits) over one batch of the headline workload, inputs resident in HBM.
L2 is flushed (a write of 2x the L2 size) before every timed step, outside
the timed region; each step is timed with CUDA events on the launching
stream.  With N > 1 (torchrun) every rank runs the workload on its own batch
of sequences (the op shards over batch with no exchange step; rank r draws
its batch with inputs.shard_seed): weak scaling, value = bytes of all ranks
over the max-over-ranks time.  Rank 0 prints one JSON line.

Keys beyond the base contract:
  roofline     dominant kernel (the split kernel) vs the measured HBM peak
  cpu_baseline the fp64 oracle timed on host cores on a bounded sample
  e2e          same metric through sparse_mla_decode_host: q / indices
               copied host -> device from pinned memory and out / lse back
               inside the timed region of every step; the value pipelines
               steps over four streams (serial: one stream, in "serial")
  per_config   microseconds per call and GB/s for every workload (the six
               headline configs, DeepSeek-V4 pages, and the indexer step
               that produces the index lists), vs roofline
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
HEADLINE = "c2"


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
KERNEL_SOURCE = os.path.join(ROOT, "sparse_mla_decode_05_b200", "csrc", "sparse_mla.cu")


def kernel_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the split kernel on `workload`,
    from the committed ncu summary profiles/smla_split_kernel_<workload>_dram.md;
    None when there is none or it was taken on another kernel source."""
    path = os.path.join(ROOT, "profiles", f"smla_split_kernel_{workload}_dram.md")
    try:
        text = open(path).read()
        src = hashlib.sha256(open(KERNEL_SOURCE, "rb").read()).hexdigest()
    except OSError:
        return None
    m_sha = re.search(r"kernel source sha256: `?([0-9a-f]{64})", text)
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


def to_dev(w: inputs.Workload, dev):
    return dict(q=w.q.to(dev), kv=w.kv.to(dev), indices=w.indices.to(dev),
                kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.to(dev),
                page_table=None if w.page_table is None else w.page_table.to(dev))


def roofline_us(w, peak_gbs, peak_tflops):
    return max(inputs.algorithmic_bytes(w) / (peak_gbs * 1e3), inputs.algorithmic_flops(w) / (peak_tflops * 1e6))


class Runner:
    """One workload on one device with a pre-marshalled decode call."""

    def __init__(self, w, dev):
        from sparse_mla_decode_05_b200 import api
        self.api = api
        self.w = w
        self.t = to_dev(w, dev)
        t = self.t
        self.plan = api.DecodePlan(t["q"], t["kv"], t["indices"], w.scale, kv_row_scale=t["kv_row_scale"],
                                   page_table=t["page_table"], page_size=w.page_size)
        self.nsplit = self.plan.nsplit
        self.out, self.lse = self.plan.out, self.plan.lse

    def decode(self):
        self.plan.run()

    def split_only(self):
        self.plan.run_split()

    def combine_only(self):
        self.plan.run_combine()

    @property
    def launches_per_step(self):
        return 1 + (1 if self.nsplit > 1 and not self.plan.clustered else 0)


def time_device(fn, steps, warmup, flush, stream):
    """Per-step CUDA-event times (ms) of fn(), L2 flushed before each step."""
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_split_breakdown(r: Runner, steps, flush, stream):
    """Per-step times (ms) of the split kernel and of the combine kernel,
    each bracketed by events on the launching stream."""
    sp, cb = [], []
    for _ in range(steps):
        flush.zero_()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        r.split_only()
        e1.record(stream)
        if r.nsplit > 1:
            r.combine_only()
        e2.record(stream)
        sp.append((e0, e1))
        cb.append((e1, e2))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in sp], [a.elapsed_time(b) for a, b in cb]


def oracle_time(w: inputs.Workload, budget_s: float = 15.0):
    """fp64 oracle on the host: returns (seconds per full-workload step
    estimated from a bounded sample, sample description, threads)."""
    from oracle import sparse_mla_ref as ref
    B = w.batch
    args = dict(d_v=w.d_v, kv_format=w.kv_format,
                kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.numpy(),
                page_table=None if w.page_table is None else w.page_table.numpy(), page_size=w.page_size)
    qb, kv, idx = w.np_q_bits(), w.np_kv(), w.indices.numpy()
    done, t_used, reps = 0, 0.0, 0
    t0 = time.perf_counter()
    while t_used < budget_s and reps < 1000:
        for b in range(B):
            ref.sparse_mla_decode(qb, kv, idx, w.scale, seqs=[b], **args)
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
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peak_gbs, peak_tf, peak_tf_sus, peak_src = load_peaks()
    w = inputs.make_config(args.workload, seed=inputs.shard_seed(args.workload, rank))
    alg_bytes = inputs.algorithmic_bytes(w)
    alg_flops = inputs.algorithmic_flops(w)
    desc = {**inputs.CONFIG_DESCRIPTIONS, **inputs.EXTRA_DESCRIPTIONS}[args.workload]
    config = {"workload": f"{args.workload}: {desc}", "batch": w.batch,
              "topk": w.topk, "heads": 64, "d_qk": int(w.q.shape[2]), "d_v": 512, "kv_dtype": w.kv_format,
              "paged": w.page_size > 0, "l2": "flushed before every timed step (2x L2 write, untimed)",
              "parallelism": f"batch shards x{world} (weak, no collective)" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return
        sec_per_step, sample, threads = oracle_time(w, budget_s=min(args.oracle_budget, 20.0))
        steps = args.steps
        val = alg_bytes / sec_per_step / 1e9
        line = {"metric": METRIC, "value": val, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
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

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    r = Runner(w, dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    # --- headline: device-resident inputs, whole call
    clk = ClockSampler(dev)
    barrier()
    t_wall0 = time.perf_counter()
    t_clk0 = time.time()
    times = time_device(r.decode, args.steps, args.warmup, flush, stream)
    barrier()
    t_clk1 = time.time()
    t_wall = time.perf_counter() - t_wall0
    clocks = clk.summary(t_clk0, t_clk1)
    ms = reduce_over_ranks(float(np.mean(times)), "max", dev)
    job_bytes = reduce_over_ranks(alg_bytes, "sum", dev)
    value = job_bytes / (ms * 1e-3) / 1e9

    # --- dominant kernel (split) and combine, each timed on its own
    sp, cb = time_split_breakdown(r, max(10, args.steps // 2), flush, stream)
    sp_ms = float(np.mean(sp))
    cb_ms = float(np.mean(cb)) if r.nsplit > 1 and not r.plan.clustered else 0.0
    achieved = alg_bytes / (sp_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak_gbs, "unit": "GB/s", "frac": achieved / peak_gbs,
            "traffic": kernel_traffic(args.workload), "algorithmic_bytes": alg_bytes, "kernel": "smla_split_kernel", "peak_source": f"{peak_src} (burst copy)",
            "split_kernel_us": sp_ms * 1e3, "combine_kernel_us": cb_ms * 1e3, "nsplit": r.nsplit,
            "split_reduction": "cluster (on chip)" if r.plan.clustered else ("partials + combine" if r.nsplit > 1 else "none"),
            "roofline_us": roofline_us(w, peak_gbs, peak_tf),
            "frac_of_step_roofline": roofline_us(w, peak_gbs, peak_tf) / (ms * 1e3),
            "frac_vs_nominal_8TBps": achieved / 8000.0}

    # --- end to end through the host-buffer call (sparse_mla_decode_host):
    #     every step copies its q and indices (+ page table) host -> device
    #     from pinned memory, decodes, and copies out + lse device -> host.
    #     (a) serial: one stream, L2 flushed before each step (untimed),
    #         CUDA events around each step;
    #     (b) pipelined (the value): four streams, nb distinct batches with
    #         their own caches, so a batch's rows have left L2 before it comes
    #         round again (no flush); step i runs batch i % nb on stream
    #         i % 4, one event pair around all steps.  One step's copies
    #         overlap other streams' decodes and copies in the other
    #         direction (measured on B200: 1 stream 97 us, 2 streams 56 us,
    #         4 streams 49 us per c2 step).
    def host_plan(wb, tb):
        return api.HostDecodePlan(wb.q.pin_memory(), tb["kv"], wb.indices.pin_memory(), wb.scale,
                                  kv_row_scale=tb["kv_row_scale"],
                                  page_table_host=None if wb.page_table is None else wb.page_table.pin_memory(),
                                  page_size=wb.page_size)

    hp = host_plan(w, r.t)
    h2d = w.q.numel() * 2 + w.indices.numel() * 4 + (0 if w.page_table is None else w.page_table.numel() * 4)
    d2h = hp.out_host.numel() * 2 + hp.lse_host.numel() * 4
    ser = time_device(hp.run, max(10, args.steps // 2), 3, flush, stream)
    ser_ms = reduce_over_ranks(float(np.mean(ser)), "max", dev)

    n_streams = 4
    nb = int(min(16, max(n_streams, math.ceil(1.5 * l2 / alg_bytes) + 1)))
    nb += (-nb) % n_streams                               # each plan stays on one stream
    extra = [inputs.make_config(args.workload, seed=1000 * (k + 31) + 100_000 * rank) for k in range(1, nb)]
    extra_t = [to_dev(b, dev) for b in extra]
    plans = [hp] + [host_plan(b, t) for b, t in zip(extra, extra_t)]
    cache_gb = sum(t["kv"].numel() * t["kv"].element_size() for t in [r.t] + extra_t) / 1e9
    streams = [torch.cuda.Stream(dev) for _ in range(n_streams)]

    def pipelined(k_steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(streams[0])
        for s in streams[1:]:
            s.wait_event(t0)
        for i in range(k_steps):
            plans[i % nb].run(streams[i % n_streams])
        for s in streams[1:]:
            j = torch.cuda.Event()
            j.record(s)
            streams[0].wait_event(j)
        t1.record(streams[0])
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    pipelined(2 * nb)                                     # warm-up
    k_pipe = max(4 * nb, args.steps)
    pipe_ms = reduce_over_ranks(pipelined(k_pipe) / k_pipe, "max", dev)
    e2e = {"value": job_bytes / (pipe_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": pipe_ms, "call": "sparse_mla_decode_host",
           "pipelined": {"streams": n_streams, "distinct_batches": nb, "steps": k_pipe,
                         "l2": f"no flush: {nb} batches with their own caches ({cache_gb:.2f} GB) > L2"},
           "serial": {"value": job_bytes / (ser_ms * 1e-3) / 1e9, "ms_per_step": ser_ms,
                      "l2": "flushed before every step (untimed)"}}
    del plans, extra, extra_t, hp
    torch.cuda.empty_cache()
    assert api.device_error() == 0, "device error word set"

    # --- back to back: 8 calls on 8 distinct batches of the workload in one
    #     CUDA graph (a serving loop over layers); programmatic dependent
    #     launch lets each call's prologue overlap the previous call's tail.
    #     L2 is flushed before every replay.
    b2b = None
    if rank == 0 and world == 1 and not args.no_per_config:
        calls = 8
        runners = [r] + [Runner(inputs.make_config(args.workload, seed=1000 * (k + 7)), dev) for k in range(1, calls)]
        for rr in runners:
            rr.decode()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for rr in runners:
                rr.plan.run(torch.cuda.current_stream(dev).cuda_stream)
        gt = time_device(graph.replay, 30, 3, flush, stream)
        b2b = {"calls": calls, "us_per_call": float(np.median(gt)) * 1e3 / calls,
               "note": f"{calls} calls on {calls} distinct {args.workload} batches in one CUDA graph, "
                       "L2 flushed before each replay"}
        del graph, runners
        torch.cuda.empty_cache()
        assert api.device_error() == 0, "device error word set"

    # --- every workload at 1 GPU (rank 0 only)
    per_config = None
    if rank == 0 and world == 1 and not args.no_per_config:
        per_config = []
        for name in inputs.CONFIG_NAMES + inputs.EXTRA_NAMES:
            wc = w if name == args.workload else inputs.make_config(name)
            rc = r if name == args.workload else Runner(wc, dev)
            tms = time_device(rc.decode, 30, 3, flush, stream)
            med = float(np.median(tms)) * 1e3
            p10, p90 = float(np.percentile(tms, 10)) * 1e3, float(np.percentile(tms, 90)) * 1e3
            spc, _ = time_split_breakdown(rc, 15, flush, stream)
            ab = inputs.algorithmic_bytes(wc)
            rl = roofline_us(wc, peak_gbs, peak_tf)
            per_config.append({"workload": name, "batch": wc.batch, "topk": wc.topk, "nsplit": rc.nsplit,
                               "clustered": rc.plan.clustered,
                               "us_per_call": med, "p10_us": p10, "p90_us": p90,
                               "gbs": ab / (med * 1e-6) / 1e9, "roofline_us": rl, "frac_roofline": rl / med,
                               "split_kernel_us": float(np.median(spc)) * 1e3,
                               "alg_bytes": ab, "alg_flops": inputs.algorithmic_flops(wc)})
            if rc is not r:
                del rc
                torch.cuda.empty_cache()
        # the indexer step that produces the index lists (scores + top-k)
        wi = inputs.make_indexer_config()
        ip = api.IndexerPlan(wi.q.to(dev), wi.w.to(dev), wi.k.to(dev), wi.page_table.to(dev),
                             wi.ctx_len.to(dev), wi.topk, max_ctx=wi.max_ctx)
        tms = time_device(ip.run, 30, 3, flush, stream)
        med = float(np.median(tms)) * 1e3
        ab = inputs.indexer_algorithmic_bytes(wi)
        fl = 2 * wi.q.shape[1] * wi.q.shape[2] * int(wi.ctx_len.sum())
        rl = max(ab / (peak_gbs * 1e3), fl / (peak_tf * 1e6))
        per_config.append({"workload": "indexer", "description": inputs.INDEXER_DESCRIPTION, "batch": wi.batch,
                           "topk": wi.topk, "max_ctx": wi.max_ctx, "us_per_call": med,
                           "p10_us": float(np.percentile(tms, 10)) * 1e3,
                           "p90_us": float(np.percentile(tms, 90)) * 1e3,
                           "gbs": ab / (med * 1e-6) / 1e9, "roofline_us": rl, "frac_roofline": rl / med,
                           "scores_kernel_us": float(np.median(time_device(ip.run_scores, 15, 3, flush, stream))) * 1e3,
                           "topk_kernel_us": float(np.median(time_device(ip.run_topk, 15, 3, flush, stream))) * 1e3,
                           "alg_bytes": ab, "alg_flops": fl})
        del ip
        torch.cuda.empty_cache()
        assert api.device_error() == 0, "device error word set"

    # --- CPU baseline: the oracle on host cores, bounded sample
    cpu = None
    if rank == 0 and world == 1:
        sec, sample, threads = oracle_time(w, budget_s=args.oracle_budget)
        cpu = {"value": alg_bytes / sec / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": sample}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks, "back_to_back": b2b,
                "wall_s_timed_region": t_wall, "per_config": per_config}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
