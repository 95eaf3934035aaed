#!/usr/bin/env python
"""Benchmark of the CSA lightning-indexer top-k step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload long_s256k] [--key-chunk C] [--fp8]

A step is one pass of the whole hot path (score contraction on tensor cores,
ReLU + weighted head sum, causal mask, streaming top-k and, when keys are
chunked, the partition merge) over one batch of synthetic input.  The metric is
causally visible query-key pairs per second; the JSON line also carries the
achieved TFLOP/s against the measured bf16 tensor-core peak and the peak HBM.
The default workload is the long-context step (S = 262,144, T = 65,536,
H_I = 64, d_I = 128, top-2048), the largest that fits one GPU.

With N > 1 (one process per GPU under torch.distributed.run) every rank runs
its own independent problem of the same shape (weak scaling, no data-path
collective); the timed region is bracketed by barriers and its maximum over
ranks is reported.  ``--impl reference`` times the fp64 CPU oracle instead
(rank 0 only), on bounded samples of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "indexer query-key pairs/sec, TFLOPS vs B200 peak, peak HBM GB at 1 GPU"
METRIC_DECODE = "decode indexer query-key pairs/sec, HBM GB/s vs B200 peak"
METRIC_PIVOT = "query-group scan: causal pairs/sec of the exact step it stands in for"
METRIC_LAYER = "sparse attention query-entry pairs/sec, TFLOPS vs B200 peak, indexer share of the layer"
UNIT = "pairs/s"
KERNEL_SRC = os.path.join(ROOT, "streaming_top_lightning_b200", "csrc", "k_score_topk.cu")


def causal_pairs(S: int, T: int, m: int) -> int:
    t = np.arange(S, dtype=np.int64)
    return int(np.minimum(T, (t + 1) // m).sum())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for name in ("k_score_topk.cu", "si_select.cuh", "si_common.cuh", "si_kernels.h"):
        with open(os.path.join(ROOT, "streaming_top_lightning_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(workload: str, fp8: bool):
    """DRAM bytes per launch of the score kernel from a committed ncu summary,
    or None when absent or taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    key = f"{workload}{'_fp8' if fp8 else ''}"
    rec = d.get(key)
    if not rec or rec.get("kernel_hash") != kernel_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            time.sleep(0.15)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle


class OracleSample:
    """A fixed set of query rows of the workload for timing the fp64 oracle,
    sized (once, untimed) so that one call takes about ``budget_s``."""

    def __init__(self, sh, budget_s: float, seed: int = 0):
        import oracle

        self.oracle, self.sh = oracle, sh
        self.kc = synth.gen_kc(sh, seed)
        S = sh.S
        n = 2
        while True:
            self._set_rows(np.unique(np.linspace(S // 2, S - 1, n).astype(np.int64)), seed)
            dt = self.run()
            if dt >= budget_s * 0.5 or n >= S // 2:
                break
            n = int(min(S // 2, max(n * 2, n * budget_s / max(dt, 1e-3))))
        self.desc = (f"{self.rows.size} query rows evenly spaced over t in [{S // 2}, {S - 1}] "
                     f"of {sh.name} ({self.pairs} causal pairs), every visible key scored in "
                     f"fp64, then sorted")

    def _set_rows(self, rows, seed):
        self.rows = rows
        self.qr, self.wr = synth.gen_rows(self.sh, rows, seed)
        self.pairs = int(np.minimum(self.sh.T, (rows % self.sh.S + 1) // self.sh.m).sum())

    def run(self) -> float:
        t0 = time.perf_counter()
        self.oracle.indexer_topk_rows(self.qr, self.wr, self.kc, self.sh.S, self.sh.m,
                                      self.sh.topk, self.rows)
        return time.perf_counter() - t0


def run_reference(args, sh):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = max(0.2, 120.0 / max(1, args.steps + args.warmup))
    smp = OracleSample(sh, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        dt = smp.run()
        if i >= args.warmup:
            times.append(dt)
    value = smp.pairs / float(statistics.median(times))
    P = causal_pairs(sh.S, sh.T, sh.m)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * P / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(sh, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.oracle.threads(),
                         "kind": "oracle", "sample": smp.desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def library_plan(sh, args) -> dict:
    """The plan the library runs for this workload and these options (host
    query, no launch): tile shape, query blocks, launches per call."""
    import streaming_top_lightning_b200 as stl

    opts = stl.options(key_chunk=args.key_chunk, row_finish=args.row_finish,
                       key_tile=args.key_tile, strip_slots=args.strip_slots)
    return stl.plan(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk, fp8=args.fp8, opts=opts)


def kernel_launches_per_step(sh, args) -> int:
    """Our kernel launches in one step: the library's own count for one call
    (a score launch per query block, the finishing launches, the row sort when
    rows need it) plus, on the FP8 path, the two quantiser launches."""
    return library_plan(sh, args)["launches"] + (2 if args.fp8 else 0)


L2_BYTES = 126 * 10 ** 6


def input_bytes(sh, fp8: bool) -> int:
    q = sh.B * sh.S * sh.H * sh.D * (1 if fp8 else 2)
    return q + sh.B * sh.S * sh.H * 4 + sh.B * sh.T * sh.D * (1 if fp8 else 2)


def config_of(sh, args):
    return {"workload": sh.name, "B": sh.B, "S": sh.S, "T": sh.T, "m": sh.m, "H_I": sh.H,
            "d_I": sh.D, "topk": sh.topk, "key_chunk": args.key_chunk,
            "row_finish": {0: "library choice", 1: "fused kernel", 2: "merge kernel"}[args.row_finish],
            "key_tile": args.key_tile or "library choice",
            "strip_slots": args.strip_slots or "library choice",
            "score_path": "fp8-e4m3" if args.fp8 else "bf16",
            "pairs_per_step": causal_pairs(sh.S, sh.T, sh.m),
            "l2": (f"inputs larger than L2: {input_bytes(sh, args.fp8) / 1e6:.0f} MB read per step"
                   if input_bytes(sh, args.fp8) > L2_BYTES else
                   f"L2 flushed between timed steps (inputs {input_bytes(sh, args.fp8) / 1e6:.0f} MB"
                   " fit in L2; a 256 MB buffer is written outside each step's events)"),
            "parallelism": f"replicas x{args.gpus} (independent problems)"}


# --------------------------------------------------------------------------- ranks


class Ranks:
    """The multi-rank plumbing of a weak-scaling run: one process per GPU (or
    per CPU process under gloo in the tests), each rank solving its own
    problem.  The only collectives are the timing barrier and the maximum
    over ranks of a measured time; the whole-job value divides the pairs all
    ranks processed by that maximum."""

    def __init__(self, dist, world: int, rank: int, device):
        self.dist, self.world, self.rank, self.device = dist, world, rank, device

    def barrier(self) -> None:
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch

        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def job_value(self, pairs_per_rank: int, ms_per_step: float) -> float:
        return self.world * pairs_per_rank / (ms_per_step / 1e3)


# --------------------------------------------------------------------------- native


def run_native(args, sh):
    import torch
    import torch.distributed as dist

    import streaming_top_lightning_b200 as stl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    ranks = Ranks(dist, world, rank, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    seed = rank
    P = causal_pairs(sh.S, sh.T, sh.m)
    flops_per_pair = 2 * sh.H * sh.D
    # inputs (host, pinned) generated blockwise; device copies
    q_h = torch.empty((sh.B, sh.S, sh.H, sh.D), dtype=torch.int16).pin_memory()
    synth.gen_q(sh, seed, out=q_h.numpy().view(np.uint16), threads=16)
    w_h = torch.from_numpy(synth.gen_w(sh, seed)).pin_memory()
    kc_h = torch.from_numpy(synth.gen_kc(sh, seed).view(np.int16)).pin_memory()
    torch.cuda.synchronize()
    free0, total = torch.cuda.mem_get_info()
    torch.cuda.reset_peak_memory_stats()
    q_d = q_h.to(dev).view(torch.bfloat16)
    w_d = w_h.to(dev)
    kc_d = kc_h.to(dev).view(torch.bfloat16)
    opts = stl.options(key_chunk=args.key_chunk, row_finish=args.row_finish,
                       key_tile=args.key_tile, strip_slots=args.strip_slots)
    timed = {"opts": None}

    def step_opts():
        # inside the timed region each step records its score-kernel events
        return opts if timed["opts"] is None else timed["opts"]
    ws = torch.empty(max(16, stl.workspace_size(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk, opts)),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.int32, device=dev)
    score = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.float32, device=dev)
    if args.fp8:
        def step():
            # the FP8 step starts from the bf16 inputs: quantise, then score + select
            a8, s_q = stl.quantize_fp8_rows(q_d)
            b8, s_k = stl.quantize_fp8_rows(kc_d)
            stl.indexer_topk_fp8(a8, s_q, w_d, b8, s_k, sh.m, sh.topk, out=(idx, score),
                                 opts=step_opts(), workspace=ws)
    else:
        def step():
            stl.indexer_topk(q_d, w_d, kc_d, sh.m, sh.topk, out=(idx, score), opts=step_opts(),
                             workspace=ws)

    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    rc = stl.device_error()
    if rc != 0:
        raise RuntimeError(f"device error {rc} during warm-up")
    peak_alloc = torch.cuda.max_memory_allocated()
    free1, _ = torch.cuda.mem_get_info()

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
    except Exception:
        uuid = None

    K = args.steps
    plan = library_plan(sh, args)
    nblk = plan["query_blocks"]
    # inputs that fit in L2 would be read from it by the next step: flush it
    # between steps (outside the step's events) and time the steps alone
    flush = input_bytes(sh, args.fp8) <= L2_BYTES
    l2buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    # the library records each query block's score-kernel launch into these,
    # so the score kernel's own time excludes the finishing launches
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nblk)] for _ in range(K)]
    for lst in kev:  # make sure the events exist before their handles are taken
        for e in lst:
            e.record(stream)
    torch.cuda.synchronize()
    kopts = [stl.options(key_chunk=args.key_chunk, score_event_list=lst,
                         row_finish=args.row_finish, key_tile=args.key_tile,
                         strip_slots=args.strip_slots) for lst in kev]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(K):
            if flush:
                l2buf.fill_(i & 0xFF)
            timed["opts"] = kopts[i]
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        timed["opts"] = None
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    rc = stl.device_error()
    if rc != 0:
        raise RuntimeError(f"device error {rc} in the timed region")
    if flush:
        total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev))
    else:
        total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    # score-kernel device time per step: the sum of its query blocks' launches
    launch_ms = statistics.mean(sum(lst[2 * b].elapsed_time(lst[2 * b + 1]) for b in range(nblk))
                                for lst in kev)

    # end to end through the public API: host -> device inputs, the call,
    # device -> host result, every step
    if args.no_e2e:
        return finish(args, sh, ranks, P, K, total_ms, launch_ms, None, None, None, None,
                      peak_alloc, free0, free1, clk, plan)
    idx_h = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.int32).pin_memory()
    score_h = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.float32).pin_memory()
    qe = torch.empty_like(q_h, device=dev)
    we = torch.empty_like(w_h, device=dev)
    ke = torch.empty_like(kc_h, device=dev)
    h2d = q_h.numel() * 2 + w_h.numel() * 4 + kc_h.numel() * 2
    d2h = idx_h.numel() * 4 + score_h.numel() * 4

    def e2e_step():
        qe.copy_(q_h, non_blocking=True)
        we.copy_(w_h, non_blocking=True)
        ke.copy_(kc_h, non_blocking=True)
        if args.fp8:
            a8, sa = stl.quantize_fp8_rows(qe.view(torch.bfloat16))
            b8, sb = stl.quantize_fp8_rows(ke.view(torch.bfloat16))
            stl.indexer_topk_fp8(a8, sa, we, b8, sb, sh.m, sh.topk, out=(idx, score), opts=opts,
                                 workspace=ws)
        else:
            stl.indexer_topk(qe.view(torch.bfloat16), we, ke.view(torch.bfloat16), sh.m, sh.topk,
                             out=(idx, score), opts=opts, workspace=ws)
        idx_h.copy_(idx, non_blocking=True)
        score_h.copy_(score, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    Ke = max(3, min(K, 20))
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    assert stl.device_error() == 0
    return finish(args, sh, ranks, P, K, total_ms, launch_ms, e2e_ms, Ke, h2d, d2h,
                  peak_alloc, free0, free1, clk, plan)


def finish(args, sh, ranks, P, K, total_ms, launch_ms, e2e_ms, Ke, h2d, d2h, peak_alloc,
           free0, free1, clk, plan):
    world, rank, dist = ranks.world, ranks.rank, ranks.dist
    flops_per_pair = 2 * sh.H * sh.D
    ms_per_step = total_ms / K
    value = ranks.job_value(P * sh.B, ms_per_step)
    peaks, peak_src = measured_peaks()
    flops_launch = flops_per_pair * P * sh.B
    achieved = flops_launch / (launch_ms / 1e3) / 1e12
    peak_tf = float(peaks["bf16_tflops"]) * (2.0 if args.fp8 else 1.0)
    tflops_step = flops_launch / (ms_per_step / 1e3) / 1e12
    traffic = traffic_record(sh.name, args.fp8)
    launches_per_step = plan["launches"] + (2 if args.fp8 else 0)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3" if args.fp8 else "bf16",
        "data": "synthetic (seeded; distributions of the workload recipe)",
        "config": config_of(sh, args),
        "tflops": tflops_step,
        "tflops_frac_of_measured_peak": tflops_step / peak_tf,
        "peak_hbm_gb": peak_alloc / 1e9,
        "peak_hbm_gib": peak_alloc / 2 ** 30,
        "hbm_in_use_delta_gb": (free0 - free1) / 1e9,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": achieved / peak_tf, "traffic": traffic,
                     "kernel": "k_score_topk", "peak_source": f"{peak_src} bf16_tflops (burst)"
                     + (" x2 nominal fp8/bf16 ratio" if args.fp8 else ""),
                     "algorithmic_flops_per_step": flops_launch,
                     "score_kernel_ms_per_step": launch_ms,
                     "score_launches_per_step": plan["query_blocks"],
                     "avg_launch_ms": launch_ms / plan["query_blocks"],
                     "timing": "sum over the step's query blocks of CUDA events recorded by "
                               "the library around each score-kernel launch"},
        "plan": {k: plan[k] for k in ("queries_per_tile", "mma_n", "key_tile", "stages",
                                      "strip_slots", "pool_keys", "query_blocks", "launches")},
        "e2e": None if e2e_ms is None else {
            "value": ranks.job_value(P * sh.B, e2e_ms / Ke), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K * launches_per_step,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        smp = OracleSample(sh, args.cpu_seconds)
        secs = smp.run()
        line["cpu_baseline"] = {"value": smp.pairs / secs, "unit": UNIT,
                                "cores": smp.oracle.threads(), "kind": "oracle",
                                "sample": smp.desc, "seconds": secs}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- decode


def decode_pairs(ds) -> int:
    """Visible query-key pairs of one decode step (all sequences)."""
    pos = ds.t0 + np.arange(ds.S_q, dtype=np.int64)
    return int(np.minimum(ds.T, (pos + 1) // ds.seq.m).sum()) * ds.seq.B


def decode_config(ds, args):
    sh = ds.seq
    kc_bytes = sh.B * ds.T * sh.D * 2
    return {"workload": ds.name, "B": sh.B, "S_q": ds.S_q, "t0": ds.t0, "T": ds.T, "m": sh.m,
            "H_I": sh.H, "d_I": sh.D, "topk": sh.topk, "key_chunk": args.key_chunk or
            "library choice", "score_path": "bf16", "pairs_per_step": decode_pairs(ds),
            "l2": f"inputs larger than L2: {kc_bytes / 1e6:.0f} MB of keys read per step",
            "parallelism": f"replicas x{args.gpus} (independent problems)"}


def run_decode_reference(args, ds):
    import oracle

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    q, w, kc = synth.gen_decode(ds)
    nb = 1
    per_step = max(0.2, 120.0 / max(1, args.steps + args.warmup))
    while True:  # sequences per sample, sized once (untimed) to the per-step budget
        t = time.perf_counter()
        oracle.indexer_decode(q[:nb], w[:nb], kc[:nb], ds.t0, ds.seq.m, ds.seq.topk)
        dt = time.perf_counter() - t
        if dt >= per_step * 0.5 or nb >= ds.seq.B:
            break
        nb = min(ds.seq.B, max(nb * 2, int(nb * per_step / max(dt, 1e-3))))
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        oracle.indexer_decode(q[:nb], w[:nb], kc[:nb], ds.t0, ds.seq.m, ds.seq.topk)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    pairs = decode_pairs(ds) * nb // ds.seq.B
    value = pairs / float(statistics.median(times))
    desc = f"{nb} of the {ds.seq.B} sequences of {ds.name}, every visible key scored in fp64"
    line = {"impl": "reference", "metric": METRIC_DECODE, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * decode_pairs(ds) / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(ds, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args, ds):
    """A decode step: the newest query of each of B sequences against the
    keys compressed so far (resident on the GPU, as a KV cache is).  The
    score kernel reads every visible key once, so its bound is HBM."""
    import torch
    import torch.distributed as dist

    import streaming_top_lightning_b200 as stl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ranks = Ranks(dist, world, rank, dev)
    sh = ds.seq
    q, w, kc = synth.gen_decode(ds, seed=rank)
    q_h = torch.from_numpy(q.view(np.int16)).pin_memory()
    w_h = torch.from_numpy(w).pin_memory()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch.cuda.reset_peak_memory_stats()
    kc_d = torch.from_numpy(kc.view(np.int16)).to(dev).view(torch.bfloat16)
    q_d = q_h.to(dev).view(torch.bfloat16)
    w_d = w_h.to(dev)
    opts = stl.options(key_chunk=args.key_chunk)
    ws = torch.empty(max(16, stl.decode_workspace_size(sh.B, ds.S_q, ds.t0, ds.T, sh.H, sh.D,
                                                       sh.m, sh.topk, opts)),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty((sh.B, ds.S_q, sh.topk), dtype=torch.int32, device=dev)
    score = torch.empty((sh.B, ds.S_q, sh.topk), dtype=torch.float32, device=dev)
    plan = stl.decode_plan(sh.B, ds.S_q, ds.t0, ds.T, sh.H, sh.D, sh.m, sh.topk, opts)
    stream = torch.cuda.current_stream()
    K = args.steps
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for lst in kev:
        for e in lst:
            e.record(stream)
    kopts = [stl.options(key_chunk=args.key_chunk, score_event_list=lst) for lst in kev]

    def step(o):
        stl.indexer_decode(q_d, w_d, kc_d, ds.t0, sh.m, sh.topk, out=(idx, score), opts=o,
                           workspace=ws)

    for _ in range(max(3, args.warmup)):
        step(opts)
    torch.cuda.synchronize()
    if stl.device_error() != 0:
        raise RuntimeError("device error during warm-up")
    peak_alloc = torch.cuda.max_memory_allocated()
    free1, _ = torch.cuda.mem_get_info()
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        pass
    with ClockSampler(uuid) as clk:
        ranks.barrier()
        torch.cuda.synchronize()
        t0e.record(stream)
        for i in range(K):
            step(kopts[i])
        t1e.record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
    if stl.device_error() != 0:
        raise RuntimeError("device error in the timed region")
    total_ms = ranks.max_over_ranks(t0e.elapsed_time(t1e))
    score_ms = statistics.mean(lst[0].elapsed_time(lst[1]) for lst in kev)

    # end to end through the public API: each step's new queries and weights
    # go host -> device, the selected rows come back; the keys stay resident
    idx_h = torch.empty(tuple(idx.shape), dtype=torch.int32).pin_memory()
    score_h = torch.empty(tuple(score.shape), dtype=torch.float32).pin_memory()
    qe, we = torch.empty_like(q_h, device=dev), torch.empty_like(w_h, device=dev)

    def e2e_step():
        qe.copy_(q_h, non_blocking=True)
        we.copy_(w_h, non_blocking=True)
        stl.indexer_decode(qe.view(torch.bfloat16), we, kc_d, ds.t0, sh.m, sh.topk,
                           out=(idx, score), opts=opts, workspace=ws)
        idx_h.copy_(idx, non_blocking=True)
        score_h.copy_(score, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    ranks.barrier()
    e2e_ms = ranks.max_over_ranks(e0.elapsed_time(e1)) / K
    assert stl.device_error() == 0

    pairs = decode_pairs(ds)
    ms_per_step = total_ms / K
    # algorithmic bytes of the score kernel: every visible key read once, the
    # queries and weights, and the candidate lists it writes
    pos = ds.t0 + np.arange(ds.S_q)
    vis = int(np.minimum(ds.T, (pos.max() + 1) // sh.m))
    kc_bytes = sh.B * vis * sh.D * 2
    qw_bytes = sh.B * ds.S_q * sh.H * (sh.D * 2 + 4)
    lists = (sh.B * plan["key_chunks"] * plan["queries_per_tile"] * plan["partial_len"] * 8
             if plan["key_chunks"] > 1 else 0)
    alg = kc_bytes + qw_bytes + lists
    peaks, peak_src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = alg / (score_ms / 1e3) / 1e9
    h2d = q_h.numel() * 2 + w_h.numel() * 4
    d2h = idx_h.numel() * 4 + score_h.numel() * 4
    line = {
        "metric": METRIC_DECODE, "value": ranks.job_value(pairs, ms_per_step), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; distributions of the workload recipe)",
        "config": decode_config(ds, args),
        "step_gbs": alg / (ms_per_step / 1e3) / 1e9,
        "peak_hbm_gb": peak_alloc / 1e9, "hbm_in_use_delta_gb": (free0 - free1) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None, "kernel": "k_score_topk",
                     "peak_source": f"{peak_src} hbm_gbs",
                     "algorithmic_bytes_per_step": alg,
                     "score_kernel_ms_per_step": score_ms,
                     "timing": "CUDA events recorded by the library around the score-kernel "
                               "launch"},
        "plan": {k: plan[k] for k in ("queries_per_tile", "mma_n", "key_tile", "stages",
                                      "strip_slots", "pool_keys", "key_chunks", "launches")},
        "e2e": {"value": ranks.job_value(pairs, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "resident": "the keys (a KV cache stays on the GPU between steps)"},
        "gpu_launches": K * plan["launches"],
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle

        nb = max(1, min(sh.B, 4))
        t = time.perf_counter()
        oracle.indexer_decode(q[:nb], w[:nb], kc[:nb], ds.t0, sh.m, sh.topk)
        secs = time.perf_counter() - t
        line["cpu_baseline"] = {"value": pairs * nb / sh.B / secs, "unit": UNIT,
                                "cores": oracle.threads(), "kind": "oracle",
                                "sample": f"{nb} of the {sh.B} sequences", "seconds": secs}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- pivot


def run_pivot(args, name):
    """The query-group candidate scan against the exact step on the same
    inputs: both timed with CUDA events; the recall it gives up is measured
    by the tests against the oracle."""
    import torch

    import streaming_top_lightning_b200 as stl

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("pivot workloads run on one GPU")
    base, G, C = synth.PIVOT_SCANS[name]
    sh = synth.shape(base)
    dev = torch.device("cuda", 0)
    q = synth.gen_q(sh, 0, threads=16)
    to_bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    q_d, kc_d = to_bf(q), to_bf(synth.gen_kc(sh, 0))
    del q
    w_d = torch.from_numpy(synth.gen_w(sh, 0)).to(dev)
    idx = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.int32, device=dev)
    score = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.float32, device=dev)
    opts = stl.options()
    ws_p = torch.empty(stl.pivot_workspace_size(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk, G, C, opts),
                       dtype=torch.uint8, device=dev)
    ws_e = torch.empty(max(16, stl.workspace_size(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk, opts)),
                       dtype=torch.uint8, device=dev)

    def pivot():
        stl.indexer_pivot(q_d, w_d, kc_d, sh.m, sh.topk, G, C, out=(idx, score), opts=opts,
                          workspace=ws_p)

    def exact():
        stl.indexer_topk(q_d, w_d, kc_d, sh.m, sh.topk, out=(idx, score), opts=opts,
                         workspace=ws_e)

    stream = torch.cuda.current_stream()
    times = {}
    for label, fn in (("pivot", pivot), ("exact", exact)):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        if stl.device_error() != 0:
            raise RuntimeError(f"device error during the {label} warm-up")
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(stream)
        for i in range(args.steps):
            fn()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        times[label] = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps))
    P = causal_pairs(sh.S, sh.T, sh.m) * sh.B
    ng = sh.S // G
    reps = (np.arange(ng) * G + G - 1)
    scan_pairs = int(np.minimum(sh.T, (reps + 1) // sh.m).sum()) * sh.B
    line = {
        "metric": METRIC_PIVOT, "value": P / (times["pivot"] / 1e3), "unit": "pairs/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": times["pivot"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; distributions of the workload recipe)",
        "config": {"workload": name, "indexer": sh.name, "B": sh.B, "S": sh.S, "T": sh.T,
                   "topk": sh.topk, "group": G, "candidates": C,
                   "scored_pairs": scan_pairs + sh.B * sh.S * C, "exact_pairs": P},
        "exact_ms": times["exact"], "speedup_vs_exact": times["exact"] / times["pivot"],
        "recall": "measured by tests/test_gpu_pivot.py against the oracle",
        "gpu_launches": args.steps * (stl.decode_plan(sh.B, ng, G - 1, sh.T, sh.H, sh.D, sh.m, C)
                                      ["launches"] + 3 + 2),
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- layer


def run_layer(args, name):
    """A compressed-sparse-attention layer: the indexer step, then multi-query
    attention of 128 heads (dim 128) over the entries it selects.  Times the
    attention kernel alone (CUDA events around its launch) and the whole
    layer; the attention's bound is the tensor cores (4 * 128 * 128 flops per
    query-entry pair: Q K^T and P V)."""
    import torch

    import streaming_top_lightning_b200 as stl

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("layer workloads run on one GPU")
    sh = synth.shape(synth.ATTENTION_LAYERS[name])
    dev = torch.device("cuda", 0)
    q, w, kc = (synth.gen_q(sh, 0, threads=16), synth.gen_w(sh, 0), synth.gen_kc(sh, 0))
    qa, ka, va = synth.gen_attention(sh.B, sh.S, sh.T, seed=1)
    to_bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    q_d, kc_d, qa_d, ka_d, va_d = to_bf(q), to_bf(kc), to_bf(qa), to_bf(ka), to_bf(va)
    w_d = torch.from_numpy(w).to(dev)
    del q, qa
    idx = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.int32, device=dev)
    score = torch.empty((sh.B, sh.S, sh.topk), dtype=torch.float32, device=dev)
    out = torch.empty((sh.B, sh.S, 128, 128), dtype=torch.float32, device=dev)
    opts = stl.options()
    ws = torch.empty(max(16, stl.workspace_size(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk, opts)),
                     dtype=torch.uint8, device=dev)
    scale = 1.0 / np.sqrt(128.0)
    stream = torch.cuda.current_stream()

    def indexer():
        stl.indexer_topk(q_d, w_d, kc_d, sh.m, sh.topk, out=(idx, score), opts=opts, workspace=ws)

    def attention():
        stl.sparse_attention(qa_d, ka_d, va_d, idx, scale, out=out)

    for _ in range(max(3, args.warmup)):
        indexer()
        attention()
    torch.cuda.synchronize()
    if stl.device_error() != 0:
        raise RuntimeError("device error during warm-up")
    pairs = int((idx >= 0).sum().item())  # listed entries, as the indexer selected them
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        pass
    with ClockSampler(uuid) as clk:
        torch.cuda.synchronize()
        for i in range(K):
            ev[i][0].record(stream)
            indexer()
            ev[i][1].record(stream)
            attention()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    if stl.device_error() != 0:
        raise RuntimeError("device error in the timed region")
    idx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    flops = pairs * 4 * 128 * 128
    peaks, peak_src = measured_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    achieved = flops / (attn_ms / 1e3) / 1e12
    line = {
        "metric": METRIC_LAYER, "value": pairs / (attn_ms / 1e3), "unit": "pairs/s",
        "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": idx_ms + attn_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; the indexer's own rows select the entries)",
        "config": {"workload": name, "indexer": sh.name, "B": sh.B, "S": sh.S, "T": sh.T,
                   "topk": sh.topk, "H_a": 128, "d_a": 128, "listed_pairs": pairs,
                   "l2": "inputs larger than L2 (query heads)"},
        "indexer_ms": idx_ms, "attention_ms": attn_ms,
        "indexer_share_of_layer": idx_ms / (idx_ms + attn_ms),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "traffic": None, "kernel": "k_sparse_attn",
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "algorithmic_flops_per_step": flops,
                     "timing": "CUDA events around the attention launch"},
        "gpu_launches": K * (stl.plan(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk)["launches"] + 1),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="long_s256k",
                    choices=sorted(synth.SHAPES) + sorted(synth.DECODE_SHAPES)
                    + sorted(synth.ATTENTION_LAYERS) + sorted(synth.PIVOT_SCANS))
    ap.add_argument("--key-chunk", type=int, default=0)
    ap.add_argument("--row-finish", type=int, default=0, choices=(0, 1, 2),
                    help="1: rows finished in the fused kernel; 2: by the merge kernel; "
                         "0: the library's choice")
    ap.add_argument("--strip-slots", type=int, default=0, choices=(0, 2, 3, 4),
                    help="score strips in flight between epilogue and selection (0: library's choice)")
    ap.add_argument("--key-tile", type=int, default=0, choices=(0, 32, 64, 128, 256, 512, 1024),
                    help="keys per score strip handed to the selection warps (0: library's choice)")
    ap.add_argument("--topk", type=int, default=0)
    ap.add_argument("--fp8", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.workload in synth.PIVOT_SCANS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "pivot workloads time the GPU "
                              "path only; the oracle's scan is timed in the tests"}))
            return 0
        return run_pivot(args, args.workload)
    if args.workload in synth.ATTENTION_LAYERS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "layer workloads time the GPU "
                              "path only; the oracle's attention is timed in the tests"}))
            return 0
        return run_layer(args, args.workload)
    if args.workload in synth.DECODE_SHAPES:
        ds = synth.DECODE_SHAPES[args.workload]
        if args.fp8 or args.topk or args.key_tile or args.strip_slots or args.row_finish:
            ap.error("decode workloads take only --key-chunk among the workload options")
        return (run_decode_reference if args.impl == "reference" else run_decode)(args, ds)
    sh = synth.shape(args.workload)
    if args.topk:
        sh = synth.shape(args.workload, topk=args.topk)
    if args.impl == "reference":
        return run_reference(args, sh)
    return run_native(args, sh)


if __name__ == "__main__":
    sys.exit(main())
