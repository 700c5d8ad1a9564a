#!/usr/bin/env python
"""Throughput of the LAGS sparsify + aggregate step on B200.

One step = error feedback + layer-wise exact top-k for all P simulated workers
(lags_sparsify) and the deterministic sparse aggregation with the weight update
(lags_aggregate_apply), over one batch of synthetic gradients already in HBM.
value = P*N elements per step / step time, in Gelem/s; under torchrun each rank
runs its own replica (no collective on the data path) and value sums the
elements of all ranks over the slowest rank's time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config gpt_1_3b]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

The default workload is the largest that fits one GPU: the 1.3B-parameter
transformer (P = 8 workers, N = 1,311,178,752 elements, 126 GB streamed per
step).  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LAGS sparsify+aggregate Gelem/s per step; achieved HBM GB/s vs peak"
DEFAULT_CONFIG = "gpt_1_3b"
# DRAM bytes (read + write) of one launch of a kernel, from single-launch ncu
# captures (dram__bytes_read.sum + dram__bytes_write.sum) of the workload or
# tensor range named by the key, with the worker-elements that launch
# processed.  A workload without its own capture takes the capture of a range
# of its own tensors (same kernel, same layer shapes), else another
# workload's, scaled by worker-elements: the passes stream over the elements,
# so their traffic grows in proportion.
EF_TRAFFIC = {  # k_ef_capture
    "vgg16": (1_885_810_432 + 895_068_928, 235_517_088),
    # one transformer block (tensors 1..8) of the 1.3B model, 8 workers
    "gpt_1_3b[1:9]": (3_225_167_616 + 1_567_329_024, 402_718_720),
}
DENSE_TRAFFIC = {  # k_dense_sum
    "vgg16": (942_088_192 + 12_455_680, 235_517_088),
}
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
POOL_BUDGET_BYTES = 48 * 1024 ** 3
# oracle timing: per worker, consecutive tensors from the second one (the first
# is the embedding of the transformer and LSTM workloads) up to this many elements
ORACLE_SAMPLE_ELEMS = 56_000_000


def traffic_for(table, name, elems):
    """(bytes per launch, where they come from) for a launch over `elems`
    worker-elements of workload `name` (a `--tensors` case is `name[a:b]`)."""
    if name in table:
        b, e = table[name]
        if e == elems:
            return b, f"ncu capture of this workload ({name})"
    base = name.split("[")[0]
    order = (lambda k: (not k.startswith(base + "["), k != base, k != "vgg16", k))
    for key in sorted(table, key=order):
        b, e = table[key]
        return b * elems / e, f"ncu capture of {key}, scaled by worker-elements"
    return None, "no capture"


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG,
                    choices=["resnet20", "vgg16", "resnet50", "lstm_ptb", "gpt_1_3b"])
    ap.add_argument("--tensors", default=None, metavar="A:B",
                    help="only tensors A..B-1 of the workload (a smaller case of the same "
                         "kernels, for profiling)")
    ap.add_argument("--pool", type=int, default=None,
                    help="at most this many pre-generated gradient steps on the device "
                         "(default: one per step, within 48 GB)")
    ap.add_argument("--global-topk", type=float, default=None, metavar="RHO",
                    help="SLGS: one top-k over the whole flattened model at density RHO "
                         "instead of layer-wise (single-GPU replicas only)")
    ap.add_argument("--dp", action="store_true",
                    help="data-parallel LAGS: split the job's P workers over the ranks and "
                         "all-gather their pick lists (strong scaling) instead of replicas")
    ap.add_argument("--layerwise", action="store_true",
                    help="--dp with layer-wise pipelining: buckets of layers from the merge "
                         "planner, each sparsified, all-gathered and aggregated on its own")
    ap.add_argument("--bwd-ps-per-elem", type=float, default=10.0,
                    help="--layerwise: backward time per gradient element (picoseconds) "
                         "the merge planner assumes")
    ap.add_argument("--dense", action="store_true",
                    help="the dense S-SGD baseline instead of LAGS: worker-ordered sum of "
                         "lr*g (lags_dense_sum), NCCL all-reduce of the ranks' sums, division "
                         "and update (lags_dense_finish); the job's P workers split over ranks")
    ap.add_argument("--adaptive", default=None, choices=["10gbe", "nvlink"],
                    help="per-layer densities from each layer's communication-to-computation "
                         "ratio: backward times measured on the device (synthetic backward), "
                         "messages over the named link, planned by lags_adaptive_densities")
    ap.add_argument("--graph", action="store_true",
                    help="capture each step (one graph per gradient buffer of the pool) in a "
                         "CUDA graph and time graph replays")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def workload(args):
    from synth.configs import WORKLOADS
    w = WORKLOADS[args.config]
    if args.tensors:
        a, b = (int(x) for x in args.tensors.split(":"))
        if not 0 <= a < b <= w.L:
            raise SystemExit(f"--tensors {args.tensors}: the workload has {w.L} tensors")
        w = w.scaled(f"{w.name}[{a}:{b}]", tensors=w.tensors[a:b])
    return w


def workload_config(w, **extra):
    dens = sorted(set(w.densities))
    cfg = {"workload": w.name, "P": w.P, "N": w.N, "layers": w.L, "elements_per_step": w.P * w.N,
           "densities": dens if len(dens) > 1 else dens[0], "lr": w.lr,
           "grad_dist": "normal(0,1/fan_in)" if w.dist == 0 else "student_t3/sqrt(fan_in)"}
    cfg.update(extra)
    return cfg


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
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
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def pinned_host_buffers(avail_bytes: int, local_ranks: int, P: int, N: int) -> int:
    """Pinned host gradient buffers of N fp32 for one rank's e2e leg: as many
    as its workers (P) while they fit in its share of a quarter of the host's
    free memory (the node's ranks split it), at least one."""
    share = int(avail_bytes * 0.25) // max(1, local_ranks)
    return max(1, min(P, share // (N * 4)))


# ------------------------------------------------------------------- oracle timing
# The CPU oracle (plain numpy: one sort per worker-layer segment, worker-ordered
# aggregation) timed on the host cores.  Gradients are generated into shared
# memory before the clock starts; a spawn pool of one process per core then
# sparsifies the (worker, layer) segments and the parent aggregates each layer
# in worker order.  The step is step 0 of the workload (zero residuals).

def oracle_sample_layers(w, budget_elems=ORACLE_SAMPLE_ELEMS):
    """Consecutive tensors of one worker from the second (or the only) one, up
    to about budget_elems elements."""
    layers, total = [], 0
    for l in range(1 if w.L > 1 else 0, w.L):
        d = w.sizes[l]
        if layers and total + d > budget_elems:
            break
        layers.append(l)
        total += d
    return layers, total


def _oracle_segment(shm_name, at, d, off, k, lr):
    """One worker's sparsification of one layer (pool job): zero residual,
    gradient read from shared memory.  Returns the picks."""
    from multiprocessing import shared_memory
    import numpy as np
    import oracle.lags_oracle as lo
    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        g = np.ndarray((d,), dtype=np.float32, buffer=shm.buf, offset=4 * at).copy()
    finally:
        shm.close()
    idx, val, _ = lo.sparsify_layer(off, k, [g], [np.zeros(d, np.float32)], lr)
    return idx[0], val[0]


def _warm(_):
    import oracle.lags_oracle  # noqa: F401
    return os.getpid()


class OracleTimer:
    """Times the oracle's sparsify + aggregate over (worker, layer) segments
    of a workload on `procs` host processes."""

    def __init__(self, w, procs=None, densities=None):
        import concurrent.futures as cf
        import multiprocessing as mp
        self.w = w
        self.dens = list(densities) if densities is not None else w.densities
        self.procs = procs or os.cpu_count() or 1
        self.ex = cf.ProcessPoolExecutor(max_workers=self.procs,
                                         mp_context=mp.get_context("spawn"))
        list(self.ex.map(_warm, range(self.procs)))  # start and import outside the clock
        self.shm = None

    def close(self):
        self.ex.shutdown()
        if self.shm is not None:
            self.shm.close()
            self.shm.unlink()
            self.shm = None

    def _fill(self, segs, step):
        """Generate the segments' gradients into shared memory (untimed)."""
        from multiprocessing import shared_memory
        import numpy as np
        import synth
        total = sum(self.w.sizes[l] for _, l in segs)
        if self.shm is None or self.shm.size < 4 * total:
            if self.shm is not None:
                self.shm.close()
                self.shm.unlink()
            self.shm = shared_memory.SharedMemory(create=True, size=max(4 * total, 4))
        at, where = 0, []
        for p, l in segs:
            d = self.w.sizes[l]
            buf = np.ndarray((d,), dtype=np.float32, buffer=self.shm.buf, offset=4 * at)
            t = self.w.tensors[l]
            synth.fill_host(buf, self.w.offsets[l], self.w.seed, p, step, self.w.dist, t.scale)
            where.append((p, l, at))
            at += d
        return where

    def run(self, segs, step=0, procs=None):
        """Seconds and worker-elements for one oracle pass over `segs`
        [(worker, layer)] (all of one layer's workers are aggregated)."""
        import oracle.lags_oracle as lo
        w = self.w
        where = self._fill(segs, step)
        ks = {l: lo.k_of(w.sizes[l], self.dens[l]) for _, l in segs}
        order = sorted(where, key=lambda x: -w.sizes[x[1]])  # largest first
        t0 = time.perf_counter()
        if procs == 1:
            res = [(p, l, _oracle_segment(self.shm.name, at, w.sizes[l], w.offsets[l], ks[l],
                                          w.lr)) for p, l, at in order]
        else:
            futs = [(p, l, self.ex.submit(_oracle_segment, self.shm.name, at, w.sizes[l],
                                          w.offsets[l], ks[l], w.lr)) for p, l, at in order]
            res = [(p, l, f.result()) for p, l, f in futs]
        by_layer = {}
        for p, l, (idx, val) in res:
            by_layer.setdefault(l, []).append((p, idx, val))
        import numpy as np
        for l, picks in by_layer.items():
            picks.sort(key=lambda x: x[0])  # worker order
            lo.aggregate_layer(w.offsets[l], w.sizes[l], np.stack([x[1] for x in picks]),
                               np.stack([x[2] for x in picks]))
        secs = time.perf_counter() - t0
        return secs, sum(w.sizes[l] for _, l in segs)


def cpu_baseline(w, densities=None):
    """The oracle on the host cores: all P workers' sample tensors in parallel
    (one process per core), plus one worker's largest sample tensor on one
    thread."""
    layers, per_worker = oracle_sample_layers(w)
    timer = OracleTimer(w, densities=densities)
    try:
        segs = [(p, l) for p in range(w.P) for l in layers]
        secs, elems = timer.run(segs)
        big = max(layers, key=lambda l: w.sizes[l])
        s1, e1 = timer.run([(0, big)], procs=1)
    finally:
        timer.close()
    return {"value": elems / secs / 1e9, "unit": "Gelem/s", "cores": timer.procs,
            "kind": "oracle",
            "sample": (f"step 0 (zero residuals) of all {w.P} workers' tensors "
                       f"{layers[0]}..{layers[-1]} ({per_worker} elements per worker, "
                       f"{elems} in all), sparsify + aggregate; numpy oracle in "
                       f"{timer.procs} spawned processes over (worker, tensor) segments, "
                       f"gradients pre-generated in shared memory"),
            "seconds": secs,
            "single_thread": {"value": e1 / s1 / 1e9, "unit": "Gelem/s", "seconds": s1,
                              "sample": f"worker 0, tensor {big} ({e1} elements), one thread"}}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, timed on the host cores
    on the same workload, metric and unit.  Each step is a bounded sample of
    the workload: all P workers of one tensor of the oracle sample (tensors
    taken in turn), in parallel over the workers, then aggregated."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args)
    layers, _ = oracle_sample_layers(w)
    timer = OracleTimer(w)
    try:
        for s in range(args.warmup):
            timer.run([(p, layers[s % len(layers)]) for p in range(w.P)], step=s)
        secs, elems = 0.0, 0
        for s in range(args.steps):
            t, e = timer.run([(p, layers[(args.warmup + s) % len(layers)]) for p in range(w.P)],
                             step=args.warmup + s)
            secs += t
            elems += e
    finally:
        timer.close()
    value = elems / secs / 1e9
    sample = (f"per step all {w.P} workers of one tensor of {layers[0]}..{layers[-1]} in "
              f"turn (zero residuals; {elems} worker-elements over {args.steps} steps), "
              f"sparsify + aggregate; numpy oracle in {timer.procs} spawned processes")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gelem/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, sample_elements=elems),
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": "Gelem/s",
                         "cores": timer.procs, "sample": sample},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- our arm
def run_dense(args):
    """Dense S-SGD baseline: same workload, metric and timing rules as LAGS."""
    import torch
    import torch.distributed as dist
    import synth
    from layer_wise_top_b200.dist import DenseSgd
    from synth.configs import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29532")
        dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                                timeout=datetime.timedelta(seconds=300))
    else:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    w = workload(args)
    if w.P % world:
        raise SystemExit(f"--dense needs the {w.P} workers to divide over {world} ranks")
    P, N = w.P // world, w.N
    ds = DenseSgd.create(N, P, dev)
    pool = max(1, min(args.warmup + args.steps, POOL_BUDGET_BYTES // (P * N * 4),
                      args.pool or 1 << 30))
    grads = []
    for s in range(pool):
        bufs = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)]
        for p in range(P):
            synth.worker_grads_device(w, rank * P + p, s, bufs[p])
        grads.append(bufs)
    dense = torch.empty(N, dtype=torch.float32, device=dev)
    weights = torch.zeros(N, dtype=torch.float32, device=dev)
    K = args.steps
    ev_sum = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]

    def step(i, evs=None):
        if evs is not None:
            evs[0].record()
        ds.kernels.sum(grads[i % pool], w.lr, ds.sum)
        if evs is not None:
            evs[1].record()
        if ds.world > 1:
            dist.all_reduce(ds.sum, op=dist.ReduceOp.SUM)
        ds.kernels.finish(ds.sum, ds.P_total, dense, weights)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record()
    for i in range(K):
        step(args.warmup + i, ev_sum[i])
    t1.record()
    torch.cuda.synchronize()
    dist.barrier(device_ids=[local])
    clk = clocks.stop()
    ms_t = torch.tensor([t0.elapsed_time(t1)], dtype=torch.float64, device=dev)
    dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    sum_ms = sum(a.elapsed_time(b) for a, b in ev_sum) / K
    dist.barrier(device_ids=[local])
    del ds
    dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_peak()
    sum_bytes = 4 * P * N + 4 * N
    achieved = sum_bytes / (sum_ms / 1e3) / 1e9
    line = {
        "metric": METRIC + " (dense S-SGD baseline)",
        "value": world * P * N * K / (ms_max / 1e3) / 1e9, "unit": "Gelem/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_max / K,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: Philox4x32-10 gradients with the workload's tensor shapes",
        "config": workload_config(
            w, parallelism=f"data-parallel: {P} workers per rank x {world} ranks, NCCL "
                           f"all-reduce of the dense sums", grad_pool_steps=pool,
            step="dense S-SGD: lags_dense_sum + all-reduce + lags_dense_finish (with update)",
            l2=f"inputs larger than L2: {4 * P * N / 1e9:.2f} GB read per step"),
        "roofline": {"kernel": "k_dense_sum", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": traffic_for(DENSE_TRAFFIC, w.name, P * N)[0],
                     "traffic_source": traffic_for(DENSE_TRAFFIC, w.name, P * N)[1],
                     "algorithmic_bytes_per_launch": sum_bytes, "avg_launch_ms": sum_ms,
                     "share_of_step": sum_ms / (ms_max / K)},
        "cpu_baseline": None, "e2e": None, "gpu_launches": 2 * K, "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    import synth
    from layer_wise_top_b200 import Plan
    from synth.configs import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    w = workload(args)
    P, N = w.P, w.N
    dens = w.densities
    adaptive_cfg = None
    if args.adaptive:
        # densities from each layer's communication-to-computation ratio, with
        # backward times measured on this device before the timed region
        from layer_wise_top_b200 import adaptive
        dens, secs = adaptive.plan_densities([t.shape for t in w.tensors], P, args.adaptive,
                                             0.001, device=dev)
        adaptive_cfg = {"link": args.adaptive, "alpha_s": adaptive.LINKS[args.adaptive][0],
                        "beta_s_per_byte": adaptive.LINKS[args.adaptive][1],
                        "backward_ms": sum(secs) * 1e3,
                        "dense_layers": sum(1 for r in dens if r >= 1.0),
                        "at_rho_min": sum(1 for r in dens if r <= 0.001),
                        "density_mean": sum(dens) / len(dens)}
    dp = None
    lw = None
    buckets = None
    if args.layerwise:
        args.dp = True
    if args.dp:
        # the job's P workers split over the ranks; every step all-gathers the
        # pick lists and aggregates all P workers on every rank
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29531")
            dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                                    timeout=datetime.timedelta(seconds=300))
        if P % world:
            raise SystemExit(f"--dp needs the {P} workers to divide over {world} ranks")
        from layer_wise_top_b200.dist import DataParallelLags, LayerwiseLags
        if args.layerwise:
            # message model: NVLink all-gather of 8 B per pick per worker,
            # 20 us start-up, the measured 770 GB/s peer bandwidth
            import layer_wise_top_b200 as lags
            h = lags.lags_plan_create(w.sizes, dens, 1)
            ks = [lags.lags_plan_layer(h, l)[1] for l in range(w.L)]
            lags.lags_plan_destroy(h)
            buckets, _ = lags.lags_merge_layers(
                [8 * P * k for k in ks], [d * args.bwd_ps_per_elem * 1e-12 for d in w.sizes],
                2e-5, 1.0 / 770e9)
            lw = LayerwiseLags.create(w.sizes, dens, P // world, buckets, dev)
            dp = lw
        else:
            dp = DataParallelLags.create(w.sizes, dens, P // world, dev)
        P = P // world  # workers held by this rank
        plan = dp.local[0] if lw is not None else dp.local
    elif args.global_topk is not None:
        plan = Plan([N], [args.global_topk], P, device=dev)
    else:
        plan = Plan(w.sizes, dens, P, device=dev)
    # plans whose fused pass is timed and whose status words are read
    local_plans = lw.local if lw is not None else [plan]
    status_plans = local_plans + (lw.total if lw is not None else [])
    step_bytes = P * N * 4
    pool = max(1, min(args.warmup + args.steps, POOL_BUDGET_BYTES // step_bytes,
                      args.pool or 1 << 30))
    grads = []
    for s in range(pool):
        bufs = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)]
        for p in range(P):
            synth.worker_grads_device(w, p, s + 1000 * rank, bufs[p])
        grads.append(bufs)
    res = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
    idx, val = plan.empty_picks() if lw is None else (None, None)
    dense = torch.empty(N, dtype=torch.float32, device=dev)
    weights = torch.zeros(N, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    launches_per_step = 0  # (the all-gather in --dp is NCCL's)
    for pl in local_plans:
        launches_per_step += pl.kernel_launches()[0]
    for pl in (lw.total if lw is not None else [plan]):
        launches_per_step += pl.kernel_launches()[1]

    def step(i):
        if dp is not None:
            dp.step(grads[i % pool], res, w.lr, dense, weights)
            return
        plan.sparsify(grads[i % pool], res, w.lr, idx, val)
        plan.aggregate_apply(idx, val, dense, weights)

    def poll_all():
        f, fb = 0, 0
        for pl in status_plans:
            a, b = pl.poll()
            f, fb = f | a, fb + b
        return f, fb

    K = args.steps

    def k1_events():
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in local_plans]

    graphs = None
    if args.graph:
        # one eager step creates the NCCL communicators; then one graph per
        # gradient buffer, with the fused-pass timing events captured inside
        step(0)
        torch.cuda.synchronize()
        from layer_wise_top_b200.dist import capture_step
        g_events = [k1_events() for _ in range(pool)]
        graphs = []
        for j in range(pool):
            for pl, evs in zip(local_plans, g_events[j]):
                pl.set_events(*evs)
            graphs.append(capture_step(step, j))
        for pl in local_plans:
            pl.set_events(None, None)
        eager_step = step

        def step(i):  # noqa: F811
            graphs[i % pool].replay()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    flags, fallbacks = poll_all()

    ev_k1 = [k1_events() for _ in range(K)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record()
    for i in range(K):
        if graphs is None:
            for pl, evs in zip(local_plans, ev_k1[i]):
                pl.set_events(*evs)
        step(args.warmup + i)
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    for pl in local_plans:
        pl.set_events(None, None)
    ms = t0.elapsed_time(t1)
    if graphs is not None:
        # each graph's events hold its last replay, all inside the timed region
        ev_k1 = [g_events[j] for j in sorted({(args.warmup + i) % pool for i in range(K)})]
    # fused-pass time per step, summed over the buckets of a layer-wise step
    k1_ms = [sum(a.elapsed_time(b) for a, b in evs) for evs in ev_k1]
    flags2, fallbacks2 = poll_all()
    ms_t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())

    # end to end through the same calls: inputs from pinned host memory each
    # step, the updated weights read back each step
    e2e = None
    if graphs is not None:
        step = eager_step  # the e2e leg below times the eager calls
    if not args.no_e2e and dp is None:
        # one pinned host buffer per worker while they fit in this rank's share
        # of a quarter of the host's free memory (the ranks of the node split
        # it); otherwise workers share buffers in turn (worker p copies buffer
        # p mod n).  Either way every worker's P*N*4 bytes cross the host link
        # every step.
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except Exception:  # pragma: no cover
            avail = 64 << 30
        local_ranks = max(1, int(os.environ.get("LOCAL_WORLD_SIZE", str(world))))
        n_host = pinned_host_buffers(avail, local_ranks, P, N)
        host = [torch.empty(N, dtype=torch.float32, pin_memory=True) for _ in range(n_host)]
        for p in range(n_host):
            host[p].copy_(grads[0][p])
        w_host = torch.empty(N, dtype=torch.float32, pin_memory=True)
        # two device gradient sets when memory allows: step i+1's inputs cross
        # the host link (copy stream) while step i computes, and step i's
        # weights go back on a third stream (the link is full duplex)
        free_b, _ = torch.cuda.mem_get_info(dev)
        sets = [grads[0]]
        if free_b > P * N * 4 + (4 << 30):
            sets.append([torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)])
        comp = torch.cuda.current_stream(dev)
        h2d = torch.cuda.Stream(device=dev)
        d2h = torch.cuda.Stream(device=dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ke = max(3, min(K, 10))
        ev_in = [torch.cuda.Event() for _ in range(ke)]
        ev_done = [torch.cuda.Event() for _ in range(ke)]
        ev_out = [torch.cuda.Event() for _ in range(ke)]

        def load(i):  # step i's inputs into set i mod 2, once the set is free
            with torch.cuda.stream(h2d):
                if i >= len(sets):
                    h2d.wait_event(ev_done[i - len(sets)])
                for p in range(P):
                    sets[i % len(sets)][p].copy_(host[p % n_host], non_blocking=True)
                ev_in[i].record(h2d)

        barrier()
        torch.cuda.synchronize()
        e0.record(comp)
        h2d.wait_event(e0)
        d2h.wait_event(e0)
        load(0)
        for i in range(ke):
            if i + 1 < ke and len(sets) > 1:
                load(i + 1)
            comp.wait_event(ev_in[i])
            plan.sparsify(sets[i % len(sets)], res, w.lr, idx, val)
            if i >= 1:
                comp.wait_event(ev_out[i - 1])  # the read-back of the weights is done
            plan.aggregate_apply(idx, val, dense, weights)
            ev_done[i].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[i])
                w_host.copy_(weights, non_blocking=True)
                ev_out[i].record(d2h)
            if i + 1 < ke and len(sets) == 1:
                load(i + 1)
        comp.wait_event(ev_out[ke - 1])
        e1.record(comp)
        torch.cuda.synchronize()
        barrier()
        e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": world * P * N * ke / (float(e_ms.item()) / 1e3) / 1e9,
               "unit": "Gelem/s", "steps": ke, "h2d_bytes_per_step": P * N * 4,
               "d2h_bytes_per_step": N * 4, "pinned_host_buffers": n_host,
               "device_input_sets": len(sets),
               "path": "per step: P pinned host->device gradient copies (the next step's "
                       "overlapping this step's compute when two device input sets fit), "
                       "lags_sparsify, lags_aggregate_apply, device->host copy of the "
                       "updated weights on a third stream"}
        del host, w_host, sets

    # lags_apply alone (outside the step: the step applies the update fused
    # into the aggregation), 12 bytes per element
    apply_ms = None
    if dp is None:
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        ka = max(3, min(K, 10))
        plan.apply(weights, dense)
        torch.cuda.synchronize()
        a0.record()
        for _ in range(ka):
            plan.apply(weights, dense)
        a1.record()
        torch.cuda.synchronize()
        apply_ms = a0.elapsed_time(a1) / ka

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, dens)

    is_dp = dp is not None
    if world > 1 or is_dp:
        dist.barrier(device_ids=[local])
        del dp, lw, graphs  # graphs holding NCCL calls go before the process group
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_kind = measured_peak()
    k1_avg = sum(k1_ms) / len(k1_ms)
    k1_bytes = 12 * P * N
    achieved = k1_bytes / (k1_avg / 1e3) / 1e9
    job_elems = world * P * N  # all ranks' elements
    K_picks = sum(pl.K for pl in local_plans)
    step_alg_bytes = 12 * P * N + 4 * N + 16 * P * K_picks
    line = {
        "metric": METRIC,
        "value": job_elems * K / (ms_max / 1e3) / 1e9,
        "unit": "Gelem/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_max / K,
        "higher_is_better": True, "scaling": "strong" if is_dp else "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic: Philox4x32-10 gradients with the workload's tensor shapes",
        "config": workload_config(
            w, parallelism=(f"data-parallel: {P} workers per rank x {world} ranks, NCCL "
                            f"all-gather of pick lists" if is_dp else f"replicas x{world}")
            + (f", layer-wise: {len(buckets)} buckets of layers (merge planner, backward "
               f"{args.bwd_ps_per_elem} ps/element, 20 us + 8 B/pick at 770 GB/s per message)"
               if buckets else ""), grad_pool_steps=pool,
            l2=f"inputs larger than L2: {12 * P * N / 1e9:.2f} GB streamed per step vs "
               f"{L2_BYTES / 1e6:.0f} MB L2",
            selection=(f"global top-k over all {N} elements at density {args.global_topk}"
                       if args.global_topk is not None else "layer-wise top-k"),
            step="lags_sparsify + lags_aggregate_apply (aggregate and apply fused)"
                 + (", replayed from CUDA graphs" if args.graph else ""),
            **({"densities": "adaptive (per layer)", "adaptive": adaptive_cfg,
                "K_per_worker": sum(pl.K for pl in local_plans)} if adaptive_cfg else {})),
        "roofline": {"kernel": "k_ef_capture", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": traffic_for(EF_TRAFFIC, w.name, P * N)[0],
                     "traffic_source": traffic_for(EF_TRAFFIC, w.name, P * N)[1],
                     "algorithmic_bytes_per_launch": k1_bytes, "avg_launch_ms": k1_avg,
                     "share_of_step": k1_avg / (ms_max / K)},
        "step_hbm": {
            "algorithmic_bytes": step_alg_bytes,
            "formula": "12 P N (grad, residual in, residual out) + 4 N (dense) + 16 P K "
                       "(picks written, then read back)",
            "achieved_gbs": step_alg_bytes / (ms_max / K / 1e3) / 1e9,
            "frac": step_alg_bytes / (ms_max / K / 1e3) / 1e9 / peak},
        "apply": None if apply_ms is None else {
            "ms": apply_ms, "bytes": 12 * N, "achieved_gbs": 12 * N / (apply_ms / 1e3) / 1e9},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
        "status": {"flags": flags | flags2, "exact_fallback_segments": fallbacks + fallbacks2},
    }
    if line["status"]["exact_fallback_segments"]:
        print(f"warning: {line['status']['exact_fallback_segments']} (worker, layer) segments "
              "took the exhaustive selection path (exact, slower)", file=sys.stderr)
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.dense:
        return run_dense(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
