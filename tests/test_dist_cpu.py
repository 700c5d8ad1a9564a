"""Data-parallel exchange over two CPU ranks (gloo).  The GPU kernels are
replaced, in this test only, by oracle-backed stand-ins with the same methods,
so what is tested is the exchange: the all-gather order (rank-major global
workers), buffer shapes, and that every rank ends with bit-identical updates
equal to one process running all workers."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SIZES = [3000, 17, 9000, 64]
DENS = [0.01, 1.0, 0.001, 0.5]
P_LOCAL = 2
LR = 0.5
STEPS = 3


def _grad(p_global, s):
    sys.path.insert(0, ROOT)
    import synth
    from synth.configs import WORKLOADS, Tensor
    w = WORKLOADS["resnet20"].scaled("dist", tensors=[Tensor(f"t{i}", (d,))
                                                      for i, d in enumerate(SIZES)])
    return synth.worker_grads_host(w, p_global, s)


class _OracleLocal:
    """Stand-in for the rank's sparsify plan."""

    def sparsify(self, grads, residuals, lr, idx, val):
        import torch
        import oracle.lags_oracle as lo
        gi = [g.numpy() for g in grads]
        ri = [r.numpy() for r in residuals]
        out_idx, out_val, new = lo.sparsify(SIZES, DENS, gi, ri, lr)
        idx.copy_(torch.from_numpy(out_idx.reshape(-1).view(np.int32)))
        val.copy_(torch.from_numpy(out_val.reshape(-1)))
        for r, n in zip(residuals, new):
            r.copy_(torch.from_numpy(n))


class _OracleTotal:
    """Stand-in for the all-workers aggregation plan."""

    def __init__(self, P_total):
        self.P = P_total

    def aggregate_apply(self, idx_all, val_all, dense, weights):
        import torch
        import oracle.lags_oracle as lo
        N = sum(SIZES)
        K = idx_all.numel() // self.P
        idx = idx_all.numpy().view(np.uint32).reshape(self.P, K)
        val = val_all.numpy().reshape(self.P, K)
        d = lo.aggregate(N, idx, val)
        dense.copy_(torch.from_numpy(d))
        weights.copy_(torch.from_numpy(lo.apply_update(weights.numpy(), d)))


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import oracle.lags_oracle as lo
    from layer_wise_top_b200.dist import DataParallelLags
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        K = lo.layer_plan(SIZES, DENS)[4]
        dp = DataParallelLags(_OracleLocal(), _OracleTotal(P_LOCAL * world), P_LOCAL, K,
                              torch.device("cpu"))
        N = sum(SIZES)
        res = [torch.zeros(N) for _ in range(P_LOCAL)]
        dense = torch.empty(N)
        weights = torch.zeros(N)
        for s in range(STEPS):
            grads = [torch.from_numpy(_grad(rank * P_LOCAL + p, s)) for p in range(P_LOCAL)]
            dp.step(grads, res, LR, dense, weights)
        q.put((rank, dense.numpy().tobytes(), weights.numpy().tobytes(),
               dp.idx_all.numpy().tobytes()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_exchange_matches_single_process():
    import oracle.lags_oracle as lo
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        out = dict((r, (d, w, i)) for r, d, w, i in (q.get(timeout=120) for _ in range(world)))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    # every rank holds the same bits
    assert out[0] == out[1]
    # and they equal one process running all P_LOCAL * world workers
    P = P_LOCAL * world
    hist = lo.run_workload(SIZES, DENS, P, LR, STEPS, lambda p, s: _grad(p, s))
    e_idx, _, _, e_dense, e_w = hist[-1]
    dense = np.frombuffer(out[0][0], dtype=np.float32)
    weights = np.frombuffer(out[0][1], dtype=np.float32)
    idx = np.frombuffer(out[0][2], dtype=np.uint32).reshape(P, -1)
    assert np.array_equal(idx, e_idx)  # rank-major global worker order
    assert np.array_equal(dense.view(np.uint32), e_dense.view(np.uint32))
    assert np.array_equal(weights.view(np.uint32), e_w.view(np.uint32))


# ----------------------------------------------------------- layer-wise pipeline
BUCKETS = [(0, 1), (1, 3), (3, 4)]


class _OracleRangeLocal:
    """Stand-in for a rank's sparsify plan over layers [lb, le)."""

    def __init__(self, lb, le):
        import oracle.lags_oracle as lo
        self.lb, self.le = lb, le
        self.off = sum(SIZES[:lb])
        self.end = sum(SIZES[:le])
        self.K = lo.layer_plan(SIZES[lb:le], DENS[lb:le])[4]

    def sparsify(self, grads, residuals, lr, idx, val):
        import torch
        import oracle.lags_oracle as lo
        a, b = self.off, self.end
        gi = [g.numpy()[a:b] for g in grads]
        ri = [r.numpy()[a:b] for r in residuals]
        out_idx, out_val, new = lo.sparsify(SIZES[self.lb:self.le], DENS[self.lb:self.le], gi,
                                            ri, lr)
        idx.copy_(torch.from_numpy((out_idx + a).reshape(-1).view(np.int32)))
        val.copy_(torch.from_numpy(out_val.reshape(-1)))
        for r, n in zip(residuals, new):
            r[a:b].copy_(torch.from_numpy(n))


class _OracleRangeTotal(_OracleRangeLocal):
    """Stand-in for the all-workers aggregation plan over layers [lb, le)."""

    def __init__(self, lb, le, P_total):
        super().__init__(lb, le)
        self.P = P_total

    def aggregate_apply(self, idx_all, val_all, dense, weights):
        import torch
        import oracle.lags_oracle as lo
        a, b = self.off, self.end
        idx = idx_all.numpy().view(np.uint32).reshape(self.P, self.K) - np.uint32(a)
        val = val_all.numpy().reshape(self.P, self.K)
        d = lo.aggregate(b - a, idx, val)
        dense[a:b].copy_(torch.from_numpy(d))
        weights[a:b].copy_(torch.from_numpy(lo.apply_update(weights.numpy()[a:b], d)))


def _layerwise_rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from layer_wise_top_b200.dist import LayerwiseLags
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local = [_OracleRangeLocal(a, b) for a, b in BUCKETS]
        total = [_OracleRangeTotal(a, b, P_LOCAL * world) for a, b in BUCKETS]
        lw = LayerwiseLags(local, total, BUCKETS, P_LOCAL, torch.device("cpu"))
        N = sum(SIZES)
        res = [torch.zeros(N) for _ in range(P_LOCAL)]
        dense = torch.full((N,), float("nan"))
        weights = torch.zeros(N)
        for s in range(STEPS):
            grads = [torch.from_numpy(_grad(rank * P_LOCAL + p, s)) for p in range(P_LOCAL)]
            lw.step(grads, res, LR, dense, weights)
        q.put((rank, dense.numpy().tobytes(), weights.numpy().tobytes(),
               [t.numpy().tobytes() for t in lw.idx_all]))
    finally:
        dist.destroy_process_group()


def test_two_rank_layerwise_pipeline_matches_single_process():
    import oracle.lags_oracle as lo
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_layerwise_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        out = dict((r, (d, w, i)) for r, d, w, i in (q.get(timeout=120) for _ in range(world)))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert out[0] == out[1]
    P = P_LOCAL * world
    hist = lo.run_workload(SIZES, DENS, P, LR, STEPS, lambda p, s: _grad(p, s))
    e_idx, _, _, e_dense, e_w = hist[-1]
    dense = np.frombuffer(out[0][0], dtype=np.float32)
    weights = np.frombuffer(out[0][1], dtype=np.float32)
    assert np.array_equal(dense.view(np.uint32), e_dense.view(np.uint32))
    assert np.array_equal(weights.view(np.uint32), e_w.view(np.uint32))
    # each bucket's gathered lists are the whole-model lists' columns of its layers
    _, ks, koffs, _, _ = lo.layer_plan(SIZES, DENS)
    for (a, b), raw in zip(BUCKETS, out[0][2]):
        got = np.frombuffer(raw, dtype=np.uint32).reshape(P, -1)
        assert np.array_equal(got, e_idx[:, koffs[a]:koffs[b - 1] + ks[b - 1]])


# ------------------------------------------------------------- dense S-SGD
class _OracleDense:
    """Stand-in for the dense S-SGD kernels."""

    def sum(self, grads, lr, out):
        import torch
        acc = np.zeros(out.numel(), dtype=np.float32)
        for g in grads:
            acc = np.add(acc, np.multiply(np.float32(lr), g.numpy(), dtype=np.float32),
                         dtype=np.float32)
        out.copy_(torch.from_numpy(acc))

    def finish(self, s, P_total, dense, weights):
        import torch
        import oracle.lags_oracle as lo
        d = np.divide(s.numpy(), np.float32(P_total), dtype=np.float32)
        dense.copy_(torch.from_numpy(d))
        weights.copy_(torch.from_numpy(lo.apply_update(weights.numpy(), d)))


def _dense_rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from layer_wise_top_b200.dist import DenseSgd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N = sum(SIZES)
        ds = DenseSgd(_OracleDense(), N, P_LOCAL, torch.device("cpu"))
        dense = torch.empty(N)
        weights = torch.zeros(N)
        grads = [torch.from_numpy(_grad(rank * P_LOCAL + p, 0)) for p in range(P_LOCAL)]
        ds.step(grads, LR, dense, weights)
        q.put((rank, dense.numpy().tobytes(), weights.numpy().tobytes()))
    finally:
        dist.destroy_process_group()


def test_two_rank_dense_sgd_all_reduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dense_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        out = dict((r, (d, w)) for r, d, w in (q.get(timeout=120) for _ in range(world)))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert out[0] == out[1]
    # each rank sums its own workers in order; the two ranks' sums are added once
    f = np.float32
    partial = []
    for r in range(world):
        acc = np.zeros(sum(SIZES), dtype=f)
        for p in range(P_LOCAL):
            acc = np.add(acc, np.multiply(f(LR), _grad(r * P_LOCAL + p, 0), dtype=f), dtype=f)
        partial.append(acc)
    want = np.divide(np.add(partial[0], partial[1], dtype=f), f(world * P_LOCAL), dtype=f)
    dense = np.frombuffer(out[0][0], dtype=f)
    assert np.array_equal(dense.view(np.uint32), want.view(np.uint32))
    import oracle.lags_oracle as lo
    w_want = lo.apply_update(np.zeros(sum(SIZES), dtype=f), want)
    assert np.array_equal(np.frombuffer(out[0][1], dtype=f).view(np.uint32),
                          w_want.view(np.uint32))
