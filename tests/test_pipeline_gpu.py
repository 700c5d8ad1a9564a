"""Layer-wise pipelining on the GPU: plans over ranges of layers
(lags_plan_create_range) against the oracle and against one whole-model plan,
and the pipelined data-parallel step (LayerwiseLags over a one-rank NCCL group,
gradients produced layer by layer on another stream) against the plain step,
bit for bit."""
import datetime
import os
import socket

import numpy as np
import pytest

import oracle.lags_oracle as lo
import synth
from synth.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def _cuts(L, rng, n):
    inner = sorted(int(x) for x in rng.choice(np.arange(1, L), size=min(n, L - 1), replace=False))
    f = [0] + inner + [L]
    return [(f[i], f[i + 1]) for i in range(len(f) - 1)]


def _run_ranges(w, buckets, steps):
    """Steps of per-bucket sparsify + aggregate_apply; returns the tensors."""
    import torch
    from layer_wise_top_b200 import Plan
    dev = torch.device("cuda")
    N, P = w.N, w.P
    plans = [Plan(w.sizes, w.densities, P, device=dev, layer_range=b) for b in buckets]
    picks = [p.empty_picks() for p in plans]
    grads = [torch.empty(N, device=dev) for _ in range(P)]
    res = [torch.zeros(N, device=dev) for _ in range(P)]
    dense = torch.full((N,), float("nan"), device=dev)
    weights = torch.zeros(N, device=dev)
    for s in range(steps):
        for p in range(P):
            synth.worker_grads_device(w, p, s, grads[p])
        for plan, (idx, val) in zip(plans, picks):
            plan.sparsify(grads, res, w.lr, idx, val)
        for plan, (idx, val) in zip(plans, picks):
            plan.aggregate_apply(idx, val, dense, weights)
    torch.cuda.synchronize()
    return plans, picks, res, dense, weights


def test_range_plans_equal_oracle_resnet20():
    w = WORKLOADS["resnet20"]
    rng = np.random.default_rng(5)
    buckets = _cuts(w.L, rng, 6)
    steps = 4
    plans, picks, res, dense, weights = _run_ranges(w, buckets, steps)
    hist = lo.run_workload(w.sizes, w.densities, w.P, w.lr, steps,
                           lambda p, s: synth.worker_grads_host(w, p, s))
    e_idx, e_val, e_res, e_dense, e_w = hist[-1]
    _, ks, koffs, _, _ = lo.layer_plan(w.sizes, w.densities)
    for (a, b), plan, (idx, val) in zip(buckets, plans, picks):
        lo_k, hi_k = koffs[a], koffs[b - 1] + ks[b - 1]
        assert plan.K == hi_k - lo_k
        assert plan.first == sum(w.sizes[:a]) and plan.N == sum(w.sizes[:b])
        got_i = _u32(idx).reshape(w.P, plan.K)
        got_v = _u32(val).reshape(w.P, plan.K)
        assert np.array_equal(got_i, e_idx[:, lo_k:hi_k])
        assert np.array_equal(got_v, e_val[:, lo_k:hi_k].view(np.uint32))
    assert np.array_equal(_u32(dense), e_dense.view(np.uint32))
    assert np.array_equal(_u32(weights), e_w.view(np.uint32))
    for r, e in zip(res, e_res):
        assert np.array_equal(_u32(r), e.view(np.uint32))


@pytest.mark.parametrize("name", ["vgg16", "resnet50"])
def test_range_plans_equal_whole_model_plan(name):
    import torch
    from layer_wise_top_b200 import Plan
    w = WORKLOADS[name]
    steps = 2
    buckets = _cuts(w.L, np.random.default_rng(9), 7) if name == "vgg16" else \
        [(l, l + 1) for l in range(w.L)]
    plans, picks, res, dense, weights = _run_ranges(w, buckets, steps)
    dev = torch.device("cuda")
    full = Plan(w.sizes, w.densities, w.P, device=dev)
    idx, val = full.empty_picks()
    grads = [torch.empty(w.N, device=dev) for _ in range(w.P)]
    res_f = [torch.zeros(w.N, device=dev) for _ in range(w.P)]
    dense_f = torch.empty(w.N, device=dev)
    w_f = torch.zeros(w.N, device=dev)
    for s in range(steps):
        for p in range(w.P):
            synth.worker_grads_device(w, p, s, grads[p])
        full.sparsify(grads, res_f, w.lr, idx, val)
        full.aggregate_apply(idx, val, dense_f, w_f)
    torch.cuda.synchronize()
    fi = _u32(idx).reshape(w.P, full.K)
    k0 = 0
    for plan, (bi, _) in zip(plans, picks):
        assert np.array_equal(_u32(bi).reshape(w.P, plan.K), fi[:, k0:k0 + plan.K])
        k0 += plan.K
    assert k0 == full.K
    assert np.array_equal(_u32(dense), _u32(dense_f))
    assert np.array_equal(_u32(weights), _u32(w_f))
    for a, b in zip(res, res_f):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_range_apply_touches_only_its_range():
    import torch
    from layer_wise_top_b200 import Plan
    sizes = [5, 8191, 3, 70001, 6]
    dens = [1.0] * 5
    dev = torch.device("cuda")
    gen = torch.Generator(device="cpu").manual_seed(3)
    N = sum(sizes)
    w0 = torch.randn(N, generator=gen).to(dev)
    d = torch.randn(N, generator=gen).to(dev)
    for a, b in [(0, 1), (1, 3), (2, 5), (3, 4), (0, 5)]:
        plan = Plan(sizes, dens, 1, device=dev, layer_range=(a, b))
        wt = w0.clone()
        plan.apply(wt, d)
        lo_e, hi_e = sum(sizes[:a]), sum(sizes[:b])
        want = w0.clone()
        want[lo_e:hi_e] = want[lo_e:hi_e] - d[lo_e:hi_e]
        assert torch.equal(wt.view(torch.int32), want.view(torch.int32)), (a, b)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name,cut", [("resnet20", "per_layer"), ("resnet50", "planner")])
def test_layerwise_pipeline_one_rank_equals_plain_step(name, cut):
    import torch
    import torch.distributed as dist
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    from layer_wise_top_b200.dist import LayerwiseLags
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = WORKLOADS[name]
        P, N = w.P, w.N
        _, ks, _, _, _ = lo.layer_plan(w.sizes, w.densities)
        if cut == "per_layer":
            buckets = [(l, l + 1) for l in range(w.L)]
        else:
            # backward time proportional to layer size, 20 us start-up per message
            buckets, _ = L.lags_merge_layers([8 * P * k for k in ks],
                                             [d * 2e-12 for d in w.sizes], 2e-5, 1.0 / 700e9)
            assert 1 < len(buckets) < w.L
        lw = LayerwiseLags.create(w.sizes, w.densities, P, buckets, dev)
        plan = Plan(w.sizes, w.densities, P, device=dev)
        grads = [torch.empty(N, device=dev) for _ in range(P)]
        grads_b = [torch.empty(N, device=dev) for _ in range(P)]
        res_a = [torch.zeros(N, device=dev) for _ in range(P)]
        res_b = [torch.zeros(N, device=dev) for _ in range(P)]
        dense_a, dense_b = torch.empty(N, device=dev), torch.empty(N, device=dev)
        w_a, w_b = torch.zeros(N, device=dev), torch.zeros(N, device=dev)
        idx, val = plan.empty_picks()
        bwd = torch.cuda.Stream(device=dev)
        main = torch.cuda.current_stream(dev)
        for s in range(3):
            # synthetic backward: layers produced from the last to the first on
            # their own stream, one event per bucket
            bwd.wait_stream(main)
            ready = [None] * len(buckets)
            with torch.cuda.stream(bwd):
                for bi in reversed(range(len(buckets))):
                    a, b = buckets[bi]
                    for p in range(P):
                        synth.worker_grads_device(w, p, s, grads[p],
                                                  layers=range(b - 1, a - 1, -1))
                    ev = torch.cuda.Event()
                    ev.record(bwd)
                    ready[bi] = ev
            lw.step(grads, res_a, w.lr, dense_a, w_a, ready=ready)
            for p in range(P):
                synth.worker_grads_device(w, p, s, grads_b[p])
            plan.sparsify(grads_b, res_b, w.lr, idx, val)
            plan.aggregate_apply(idx, val, dense_b, w_b)
        torch.cuda.synchronize()
        assert np.array_equal(_u32(dense_a), _u32(dense_b))
        assert np.array_equal(_u32(w_a), _u32(w_b))
        for a, b in zip(res_a, res_b):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
        fi = _u32(idx).reshape(P, plan.K)
        k0 = 0
        for t in lw.idx_all:
            kb = t.numel() // P
            assert np.array_equal(_u32(t).reshape(P, kb), fi[:, k0:k0 + kb])
            k0 += kb
        assert k0 == plan.K
    finally:
        dist.destroy_process_group()


def test_layerwise_step_replayed_from_cuda_graph():
    import torch
    import torch.distributed as dist
    from layer_wise_top_b200 import Plan
    from layer_wise_top_b200.dist import LayerwiseLags, capture_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                            timeout=datetime.timedelta(seconds=60))
    graph = None
    try:
        w = WORKLOADS["resnet20"]
        P, N = w.P, w.N
        buckets = [(0, 5), (5, 6), (6, 20), (20, 21)]
        lw = LayerwiseLags.create(w.sizes, w.densities, P, buckets, dev)
        plan = Plan(w.sizes, w.densities, P, device=dev)
        grads = [torch.empty(N, device=dev) for _ in range(P)]
        res_a = [torch.zeros(N, device=dev) for _ in range(P)]
        res_b = [torch.zeros(N, device=dev) for _ in range(P)]
        dense_a, dense_b = torch.empty(N, device=dev), torch.empty(N, device=dev)
        w_a, w_b = torch.zeros(N, device=dev), torch.zeros(N, device=dev)
        idx, val = plan.empty_picks()
        steps = 4
        for s in range(steps):
            for p in range(P):
                synth.worker_grads_device(w, p, s, grads[p])
            if s == 0:
                lw.step(grads, res_a, w.lr, dense_a, w_a)  # eager: creates the communicator
                graph = capture_step(lw.step, grads, res_a, w.lr, dense_a, w_a)
            else:
                graph.replay()
            plan.sparsify(grads, res_b, w.lr, idx, val)
            plan.aggregate_apply(idx, val, dense_b, w_b)
        torch.cuda.synchronize()
        assert np.array_equal(_u32(dense_a), _u32(dense_b))
        assert np.array_equal(_u32(w_a), _u32(w_b))
        for a, b in zip(res_a, res_b):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    finally:
        graph = None
        dist.destroy_process_group()
