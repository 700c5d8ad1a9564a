"""GPU features around the hot path: global top-k over a whole model buffer
(one segment), capture of a step in a CUDA graph, and malformed pick lists
reported through the status word."""
import numpy as np
import pytest

import oracle.lags_oracle as lo
import synth
from synth.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("name,P,steps,max_fallbacks", [("resnet20", 4, 3, 0),
                                                       ("vgg16", 2, 2, None)])
def test_global_topk_one_segment(name, P, steps, max_fallbacks):
    """Single-layer (global) top-k over the flattened model: the plan has one
    layer of N elements.  Over VGG-16 the largest values crowd into the first
    tensors (gradient scales differ 13x), overflow the candidate slots and take
    the exhaustive path; the result is exact either way."""
    import torch
    from gpu_harness import GpuRun
    w = WORKLOADS[name]
    N = w.N
    run = GpuRun([N], [0.001], P, w.lr)
    hist = lo.run_workload([N], [0.001], P, w.lr, steps,
                           lambda p, s: synth.worker_grads_host(w, p, s))
    for s in range(steps):
        for p in range(P):
            synth.worker_grads_device(w, p, s, run.grads[p])
        run.step(fused=True)
        flags, fb = run.plan.poll()
        assert flags == 0
        if max_fallbacks is not None:
            assert fb <= max_fallbacks
        e_idx, e_val, e_res, e_dense, e_w = hist[s]
        assert np.array_equal(_u32(run.idx).reshape(P, -1), e_idx)
        assert np.array_equal(_u32(run.val).reshape(P, -1), e_val.view(np.uint32))
        for p in range(P):
            assert np.array_equal(_u32(run.res[p]), e_res[p].view(np.uint32))
        assert np.array_equal(_u32(run.dense), e_dense.view(np.uint32))
        assert np.array_equal(_u32(run.weights), e_w.view(np.uint32))


def test_global_topk_1_3b_one_segment():
    """SLGS on the 1.3B transformer: one segment of 1,311,178,752 elements
    (k = 1,311,179), two workers, two steps, checked in chunks against the
    properties that fix the selection and the worker-ordered dense update."""
    import torch
    from gpu_harness import GpuRun, check_layer_chunked
    w = WORKLOADS["gpt_1_3b"]
    P = 2
    run = GpuRun([w.N], [0.001], P, w.lr, keep_prev=True)
    assert run.plan.K == 1_311_179
    for s in range(2):
        for p in range(P):
            synth.worker_grads_device(w, p, s, run.grads[p])
        run.step(fused=s == 1)
        flags, _ = run.plan.poll()
        assert flags == 0
        check_layer_chunked(run, 0, w.lr)
    del run
    torch.cuda.empty_cache()


def test_step_captured_in_cuda_graph():
    """The calls only enqueue kernels (no allocation, no synchronisation), so a
    step can be captured; replays give the eager results bit for bit."""
    import torch
    from layer_wise_top_b200 import Plan
    w = WORKLOADS["vgg16"]
    P, N = w.P, w.N
    outs = []
    for use_graph in (False, True):
        plan = Plan(w.sizes, w.densities, P)
        grads = [torch.empty(N, device="cuda") for _ in range(P)]
        res = [torch.zeros(N, device="cuda") for _ in range(P)]
        idx, val = plan.empty_picks()
        dense, weights = torch.empty(N, device="cuda"), torch.zeros(N, device="cuda")
        for p in range(P):
            synth.worker_grads_device(w, p, 0, grads[p])
        torch.cuda.synchronize()

        def step():
            plan.sparsify(grads, res, w.lr, idx, val)
            plan.aggregate_apply(idx, val, dense, weights)

        if use_graph:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    step()
            torch.cuda.current_stream().wait_stream(s)
            torch.cuda.synchronize()
            # capture enqueued nothing; three replays = three steps
            for _ in range(3):
                g.replay()
        else:
            for _ in range(3):
                step()
        torch.cuda.synchronize()
        outs.append([_u32(x) for x in (idx, val, dense, weights, res[0], res[P - 1])])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_bad_pick_list_is_reported():
    import torch
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    sizes, dens, P = [5000, 20000], [0.01, 0.01], 2
    plan = Plan(sizes, dens, P)
    N, K = plan.N, plan.K
    idx = torch.zeros(P * K, dtype=torch.int32, device="cuda")  # not ascending
    val = torch.ones(P * K, dtype=torch.float32, device="cuda")
    dense = torch.empty(N, device="cuda")
    plan.aggregate(idx, val, dense)
    with pytest.raises(L.LagsError) as e:
        plan.poll()
    assert e.value.status == L.LAGS_ERR_BAD_PICKS
    # the status word is cleared by the poll; a valid list afterwards is fine
    grads = [torch.randn(N, device="cuda") for _ in range(P)]
    res = [torch.zeros(N, device="cuda") for _ in range(P)]
    i2, v2 = plan.empty_picks()
    plan.sparsify(grads, res, 0.1, i2, v2)
    plan.aggregate(i2, v2, dense)
    assert plan.poll() == (0, 0)
