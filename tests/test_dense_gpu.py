"""Dense S-SGD baseline on the GPU (lags_dense_sum + lags_dense_finish)
against the oracle, bit for bit, and against a LAGS plan at density 1."""
import datetime
import os
import socket

import numpy as np
import pytest

import oracle.lags_oracle as lo
import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("P,sizes", [(4, None), (17, [1, 3, 8191, 65537, 2]), (1, [5]),
                                     (9, [4097])])
def test_dense_step_equals_oracle(P, sizes):
    import torch
    from layer_wise_top_b200 import DenseKernels
    w = WORKLOADS["resnet20"]
    if sizes is not None:
        w = w.scaled("dense", P=P, tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    N = w.N
    dev = torch.device("cuda")
    grads = [torch.empty(N, device=dev) for _ in range(w.P)]
    for p in range(w.P):
        synth.worker_grads_device(w, p, 0, grads[p])
    kern = DenseKernels(N, dev)
    total = torch.empty(N, device=dev)
    dense = torch.full((N,), float("nan"), device=dev)
    rng = np.random.default_rng(P)
    w0 = rng.standard_normal(N).astype(np.float32)
    weights = torch.from_numpy(w0).to(dev)
    kern.sum(grads, w.lr, total)
    kern.finish(total, w.P, dense, weights)
    torch.cuda.synchronize()
    host = [synth.worker_grads_host(w, p, 0) for p in range(w.P)]
    want = lo.dense_sgd_update(host, w.lr)
    assert np.array_equal(_u32(dense), want.view(np.uint32))
    assert np.array_equal(_u32(weights), lo.apply_update(w0, want).view(np.uint32))


def test_dense_full_vgg16_sampled_windows():
    # the update is independent per position: windows of the full-size output
    # (with ragged edges) against the oracle on the same windows
    import torch
    from layer_wise_top_b200 import DenseKernels
    w = WORKLOADS["vgg16"]
    N, P = w.N, w.P
    dev = torch.device("cuda")
    grads = [torch.empty(N, device=dev) for _ in range(P)]
    for p in range(P):
        synth.worker_grads_device(w, p, 3, grads[p])
    kern = DenseKernels(N, dev)
    total = torch.empty(N, device=dev)
    dense = torch.empty(N, device=dev)
    kern.sum(grads, w.lr, total)
    kern.finish(total, P, dense)
    torch.cuda.synchronize()
    host = [synth.worker_grads_host(w, p, 3) for p in range(P)]
    for a, b in [(0, 4099), (N // 2 - 3, N // 2 + 70001), (N - 9999, N)]:
        want = lo.dense_sgd_update([h[a:b] for h in host], w.lr)
        assert np.array_equal(_u32(dense[a:b]), want.view(np.uint32)), (a, b)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dense_sgd_one_rank_equals_lags_at_density_one():
    import torch
    import torch.distributed as dist
    from layer_wise_top_b200 import Plan
    from layer_wise_top_b200.dist import DenseSgd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = WORKLOADS["resnet20"]
        P, N = w.P, w.N
        dense_sgd = DenseSgd.create(N, P, dev)
        plan = Plan(w.sizes, [1.0] * w.L, P, device=dev)
        grads = [torch.empty(N, device=dev) for _ in range(P)]
        res = [torch.zeros(N, device=dev) for _ in range(P)]
        idx, val = plan.empty_picks()
        d_a, d_b = torch.empty(N, device=dev), torch.empty(N, device=dev)
        w_a, w_b = torch.zeros(N, device=dev), torch.zeros(N, device=dev)
        for s in range(3):
            for p in range(P):
                synth.worker_grads_device(w, p, s, grads[p])
            dense_sgd.step(grads, w.lr, d_a, w_a)
            plan.sparsify(grads, res, w.lr, idx, val)
            plan.aggregate_apply(idx, val, d_b, w_b)
        torch.cuda.synchronize()
        assert np.array_equal(_u32(d_a), _u32(d_b))
        assert np.array_equal(_u32(w_a), _u32(w_b))
    finally:
        dist.destroy_process_group()
