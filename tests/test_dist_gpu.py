"""DataParallelLags with the real kernels on one GPU (a one-rank NCCL group):
the step through the exchange path equals the step of one plan holding all
workers, bit for bit."""
import datetime
import os
import socket

import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_dp_step_equals_plain_step():
    import torch
    import torch.distributed as dist
    from layer_wise_top_b200 import Plan
    from layer_wise_top_b200.dist import DataParallelLags
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = WORKLOADS["resnet20"]
        P, N = w.P, w.N
        dp = DataParallelLags.create(w.sizes, w.densities, P, dev)
        plan = Plan(w.sizes, w.densities, P, device=dev)
        grads = [torch.empty(N, device=dev) for _ in range(P)]
        res_a = [torch.zeros(N, device=dev) for _ in range(P)]
        res_b = [torch.zeros(N, device=dev) for _ in range(P)]
        dense_a, dense_b = torch.empty(N, device=dev), torch.empty(N, device=dev)
        w_a, w_b = torch.zeros(N, device=dev), torch.zeros(N, device=dev)
        idx, val = plan.empty_picks()
        for s in range(3):
            for p in range(P):
                synth.worker_grads_device(w, p, s, grads[p])
            dp.step(grads, res_a, w.lr, dense_a, w_a)
            plan.sparsify(grads, res_b, w.lr, idx, val)
            plan.aggregate_apply(idx, val, dense_b, w_b)
        torch.cuda.synchronize()
        u = lambda t: t.cpu().numpy().view(np.uint32)  # noqa: E731
        assert np.array_equal(u(dp.idx_all), u(idx))
        assert np.array_equal(u(dense_a), u(dense_b))
        assert np.array_equal(u(w_a), u(w_b))
        for a, b in zip(res_a, res_b):
            assert np.array_equal(u(a), u(b))
    finally:
        dist.destroy_process_group()
