"""The largest plan on the GPU: N = LAGS_MAX_ELEMENTS (2^32 - 65536), one
worker, two steps.  The small ragged layers at the top of the index range are
compared with the oracle bit for bit.  The 4.29-billion-element layer below
them is checked, in chunks on the GPU, against the properties that fix its
top-k: picks ascending and inside the layer, each value equal to acc at its
index, picked residuals +0 and all others acc, every picked magnitude at
least every unpicked one, ties to the lower index, and the dense update equal
to the picks (P = 1) and +0 elsewhere.  About 105 GB of device memory."""
import pytest

import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu

def _workload():
    import layer_wise_top_b200 as L
    tail = [8193, 100_003, 7]
    big = L.LAGS_MAX_ELEMENTS - sum(tail)
    sizes = [big] + tail
    dens = {big: 1e-7, 8193: 0.01, 100_003: 0.001, 7: 0.5}
    base = WORKLOADS["resnet20"]
    w = type(base)("max_size", [Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)], 1, 0.1, 2,
                   synth.NORMAL, 3, lambda d: dens[d])
    assert w.N == L.LAGS_MAX_ELEMENTS
    return w


def test_max_size_plan():
    import torch
    from gpu_harness import GpuRun, check_layer_chunked, compare_layer, oracle_layer_steps
    w = _workload()
    run = GpuRun(w.sizes, w.densities, 1, w.lr, keep_prev=True)
    assert run.plan.N == w.N
    exp = {}
    for l in (1, 2, 3):
        off, k, _ = run.plan.layers[l]
        exp[l] = oracle_layer_steps(off, w.sizes[l], k, 1, w.lr, w.steps,
                                    lambda p, s, l=l: synth.layer_grads_host(w, p, s, l))
    for s in range(w.steps):
        synth.worker_grads_device(w, 0, s, run.grads[0])
        run.step(fused=s == 1)
        flags, _ = run.plan.poll()
        assert flags == 0
        for l in (1, 2, 3):
            compare_layer(run, l, exp[l][s], f"max size step {s} layer {l}")
        check_layer_chunked(run, 0, w.lr)  # the 4.29-billion-element layer
        torch.cuda.synchronize()
    del run
    torch.cuda.empty_cache()  # about 100 GB: leave the device to the next tests
