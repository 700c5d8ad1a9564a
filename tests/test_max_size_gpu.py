"""The largest plan on the GPU: N = LAGS_MAX_ELEMENTS (2^32 - 65536), one
worker, two steps.  The small ragged layers at the top of the index range are
compared with the oracle bit for bit.  The 4.29-billion-element layer below
them is checked, in chunks on the GPU, against the properties that fix its
top-k: picks ascending and inside the layer, each value equal to acc at its
index, picked residuals +0 and all others acc, every picked magnitude at
least every unpicked one, ties to the lower index, and the dense update equal
to the picks (P = 1) and +0 elsewhere.  About 105 GB of device memory."""
import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28


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


def _bits(t):
    import torch
    return t.view(torch.int32)


def test_max_size_plan():
    import torch
    from gpu_harness import GpuRun, compare_layer, oracle_layer_steps
    w = _workload()
    run = GpuRun(w.sizes, w.densities, 1, w.lr, keep_prev=True)
    assert run.plan.N == w.N
    exp = {}
    for l in (1, 2, 3):
        off, k, _ = run.plan.layers[l]
        exp[l] = oracle_layer_steps(off, w.sizes[l], k, 1, w.lr, w.steps,
                                    lambda p, s, l=l: synth.layer_grads_host(w, p, s, l))
    off0, k0, koff0 = run.plan.layers[0]
    d0 = w.sizes[0]
    lr = torch.tensor(w.lr, dtype=torch.float32, device="cuda")
    for s in range(w.steps):
        synth.worker_grads_device(w, 0, s, run.grads[0])
        run.step(fused=s == 1)
        flags, _ = run.plan.poll()
        assert flags == 0
        for l in (1, 2, 3):
            compare_layer(run, l, exp[l][s], f"max size step {s} layer {l}")

        # ---- the 4.29-billion-element layer ----
        idx = run.idx[koff0:koff0 + k0].to(torch.int64) & 0xFFFFFFFF
        val = run.val[koff0:koff0 + k0]
        assert bool((idx[1:] > idx[:-1]).all()) and int(idx[0]) >= off0
        assert int(idx[-1]) < off0 + d0
        g, prev, res, dense = run.grads[0], run.prev[0], run.res[0], run.dense
        acc_at = prev[idx] + lr * g[idx]
        assert torch.equal(_bits(val), _bits(acc_at))
        assert int(_bits(res[idx]).abs().max()) == 0  # +0 exactly
        vmin = float(val.abs().min())
        top_unpicked = 0.0
        first_tie = None  # lowest unpicked index whose magnitude equals vmin
        for a in range(off0, off0 + d0, CHUNK):
            b = min(a + CHUNK, off0 + d0)
            acc = prev[a:b] + lr * g[a:b]
            sel = idx[(idx >= a) & (idx < b)] - a
            want = acc.clone()
            want[sel] = 0.0
            assert torch.equal(_bits(res[a:b]), _bits(want)), f"residual chunk {a}"
            mag = want.abs()
            mag[sel] = -1.0  # picked: out of the unpicked maximum
            top_unpicked = max(top_unpicked, float(mag.max()))
            ties = torch.nonzero(mag == vmin)
            if first_tie is None and ties.numel():
                first_tie = a + int(ties[0])
            dz = dense[a:b].clone()
            assert torch.equal(_bits(dz[sel]), _bits(val[(idx >= a) & (idx < b)]))
            dz[sel] = 0.0
            assert int(_bits(dz).abs().max()) == 0, f"dense chunk {a}"
        assert vmin >= top_unpicked
        if first_tie is not None:
            picked_ties = idx[val.abs() == vmin]
            assert first_tie > int(picked_ties.max())
        torch.cuda.synchronize()
    del run, g, prev, res, dense
    torch.cuda.empty_cache()  # about 100 GB: leave the device to the next tests
