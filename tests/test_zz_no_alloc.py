"""lags_sparsify_static, the entry point for callers that cannot allocate
device memory (code inside an allocator or memory-pool callback, runtimes that
own every device allocation, hosts that forbid cudaMalloc after start-up).  It
keeps its scratch in a 16 MiB array with static storage instead of a
caller-provided workspace, and must give exactly what lags_sparsify gives.

This file is collected last on purpose; it runs alone in a fresh process as
well as after the other tests."""
import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def _two_calls_match(w, sizes=None, dens=None):
    import torch
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    sizes = sizes or w.sizes
    dens = dens or w.densities
    P, N = w.P, sum(sizes)
    plan = Plan(sizes, dens, P)           # the workspace path, for reference
    dev = torch.device("cuda")
    grads = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)]
    res_ws = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
    res_st = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
    idx_ws, val_ws = plan.empty_picks()
    idx_st, val_st = plan.empty_picks()
    stream = torch.cuda.current_stream().cuda_stream
    for step in range(2):                 # two calls in a row: residuals carry over
        for p in range(P):
            synth.worker_grads_device(w, p, step, grads[p])
        plan.sparsify(grads, res_ws, w.lr, idx_ws, val_ws)
        L.lags_sparsify_static(plan.handle, [g.data_ptr() for g in grads],
                               [r.data_ptr() for r in res_st], w.lr, idx_st.data_ptr(),
                               val_st.data_ptr(), stream)
        torch.cuda.synchronize()
        # the library's tests demand bit-identical results
        assert np.array_equal(_u32(idx_st), _u32(idx_ws)), f"call {step}: indices"
        assert np.array_equal(_u32(val_st), _u32(val_ws)), f"call {step}: values"
        for p in range(P):
            assert np.array_equal(_u32(res_st[p]), _u32(res_ws[p])), f"call {step}: residual {p}"


def test_static_scratch_matches_workspace_resnet20():
    _two_calls_match(WORKLOADS["resnet20"])


def test_static_scratch_matches_workspace_ragged():
    sizes = [3, 8193, 65537, 1 << 20, 11]
    dens = [1.0, 0.01, 0.001, 0.001, 0.5]
    w = WORKLOADS["lstm_ptb"].scaled("ragged", P=3,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    _two_calls_match(w, sizes, dens)


def test_static_scratch_rejects_large_plan():
    import layer_wise_top_b200 as L
    w = WORKLOADS["resnet50"]            # workspace of ~118 MB > 16 MiB
    h = L.lags_plan_create(w.sizes, w.densities, w.P)
    try:
        with pytest.raises(L.LagsError) as e:
            L.lags_sparsify_static(h, [16] * w.P, [16] * w.P, 0.1, 16, 16)
        assert e.value.status == L.LAGS_ERR_WORKSPACE
    finally:
        L.lags_plan_destroy(h)
