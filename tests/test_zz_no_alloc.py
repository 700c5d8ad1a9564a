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


def _two_calls_match(w, sizes=None, dens=None, static_wait_limit=None):
    import torch
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    sizes = sizes or w.sizes
    dens = dens or w.densities
    P, N = w.P, sum(sizes)
    plan = Plan(sizes, dens, P)           # the workspace path, for reference
    stream = torch.cuda.current_stream().cuda_stream
    try:                                  # start from clear static status words
        L.lags_static_status_poll(stream)
    except L.LagsError:
        pass
    dev = torch.device("cuda")
    grads = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)]
    res_ws = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
    res_st = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
    idx_ws, val_ws = plan.empty_picks()
    idx_st, val_st = plan.empty_picks()
    for step in range(2):                 # two calls in a row: residuals carry over
        for p in range(P):
            synth.worker_grads_device(w, p, step, grads[p])
        plan.sparsify(grads, res_ws, w.lr, idx_ws, val_ws)
        if static_wait_limit is not None:
            plan.set_stage_wait_limit(static_wait_limit)
        L.lags_sparsify_static(plan.handle, [g.data_ptr() for g in grads],
                               [r.data_ptr() for r in res_st], w.lr, idx_st.data_ptr(),
                               val_st.data_ptr(), stream)
        if static_wait_limit is not None:
            plan.set_stage_wait_limit(L.LAGS_STAGE_WAIT_POLLS)
            # the injected timeout is reported through the static status words
            with pytest.raises(L.LagsError) as e:
                L.lags_static_status_poll(stream)
            assert e.value.status == L.LAGS_ERR_TIMEOUT
            assert e.value.flags == L.LAGS_FLAG_TIMEOUT
        else:
            assert L.lags_static_status_poll(stream) == (0, 0)
        assert plan.poll() == (0, 0)
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


def test_static_timeout_reported_by_static_poll():
    # a staging wait limit of 0 makes the selection give up at once; the
    # static path reports it in its own status words, and the picks, found
    # from global memory instead, still equal the workspace path's
    _two_calls_match(WORKLOADS["resnet20"], static_wait_limit=0)


_FRESH = r"""
import sys
import numpy as np
import torch
import layer_wise_top_b200 as L
from layer_wise_top_b200 import Plan
import synth
from synth.configs import WORKLOADS
w = WORKLOADS["resnet20"]
P, N = w.P, w.N
dev = torch.device("cuda")
grads = [torch.empty(N, device=dev) for _ in range(P)]
res_st = [torch.zeros(N, device=dev) for _ in range(P)]
res_ws = [torch.zeros(N, device=dev) for _ in range(P)]
h = L.lags_plan_create(w.sizes, w.densities, P)   # no workspace bound, ever
K = L.lags_plan_info(h)[1]
idx_st = torch.empty(P * K, dtype=torch.int32, device=dev)
val_st = torch.empty(P * K, device=dev)
outs = []
for step in range(2):
    for p in range(P):
        synth.worker_grads_device(w, p, step, grads[p])
    # the first call in this process sets the static path up itself
    L.lags_sparsify_static(h, [g.data_ptr() for g in grads], [r.data_ptr() for r in res_st],
                           w.lr, idx_st.data_ptr(), val_st.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
    assert L.lags_static_status_poll(torch.cuda.current_stream().cuda_stream) == (0, 0)
    outs.append((idx_st.clone(), val_st.clone(), [r.clone() for r in res_st]))
L.lags_plan_destroy(h)
# the workspace path afterwards, on the same inputs
plan = Plan(w.sizes, w.densities, P)
idx, val = plan.empty_picks()
u = lambda t: t.cpu().numpy().view(np.uint32)
for step in range(2):
    for p in range(P):
        synth.worker_grads_device(w, p, step, grads[p])
    plan.sparsify(grads, res_ws, w.lr, idx, val)
    assert plan.poll() == (0, 0)
    i_st, v_st, r_st = outs[step]
    assert np.array_equal(u(i_st), u(idx)), step
    assert np.array_equal(u(v_st), u(val)), step
    for a, b in zip(r_st, res_ws):
        assert np.array_equal(u(a), u(b)), step
print("FRESH_OK")
"""


def test_static_first_in_fresh_process_without_workspace():
    """The advertised use: a plan that never gets a workspace, and the static
    entry point's own first-call set-up, in a process where nothing else has
    configured the kernels."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root + os.pathsep + os.environ.get("PYTHONPATH", ""))
    out = subprocess.run([sys.executable, "-c", _FRESH], cwd=root, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and "FRESH_OK" in out.stdout, out.stdout + out.stderr


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


_EXIT_WITH_PLAN = """
import torch
from layer_wise_top_b200 import Plan
plan = Plan([1000, 77], [0.01, 1.0], 2)   # still alive when the interpreter exits
idx, val = plan.empty_picks()
torch.cuda.synchronize()
print("EXIT_OK")
"""


def test_plan_alive_at_interpreter_exit_is_destroyed_quietly():
    """A Plan held by a module global is destroyed during interpreter exit,
    after the binding's globals may be gone: no exception is reported."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root + os.pathsep + os.environ.get("PYTHONPATH", ""))
    out = subprocess.run([sys.executable, "-c", _EXIT_WITH_PLAN], cwd=root, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and "EXIT_OK" in out.stdout, out.stdout + out.stderr
    assert "Exception ignored" not in out.stderr and "Traceback" not in out.stderr, out.stderr
