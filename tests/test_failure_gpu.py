"""Failure reporting on the GPU, without faulting it: the selection's bounded
wait is made to give up at once (a limit of 0 polls on its staging barrier),
which must be reported as LAGS_FLAG_TIMEOUT / LAGS_ERR_TIMEOUT by the status
poll while the picks, found from global memory instead, stay exact; a plan
bound to the aggregation-only workspace refuses to sparsify."""
import numpy as np
import pytest

import oracle.lags_oracle as lo
import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu

F32 = np.float32


def _u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def _run_against_oracle(sizes, dens, P, lr, steps, grad_fn, wait_limit, index_limit=None):
    """Steps with the given staging-wait limit (and index-copy wait limit);
    every output compared with the oracle.  Returns the (status, flags,
    fallbacks) of each step's poll."""
    import torch
    import layer_wise_top_b200 as L
    from gpu_harness import GpuRun
    run = GpuRun(sizes, dens, P, lr)
    run.plan.set_stage_wait_limit(wait_limit)
    if index_limit is not None:
        run.plan.set_index_wait_limit(index_limit)
    hist = lo.run_workload(sizes, dens, P, lr, steps, grad_fn)
    polls = []
    for s in range(steps):
        for p in range(P):
            run.grads[p].copy_(torch.from_numpy(grad_fn(p, s)))
        run.step(fused=s % 2 == 1)
        try:
            flags, fb = run.plan.poll()
            polls.append((L.LAGS_OK, flags, fb))
        except L.LagsError as e:
            polls.append((e.status, e.flags, e.fallbacks))
        e_idx, e_val, e_res, e_dense, e_w = hist[s]
        K = run.plan.K
        assert np.array_equal(_u32(run.idx).reshape(P, K), e_idx), f"step {s}: idx"
        assert np.array_equal(_u32(run.val).reshape(P, K), e_val.view(np.uint32)), f"step {s}"
        for p in range(P):
            assert np.array_equal(_u32(run.res[p]), e_res[p].view(np.uint32)), f"step {s} res {p}"
        assert np.array_equal(_u32(run.dense), e_dense.view(np.uint32)), f"step {s}: dense"
        assert np.array_equal(_u32(run.weights), e_w.view(np.uint32)), f"step {s}: weights"
    return polls


def test_staging_wait_timeout_is_reported_and_picks_stay_exact():
    import layer_wise_top_b200 as L
    w = WORKLOADS["resnet20"]
    cache = {}

    def fn(p, s):
        if (p, s) not in cache:
            cache[(p, s)] = synth.worker_grads_host(w, p, s)
        return cache[(p, s)]
    polls = _run_against_oracle(w.sizes, w.densities, w.P, w.lr, 3, fn, wait_limit=0)
    for status, flags, fb in polls:
        assert status == L.LAGS_ERR_TIMEOUT
        assert flags & L.LAGS_FLAG_TIMEOUT
        assert not flags & L.LAGS_FLAG_INTERNAL and fb == 0


def _crowded_tile_case():
    # one tile of a 40-tile layer holds 5000 values a thousand times larger
    # than the rest (k = 3277): far more candidates than that tile's slots
    # (a few thousand at most), few enough for the selecting CTA to stage (it
    # recompacts the tile from its acc)
    rng = np.random.default_rng(17)
    sizes = [40 * 8192, 12345, 5000]
    dens = [0.01, 0.001, 1.0]
    N = sum(sizes)
    data = {}
    for p in range(2):
        for s in range(3):
            g = rng.standard_normal(N).astype(F32)
            g[7 * 8192 + 1000 + 300 * p:7 * 8192 + 6000 + 300 * p] *= F32(1000.0)
            data[(p, s)] = g
    return sizes, dens, lambda p, s: data[(p, s)]


def test_crowded_tile_recompaction_exact():
    import layer_wise_top_b200 as L
    sizes, dens, fn = _crowded_tile_case()
    polls = _run_against_oracle(sizes, dens, 2, 1.0, 3, fn,
                                wait_limit=L.LAGS_STAGE_WAIT_POLLS)
    for status, flags, fb in polls:
        assert status == L.LAGS_OK and flags == 0
        assert fb == 0  # staged and recompacted, not the exhaustive path


def test_values_only_select_with_recompacted_tiles_exact():
    # 4-CTA values-only selects (19 layers x 2 workers fill the GPU) where one
    # tile of every layer holds 6000 values three times larger than the rest:
    # about 2.2k candidates there, more than the tile's ~1.5k slots, so the
    # CTA recompacts the tile from its acc and recovers those picks' indices
    # with a second walk (moderate scaling keeps the sampled threshold below
    # the k-th largest even when a sample run lands in the crowded tile)
    import layer_wise_top_b200 as L
    # (a seed whose sampled thresholds keep the k largest of every segment in
    # both steps, so every segment takes the staged path checked here)
    rng = np.random.default_rng(37)
    sizes = [2_000_003 + 977 * i for i in range(19)] + [3]
    dens = [0.005] * 19 + [1.0]
    N = sum(sizes)
    offs = np.cumsum([0] + sizes[:-1])
    data = {}
    for p in range(2):
        for s in range(2):
            g = rng.standard_normal(N).astype(F32)
            for o in offs[:19]:
                a = int(o) + 91 * 8192 + 700 + 200 * p
                g[a:a + 6000] *= F32(3.0)
            data[(p, s)] = g
    polls = _run_against_oracle(sizes, dens, 2, 1.0, 2, lambda p, s: data[(p, s)],
                                wait_limit=L.LAGS_STAGE_WAIT_POLLS)
    for status, flags, fb in polls:
        assert status == L.LAGS_OK and flags == 0
        assert fb == 0  # staged and recompacted, not the exhaustive path


def test_timeout_with_overflowed_tile_walks_acc_exactly():
    # after a timeout the selecting CTA takes its candidates from acc, so an
    # overflowed tile (only part of its candidates in the slots) is complete
    import layer_wise_top_b200 as L
    sizes, dens, fn = _crowded_tile_case()
    polls = _run_against_oracle(sizes, dens, 2, 1.0, 3, fn, wait_limit=0)
    for status, flags, fb in polls:
        assert status == L.LAGS_ERR_TIMEOUT and flags == L.LAGS_FLAG_TIMEOUT and fb == 0


def test_index_copy_wait_timeout_reads_slots_exactly():
    # 4-CTA values-only selects (19 layers x 2 workers fill the GPU) whose
    # wait for the index copies gives up at once: each pick's index comes from
    # its candidate slot instead, and the poll reports the timeout
    import layer_wise_top_b200 as L
    from gpu_harness import synth_grad_fn
    sizes = [400_003 + 977 * i for i in range(19)] + [3]
    dens = [0.05] * 19 + [1.0]
    w = WORKLOADS["lstm_ptb"].scaled("mid", P=2, steps=2,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    polls = _run_against_oracle(sizes, dens, 2, w.lr, 2, synth_grad_fn(w),
                                wait_limit=L.LAGS_STAGE_WAIT_POLLS, index_limit=0)
    for status, flags, fb in polls:
        assert status == L.LAGS_ERR_TIMEOUT and flags == L.LAGS_FLAG_TIMEOUT and fb == 0


def test_aggregate_only_plan():
    import torch
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    w = WORKLOADS["vgg16"].scaled("vgg_head", P=4,
                                  tensors=WORKLOADS["vgg16"].tensors[:12])
    full = Plan(w.sizes, w.densities, w.P)
    agg = Plan(w.sizes, w.densities, w.P, aggregate_only=True)
    assert agg.workspace_bytes < full.workspace_bytes
    dev = torch.device("cuda")
    grads = [torch.empty(w.N, device=dev) for _ in range(w.P)]
    res = [torch.zeros(w.N, device=dev) for _ in range(w.P)]
    for p in range(w.P):
        synth.worker_grads_device(w, p, 0, grads[p])
    idx, val = full.empty_picks()
    with pytest.raises(L.LagsError) as e:
        agg.sparsify(grads, res, w.lr, idx, val)
    assert e.value.status == L.LAGS_ERR_WORKSPACE
    full.sparsify(grads, res, w.lr, idx, val)
    d_full, d_agg = torch.empty(w.N, device=dev), torch.empty(w.N, device=dev)
    w_full, w_agg = torch.zeros(w.N, device=dev), torch.zeros(w.N, device=dev)
    full.aggregate_apply(idx, val, d_full, w_full)
    agg.aggregate_apply(idx, val, d_agg, w_agg)
    assert full.poll() == (0, 0) and agg.poll() == (0, 0)
    assert np.array_equal(_u32(d_full), _u32(d_agg))
    assert np.array_equal(_u32(w_full), _u32(w_agg))


def test_calls_on_another_device_are_refused():
    import torch
    import layer_wise_top_b200 as L
    from layer_wise_top_b200 import Plan
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two devices")
    plan = Plan([1000], [0.01], 1, device=torch.device("cuda", 0))
    with torch.cuda.device(1):
        with pytest.raises(L.LagsError) as e:
            L.lags_aggregate(plan.handle, 256, 256, 256)
        assert e.value.status == L.LAGS_ERR_WRONG_DEVICE
