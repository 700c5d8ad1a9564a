"""CUDA path vs the CPU oracle, bit for bit, through the C ABI.

Small cases are compared element by element over every output.  The
full-size workloads are compared element by element on sampled layers, among
them each workload's largest layers (the oracle replays those layers for all
workers, which is exact because layers are independent), and on the
invariants that determine the result uniquely, for every layer and worker."""
import numpy as np
import pytest

import oracle.lags_oracle as lo
import synth
from synth.configs import WORKLOADS, Tensor

pytestmark = pytest.mark.gpu

F32 = np.float32

from gpu_harness import run_full_compare, same_bits_or_nan, synth_grad_fn  # noqa: E402


def _torch():
    import torch
    return torch


# ----------------------------------------------------------------- full small
def test_resnet20_all_steps_bitexact():
    w = WORKLOADS["resnet20"]
    run_full_compare(w.sizes, w.densities, w.P, w.lr, w.steps, synth_grad_fn(w),
                     expect_fallbacks=lambda fb: fb == 0)


RAGGED = [1, 3, 5, 7, 8191, 8192, 8193, 20000, 100003, 36864, 2, 65537]


@pytest.mark.parametrize("dist", [synth.NORMAL, synth.STUDENT_T3])
def test_ragged_layers_mixed_density(dist):
    rng = np.random.default_rng(11)
    dens = [float(x) for x in rng.choice([0.001, 0.01, 0.1, 0.5, 1.0], len(RAGGED))]
    w = WORKLOADS["resnet20"].scaled(
        "ragged", P=3, steps=4,
        tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(RAGGED)],
        density_rule=lambda d: 0.0)
    w = type(w)(w.name, w.tensors, w.P, 0.5, w.steps, dist, 21, w.density_rule)
    run_full_compare(RAGGED, dens, w.P, w.lr, w.steps, synth_grad_fn(w))


def test_large_layers_cluster_select():
    # up to ~15k expected candidates: one-CTA selects
    sizes = [1_100_003, 5, 2_000_001, 1 << 20]
    dens = [0.001, 1.0, 0.003, 0.01]
    w = WORKLOADS["lstm_ptb"].scaled("big", P=2, steps=3,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    run_full_compare(sizes, dens, 2, w.lr, 3, synth_grad_fn(w),
                     expect_fallbacks=lambda fb: fb == 0)


def test_four_cta_values_only_cluster_select():
    # ~23k expected candidates per layer: 4-CTA clusters staging values only
    # (the picks' indices read back from the candidate slots); 19 layers x 2
    # workers make the launch fill the GPU (at least one CTA per SM)
    sizes = [400_003 + 977 * i for i in range(19)] + [3]
    dens = [0.05] * 19 + [1.0]
    w = WORKLOADS["lstm_ptb"].scaled("mid", P=2, steps=2,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    run_full_compare(sizes, dens, 2, w.lr, 2, synth_grad_fn(w),
                     expect_fallbacks=lambda fb: fb == 0)


def test_eight_cta_cluster_select():
    # ~57k expected candidates: an 8-CTA cluster
    sizes = [4_000_037, 3, 129]
    dens = [0.01, 1.0, 0.5]
    w = WORKLOADS["lstm_ptb"].scaled("large", P=2, steps=3,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    run_full_compare(sizes, dens, 2, w.lr, 3, synth_grad_fn(w),
                     expect_fallbacks=lambda fb: fb == 0)


def test_sixteen_cta_cluster_select():
    # ~149k expected candidates: more than eight CTAs stage, so the layer is
    # selected by a 16-CTA cluster (or 8 CTAs reading from global memory if
    # the device cannot host the larger cluster)
    sizes = [2_600_000, 7]
    dens = [0.05, 1.0]
    w = WORKLOADS["resnet50"].scaled("huge", P=2, steps=2,
                                     tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    run_full_compare(sizes, dens, 2, w.lr, 2, synth_grad_fn(w),
                     expect_fallbacks=lambda fb: fb == 0)


# ----------------------------------------------------------------- ties / degenerate
def _np_grads(gen, sizes, P, steps):
    N = sum(sizes)
    data = {(p, s): gen(N) for p in range(P) for s in range(steps)}
    return lambda p, s: data[(p, s)]


def test_integer_ties_force_exact_path():
    rng = np.random.default_rng(5)
    sizes = [9000, 40000, 1_048_577, 17, 600_000]
    dens = [0.01, 0.001, 0.001, 0.3, 0.01]
    fn = _np_grads(lambda n: rng.integers(-2, 3, n).astype(F32), sizes, 2, 3)
    fb = run_full_compare(sizes, dens, 2, 1.0, 3, fn)
    assert fb > 0  # massive ties overflow the candidate slots


def test_all_zero_gradients():
    # all picks tie at 0 and go to the lowest indices: the first tile of the
    # 1M layer at 0.005 receives 2 x 5243 picks, more than aggregation stages
    sizes = [100, 8192, 30000, 1_048_576, 600_000, 1_000_000]
    fn = _np_grads(lambda n: np.zeros(n, dtype=F32), sizes, 2, 2)
    run_full_compare(sizes, [0.01, 0.001, 0.5, 0.001, 0.01, 0.005], 2, 0.1, 2, fn)


def test_signed_zero_denormal_inf():
    rng = np.random.default_rng(6)

    def gen(n):
        x = rng.standard_normal(n).astype(F32)
        x[rng.random(n) < 0.3] = F32(-0.0)
        x[rng.random(n) < 0.1] = F32(0.0)
        x[rng.random(n) < 0.05] = (rng.integers(1, 100, 1) * F32(1e-45)).astype(F32)[0]
        x[rng.random(n) < 0.0005] = F32(np.inf)
        x[rng.random(n) < 0.0005] = F32(-np.inf)
        return x
    sizes = [5000, 70000, 3]
    fn = _np_grads(gen, sizes, 3, 2)
    run_full_compare(sizes, [0.01, 0.001, 1.0], 3, 1.0, 2, fn)


def test_single_worker_and_k_equals_d():
    rng = np.random.default_rng(7)
    sizes = [4096, 10, 12345]
    fn = _np_grads(lambda n: rng.standard_normal(n).astype(F32), sizes, 1, 2)
    run_full_compare(sizes, [1.0, 1.0, 0.999], 1, 0.1, 2, fn)


def test_k_equals_one_everywhere():
    rng = np.random.default_rng(8)
    sizes = [1, 2, 3, 64, 9000, 300000]
    fn = _np_grads(lambda n: rng.standard_normal(n).astype(F32), sizes, 4, 2)
    run_full_compare(sizes, [1e-9] * len(sizes), 4, 0.1, 2, fn)


def test_deterministic_repeat():
    torch = _torch()
    from gpu_harness import GpuRun, u32
    w = WORKLOADS["vgg16"]
    outs = []
    for _ in range(2):
        run = GpuRun(w.sizes, w.densities, w.P, w.lr)
        for s in range(2):
            for p in range(w.P):
                synth.worker_grads_device(w, p, s, run.grads[p])
            run.step()
        torch.cuda.synchronize()
        outs.append((u32(run.idx), u32(run.val), u32(run.dense), u32(run.res[3])))
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


# ----------------------------------------------------------------- full size
SAMPLED = {
    "vgg16": [1, 0, 2, 27, 26],                      # biases, conv0, conv1, fc
    "resnet50": [1, 2, 0, 3, 12, 15, 160, 41],       # BN (dense), convs at 0.01, fc bias
    "lstm_ptb": [2, 3, 8],                           # the bias vectors
    "gpt_1_3b": [1, 2, 5, 6],                        # LayerNorm gamma/beta
}
# Large layers replayed through the oracle for every worker over the first
# steps (in spawned processes, while the GPU runs): they are selected by the
# clustered kernels and, above 2^23 elements, sampled with short runs.
BIG = {
    "vgg16": ([16], 10),          # conv8 3x3x512x512, k = 2360 (one-CTA select)
    "resnet50": ([132], 10),      # layer4.0.conv2, k = 2360
    "lstm_ptb": ([1], 3),         # lstm0.weight 6000x3000, k = 18000 (4-CTA cluster)
    "gpt_1_3b": ([0, 7], 2),      # wte 50304x2048, k = 103,023 (16-CTA cluster, short
                                  # sample runs); h0.mlp.fc1 8192x2048, k = 16,778
                                  # (4-CTA cluster)
}


def _full_size(name, steps):
    torch = _torch()
    import oracle_jobs
    from gpu_harness import GpuRun, check_invariants, compare_layer, oracle_layer_steps
    w = WORKLOADS[name]
    big_layers, big_steps = BIG[name]
    big_bytes = max(w.sizes[l] for l in big_layers) * 40  # grads, residual, sort keys
    with oracle_jobs.pool(len(big_layers) * w.P, big_bytes) as ex:
        futures = oracle_jobs.submit_layers(ex, name, big_layers, range(w.P), big_steps)
        run = GpuRun(w.sizes, w.densities, w.P, w.lr, keep_prev=True)
        exp = {}
        for l in SAMPLED[name]:
            off, k, _ = run.plan.layers[l]
            exp[l] = oracle_layer_steps(off, w.sizes[l], k, w.P, w.lr, steps,
                                        lambda p, s, l=l: synth.layer_grads_host(w, p, s, l))
        big = None
        fallbacks = 0
        for s in range(steps):
            for p in range(w.P):
                synth.worker_grads_device(w, p, s, run.grads[p])
            run.step(fused=s % 2 == 1)
            flags, fb = run.plan.poll()
            assert flags == 0
            fallbacks += fb
            for l in SAMPLED[name]:
                compare_layer(run, l, exp[l][s], f"{name} step {s} layer {l}")
            if s < big_steps:
                if big is None:
                    big = {l: oracle_jobs.layer_history(futures, name, l, w.P)
                           for l in big_layers}
                for l in big_layers:
                    compare_layer(run, l, big[l][s], f"{name} step {s} large layer {l}")
            check_invariants(run, range(w.P), check_dense=True)
    assert fallbacks == 0, f"{fallbacks} segments took the exhaustive path"


def test_full_vgg16():
    _full_size("vgg16", 10)


def test_full_resnet50():
    _full_size("resnet50", 10)


def test_full_lstm():
    _full_size("lstm_ptb", 10)


@pytest.mark.slow
def test_full_gpt_1_3b():
    _full_size("gpt_1_3b", 2)


@pytest.mark.parametrize("fused", [False, True])
def test_negative_zero_weights_and_underflowing_update(fused):
    """Updates of -tiny / P round to -0; w - (-0) turns a -0 weight into +0,
    so skipping such an update would be visible.  Weights start at -0."""
    torch = _torch()
    from gpu_harness import GpuRun, u32
    rng = np.random.default_rng(9)
    sizes, dens, P = [64, 10000, 8193], [1.0, 0.01, 0.001], 16
    N = sum(sizes)
    grads = []
    for p in range(P):
        g = np.zeros(N, dtype=F32)
        hot = rng.choice(N, 300, replace=False)
        g[hot] = (rng.integers(1, 4, hot.size) * np.float32(-1e-45)).astype(F32)
        g[hot[:50]] = F32(1e-45)
        grads.append(g)
    run = GpuRun(sizes, dens, P, 1.0)
    run.weights.fill_(-0.0)
    for p in range(P):
        run.grads[p].copy_(torch.from_numpy(grads[p]))
    run.step(fused=fused)
    res0 = [np.zeros(N, dtype=F32) for _ in range(P)]
    e_idx, e_val, e_res = lo.sparsify(sizes, dens, grads, res0, 1.0)
    e_dense = lo.aggregate(N, e_idx, e_val)
    e_w = lo.apply_update(np.full(N, -0.0, dtype=F32), e_dense)
    assert np.signbit(e_dense).any() and not np.signbit(e_w).all()  # the case occurs
    assert np.array_equal(u32(run.dense), e_dense.view(np.uint32))
    assert np.array_equal(u32(run.weights), e_w.view(np.uint32))
