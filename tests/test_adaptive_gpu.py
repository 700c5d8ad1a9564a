"""Adaptive densities end to end on the GPU: each layer's backward time is
measured (CUDA events around a synthetic backward), the library's planner
turns the times into densities (communication-to-computation ratio, "Layer-
wise Adaptive Gradient Sparsification ..." review, "proposed method"), and a
plan at those densities runs steps that equal the oracle bit for bit."""
import numpy as np
import pytest

import oracle.lags_oracle as lo
from synth.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def test_measured_times_and_planned_densities():
    from layer_wise_top_b200 import adaptive
    w = WORKLOADS["resnet50"]
    shapes = [t.shape for t in w.tensors]
    secs = adaptive.measure_backward_seconds(shapes, rows=2048, repeats=3)
    assert len(secs) == w.L and all(s > 0.0 for s in secs)
    # a 3x3x512x512 convolution's GEMMs take longer than a 64-wide BN scale
    assert secs[132] > secs[1]
    alpha, beta = adaptive.LINKS["10gbe"]
    rho = adaptive.adaptive_densities(w.sizes, secs, w.P, "10gbe", 0.001)
    assert rho == lo.adaptive_densities(w.sizes, secs, alpha, beta * (w.P - 1), 0.001)
    assert all(0.001 <= r <= 1.0 for r in rho)


@pytest.mark.parametrize("name,P,steps", [("resnet20", 4, 3), ("resnet50", 2, 2)])
def test_adaptive_plan_equals_oracle(name, P, steps):
    from gpu_harness import run_full_compare, synth_grad_fn
    from layer_wise_top_b200 import adaptive
    w = WORKLOADS[name]
    rho, secs = adaptive.plan_densities([t.shape for t in w.tensors], w.P, "10gbe", 0.001,
                                        rows=2048)
    assert len(set(rho)) > 1, "the planner should give the layers different densities"
    w = w.scaled(f"{name}_p{P}", P=P)  # fewer workers keep the host oracle quick
    run_full_compare(w.sizes, rho, w.P, w.lr, steps, synth_grad_fn(w))
