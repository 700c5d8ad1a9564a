"""Seeded random plans against the CPU oracle, every output bit for bit.

Each case draws the layer count, the layer sizes (tiny layers, sizes a few
elements either side of a tile multiple, mid-size and large layers), the
per-layer densities (dense layers among them), the worker count, the learning
rate and the gradient distribution, then runs several steps through the C ABI
and compares the pick lists, residuals, dense update and weights of every step
with the oracle's."""
import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS, Tensor

from gpu_harness import run_full_compare, synth_grad_fn

pytestmark = pytest.mark.gpu

TILE = 8192
N_CASES = 24


def _case(seed: int):
    rng = np.random.default_rng(1000 + seed)
    sizes = []
    for _ in range(int(rng.integers(1, 11))):
        kind = int(rng.integers(0, 4))
        if kind == 0:
            d = int(rng.integers(1, 65))
        elif kind == 1:
            d = TILE * int(rng.integers(1, 9)) + int(rng.integers(-5, 6))
        elif kind == 2:
            d = int(rng.integers(100, 50_001))
        else:
            d = int(rng.integers(100_000, 700_001))
        sizes.append(max(1, d))
    dens = [float(x) for x in rng.choice([0.0005, 0.001, 0.01, 0.05, 0.3, 1.0], len(sizes))]
    P = int(rng.integers(1, 7))
    steps = int(rng.integers(2, 4))
    lr = float(rng.choice([0.5, 0.01]))
    dist = synth.NORMAL if rng.integers(0, 2) == 0 else synth.STUDENT_T3
    base = WORKLOADS["resnet20"].scaled(
        f"fuzz{seed}", P=P, steps=steps,
        tensors=[Tensor(f"t{i}", (d,)) for i, d in enumerate(sizes)])
    w = type(base)(base.name, base.tensors, P, lr, steps, dist, 5000 + seed, base.density_rule)
    return sizes, dens, w


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_plan_matches_oracle(seed):
    sizes, dens, w = _case(seed)
    run_full_compare(sizes, dens, w.P, w.lr, w.steps, synth_grad_fn(w))
