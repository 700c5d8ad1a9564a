"""Adaptive per-layer densities (host planner in the C ABI) against the
oracle's restatement, a hand-worked fixture, special cases and the
"message hidden by the end of backward" property."""

import numpy as np
import pytest

import layer_wise_top_b200 as L
import oracle.lags_oracle as lo
from conftest import read_golden


def test_hand_example():
    g = read_golden("adaptive_two_layers.txt")
    args = ([int(x) for x in g["sizes"]], [float(x) for x in g["backward"]],
            float(g["alpha"][0]), float(g["beta"][0]), float(g["rho_min"][0]))
    exp = [float(x) for x in g["rho"]]
    assert L.lags_adaptive_densities(*args) == exp
    assert lo.adaptive_densities(*args) == exp


@pytest.mark.parametrize("seed", range(5))
def test_library_equals_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    sizes = [int(x) for x in rng.integers(1, 5_000_000, n)]
    t = [float(x) for x in rng.exponential(1e-3, n)]
    alpha, beta = float(rng.uniform(0, 5e-5)), float(rng.uniform(1e-11, 1e-8))
    assert L.lags_adaptive_densities(sizes, t, alpha, beta, 0.001) == \
        lo.adaptive_densities(sizes, t, alpha, beta, 0.001)


def test_free_network_sends_everything():
    sizes, t = [10, 2000, 77], [1e-3, 2e-3, 5e-4]
    assert L.lags_adaptive_densities(sizes, t, 0.0, 0.0, 0.01) == [1.0, 1.0, 1.0]


def test_no_compute_to_hide_behind():
    assert L.lags_adaptive_densities([100, 100], [0.0, 0.0], 1e-6, 1e-9, 0.05) == [0.05, 0.05]


def test_messages_hidden_within_one_pick():
    rng = np.random.default_rng(7)
    sizes = [int(x) for x in rng.integers(1000, 3_000_000, 30)]
    t = [float(x) for x in rng.exponential(2e-3, 30)]
    alpha, beta, rmin = 1e-5, 2e-10, 1e-3
    rho = L.lags_adaptive_densities(sizes, t, alpha, beta, rmin)
    end = sum(t)
    produced, free = 0.0, 0.0
    for l in range(len(sizes) - 1, -1, -1):
        produced += t[l]
        start = max(produced, free)
        k = lo.k_of(sizes[l], rho[l])
        free = start + alpha + 8 * beta * k
        assert rmin <= rho[l] <= 1.0
        if rho[l] > rmin:
            assert free <= end + 8 * beta + 1e-12  # within one pick's transfer


def test_rejects_bad_arguments():
    for args in (([], [], 0, 0, 0.1), ([10], [-1.0], 0, 0, 0.1), ([10], [1.0], -1, 0, 0.1),
                 ([10], [1.0], 0, 0, 0.0), ([0], [1.0], 0, 0, 0.1)):
        with pytest.raises(L.LagsError):
            L.lags_adaptive_densities(*args)
