"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle.lags_oracle as lo
import oracle_pins as pins
from synth.configs import WORKLOADS


def test_bruteforce_rank_definition():
    pins.check_bruteforce(lo)


def test_hand_example():
    pins.check_hand_topk(lo)


def test_two_worker_two_step():
    pins.check_two_worker(lo)


def test_error_feedback_two_roundings():
    pins.check_error_feedback_fp64(lo)


def test_aggregate_order_and_division():
    pins.check_aggregate_fp64(lo)


def test_apply():
    pins.check_apply_fp64(lo)


def test_invariants():
    pins.check_invariants(lo)


def test_rho_one_is_dense_ssgd():
    pins.check_dense_rho1(lo)


def test_single_worker_scatter():
    pins.check_single_worker(lo)


def test_k_rule_all_workloads():
    pins.check_k_rule(lo, WORKLOADS.values())


def test_k_rule_needs_double_density():
    # A float32 density would change k on the LSTM layers (0.001f > 0.001).
    d = 18_000_000
    assert lo.k_of(d, 0.001) == 18000
    assert lo.k_of(d, float(np.float32(0.001))) == 18001


def test_k_rule_edges():
    assert lo.k_of(10, 0.001) == 1
    assert lo.k_of(5, 1.0) == 5
    for bad in (0.0, -0.1, 1.5):
        with pytest.raises(ValueError):
            lo.k_of(10, bad)


def test_nan_rejected():
    with pytest.raises(ValueError):
        lo.select_layer(np.array([1.0, np.nan], dtype=np.float32), 1)


def test_run_workload_carries_residual():
    # Constant gradient 1 on a layer of 4 with k = 1 and lr = 1: every entry
    # grows by 1 per step until it is picked; the pick cycles by index.
    hist = lo.run_workload([4], [0.25], 1, 1.0, 5,
                           lambda p, s: np.ones(4, dtype=np.float32))
    picks = [int(h[0][0, 0]) for h in hist]
    vals = [float(h[1][0, 0]) for h in hist]
    assert picks == [0, 1, 2, 3, 0]
    assert vals == [1.0, 2.0, 3.0, 4.0, 4.0]


def test_merge_hand_example():
    pins.check_merge_hand(lo)


def test_merge_against_every_cut():
    pins.check_merge_bruteforce(lo)


def test_dense_sgd_integer_closed_form():
    # integer gradients, lr = 1: every partial sum is exact, so P * dense is
    # the integer sum and dense is its correctly rounded quotient
    rng = np.random.default_rng(12)
    P, N = 5, 257
    g = [rng.integers(-1000, 1000, N).astype(np.float32) for _ in range(P)]
    tot = np.sum(np.stack(g).astype(np.int64), axis=0)
    got = lo.dense_sgd_update(g, 1.0)
    assert np.array_equal(got, (tot.astype(np.float64) / P).astype(np.float32))


def test_dense_sgd_is_lags_at_density_one():
    rng = np.random.default_rng(13)
    sizes = [7, 300, 33]
    g = [rng.standard_normal(sum(sizes)).astype(np.float32) for _ in range(3)]
    hist = lo.run_workload(sizes, [1.0] * 3, 3, 0.25, 1, lambda p, s: g[p])
    assert np.array_equal(lo.dense_sgd_update(g, 0.25).view(np.uint32), hist[0][3].view(np.uint32))
