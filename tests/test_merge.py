"""Merged-message planner (reading R9): the C planner and the oracle's
dynamic program against a hand-worked fixture, brute force over every cut of
small models, and the special cases the timing model fixes."""

import numpy as np
import pytest

import layer_wise_top_b200 as L
import oracle.lags_oracle as lo
from conftest import read_golden


def _golden():
    g = read_golden("merge_four_layers.txt")
    return ([int(x) for x in g["bytes"]], [float(x) for x in g["backward"]],
            float(g["alpha"][0]), float(g["beta"][0]), g)


def _buckets(first, n):
    f = [int(x) for x in first] + [n]
    return [(f[i], f[i + 1]) for i in range(len(first))]


def test_schedule_end_hand_example():
    b, t, a, beta, g = _golden()
    n = len(b)
    assert lo.message_schedule_end([(l, l + 1) for l in range(n)], b, t, a, beta) == \
        float(g["singles_end"][0])
    assert lo.message_schedule_end([(0, n)], b, t, a, beta) == float(g["all_end"][0])
    assert lo.message_schedule_end(_buckets(g["first"], n), b, t, a, beta) == float(g["end"][0])


def test_merge_hand_example():
    b, t, a, beta, g = _golden()
    want = (_buckets(g["first"], len(b)), float(g["end"][0]))
    assert lo.merge_layers(b, t, a, beta) == want
    assert L.lags_merge_layers(b, t, a, beta) == want


def _all_cuts(n):
    for mask in range(1 << (n - 1)):
        first = [0] + [i + 1 for i in range(n - 1) if mask >> i & 1]
        yield _buckets(first, n)


@pytest.mark.parametrize("seed", range(40))
def test_optimal_against_every_cut(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 10))
    b = [int(x) for x in rng.integers(0, 4_000_000, n)]
    t = [float(x) for x in rng.exponential(1e-3, n)]
    alpha = float(rng.choice([0.0, 1e-6, 5e-5, 1e-3]))
    beta = float(rng.choice([0.0, 1e-10, 1e-9, 1e-8]))
    best = min(lo.message_schedule_end(c, b, t, alpha, beta) for c in _all_cuts(n))
    for buckets, end in (lo.merge_layers(b, t, alpha, beta), L.lags_merge_layers(b, t, alpha, beta)):
        assert end == lo.message_schedule_end(buckets, b, t, alpha, beta)
        assert end == pytest.approx(best, rel=1e-12, abs=0.0)
        assert buckets[0][0] == 0 and buckets[-1][1] == n
        assert all(x[1] == y[0] for x, y in zip(buckets, buckets[1:]))


@pytest.mark.parametrize("seed", range(5))
def test_library_equals_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 200))
    b = [8 * int(x) for x in rng.integers(1, 200_000, n)]
    t = [float(x) for x in rng.exponential(2e-4, n)]
    alpha, beta = float(rng.uniform(0, 5e-5)), float(rng.uniform(1e-12, 1e-9))
    assert L.lags_merge_layers(b, t, alpha, beta) == lo.merge_layers(b, t, alpha, beta)


def test_free_start_up_sends_every_layer_alone():
    # alpha = 0: splitting a bucket never delays its last message
    rng = np.random.default_rng(3)
    b = [int(x) for x in rng.integers(1, 10_000, 12)]
    t = [float(x) for x in rng.exponential(1e-3, 12)]
    buckets, end = L.lags_merge_layers(b, t, 0.0, 1e-9)
    assert end == pytest.approx(
        lo.message_schedule_end([(l, l + 1) for l in range(12)], b, t, 0.0, 1e-9), rel=1e-12)


def test_everything_ready_at_once_is_one_message():
    # no backward time: all layers exist at t = 0, so one message (one alpha) wins
    b = [100, 5, 70000, 3]
    assert L.lags_merge_layers(b, [0.0] * 4, 1e-5, 1e-9) == ([(0, 4)], 1e-5 + 1e-9 * sum(b))


def test_rejects_bad_arguments():
    with pytest.raises(L.LagsError):
        L.lags_merge_layers([], [], 0.0, 0.0)
    with pytest.raises(L.LagsError):
        L.lags_merge_layers([1, -1], [0.0, 0.0], 0.0, 0.0)
    with pytest.raises(L.LagsError):
        L.lags_merge_layers([1], [0.0], -1.0, 0.0)


def test_check_buckets_accepts_only_ordered_partitions():
    from layer_wise_top_b200.dist import check_buckets
    check_buckets([(0, 2), (2, 3), (3, 7)], 7)
    check_buckets(L.lags_merge_layers([8] * 5, [1e-3] * 5, 1e-5, 1e-9)[0], 5)
    for bad in ([(0, 2), (3, 7)], [(0, 2), (2, 2), (2, 7)], [(1, 7)], [(0, 6)],
                [(0, 4), (2, 7)]):
        with pytest.raises(ValueError):
            check_buckets(bad, 7)
