"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand-derived fixtures, brute-force rank definitions, fp64 re-derivations of the
fp32 roundings (a double-precision result rounded to fp32 equals the correctly
rounded fp32 result for +, -, *, / because 53 >= 2*24 + 2), closed forms and
invariants.  Each check takes the oracle module so that a planted mistake can
be shown to fail at least one pin (see test_oracle_mutations.py).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

from conftest import read_golden

F32 = np.float32


def _f32(vals):
    return np.array([float(v) for v in vals], dtype=F32)


def _bits(a):
    return np.asarray(a, dtype=F32).view(np.uint32)


# ---------------------------------------------------------------- brute force
def brute_topk(acc, k):
    """i is picked iff fewer than k entries beat it: |a_j| > |a_i|, or equal
    magnitude with a lower index (ranking definition, O(d^2))."""
    mags = [abs(float(x)) for x in acc]
    picked = []
    for i, mi in enumerate(mags):
        beat = sum(1 for j, mj in enumerate(mags) if mj > mi or (mj == mi and j < i))
        if beat < k:
            picked.append(i)
    return picked


def tiny_cases(rng):
    cases = []
    for d in (1, 2, 3, 7, 8, 13, 31, 64):
        cases.append(rng.standard_normal(d).astype(F32))
        cases.append(rng.integers(-3, 4, d).astype(F32))              # heavy ties
        cases.append(np.zeros(d, dtype=F32))                           # all tie at 0
        z = np.zeros(d, dtype=F32)
        z[::2] = F32(-0.0)                                             # +-0 mix
        cases.append(z)
        den = (rng.integers(1, 5, d) * np.float32(1e-45)).astype(F32)  # denormals
        den[::3] *= F32(-1)
        cases.append(den)
        inf = rng.standard_normal(d).astype(F32)
        inf[0] = F32(np.inf)
        inf[-1] = F32(-np.inf)
        cases.append(inf)
    return cases


def check_bruteforce(lo, seed=0):
    rng = np.random.default_rng(seed)
    for acc in tiny_cases(rng):
        d = acc.size
        for k in sorted({1, max(1, d // 3), max(1, d - 1), d}):
            got = lo.select_layer(acc, k)
            exp = brute_topk(acc, k)
            assert list(got) == exp, (acc, k, got, exp)


# ---------------------------------------------------------------- fixtures
def check_hand_topk(lo):
    g = read_golden("topk_hand_example.txt")
    d = int(g["d"][0])
    rho = float(g["rho"][0])
    k = lo.k_of(d, rho)
    assert k == int(g["k"][0])
    idx, val, res = lo.sparsify_layer(0, k, [_f32(g["grad"])], [_f32(g["residual"])],
                                      float(g["lr"][0]))
    assert idx[0].tolist() == [int(x) for x in g["idx"]]
    assert np.array_equal(_bits(val[0]), _bits(_f32(g["val"])))
    assert np.array_equal(_bits(res[0]), _bits(_f32(g["residual_new"])))


def check_two_worker(lo):
    g = read_golden("two_worker_two_step.txt")
    d, P, lr, rho = int(g["d"][0]), int(g["P"][0]), float(g["lr"][0]), float(g["rho"][0])
    res = [_f32(g[f"residual{p}"]) for p in range(P)]
    w = np.zeros(d, dtype=F32)
    for s in range(2):
        grads = [_f32(g[f"s{s}_grad{p}"]) for p in range(P)]
        idx, val, res = lo.sparsify([d], [rho], grads, res, lr)
        for p in range(P):
            assert idx[p].tolist() == [int(x) for x in g[f"s{s}_idx{p}"]], (s, p)
            assert np.array_equal(_bits(val[p]), _bits(_f32(g[f"s{s}_val{p}"]))), (s, p)
            assert np.array_equal(_bits(res[p]), _bits(_f32(g[f"s{s}_res{p}"]))), (s, p)
        dense = lo.aggregate(d, idx, val)
        assert np.array_equal(_bits(dense), _bits(_f32(g[f"s{s}_dense"]))), s
        w = lo.apply_update(w, dense)
        assert np.array_equal(_bits(w), _bits(_f32(g[f"s{s}_weights"]))), s


# ---------------------------------------------------------------- fp64 re-derivation
def wide_f32(rng, n):
    """fp32 values spanning many binades, with signs, so that single vs double
    rounding and operand order visibly matter."""
    m = rng.uniform(1.0, 2.0, n)
    e = rng.integers(-40, 40, n)
    s = rng.choice([-1.0, 1.0], n)
    return (s * m * np.exp2(e)).astype(F32)


def check_error_feedback_fp64(lo, seed=1):
    rng = np.random.default_rng(seed)
    n = 20000
    r, g = wide_f32(rng, n), wide_f32(rng, n)
    for lr in (0.1, 1.0, 0.01, 3.0e-3):
        got = lo.error_feedback(r, g, lr)
        t = (np.float64(F32(lr)) * g.astype(np.float64)).astype(F32)   # exact, then round
        exp = (r.astype(np.float64) + t.astype(np.float64)).astype(F32)
        assert np.array_equal(_bits(got), _bits(exp)), lr


def check_aggregate_fp64(lo, seed=2):
    """Sum in worker order with one rounding per add, then a true division."""
    rng = np.random.default_rng(seed)
    N = 4096
    for P in (3, 5, 12):
        idx, val = [], []
        for p in range(P):
            loc = np.sort(rng.choice(N, N // 2, replace=False)).astype(np.uint32)
            idx.append(loc)
            val.append(wide_f32(rng, loc.size))
        idx, val = np.stack(idx), np.stack(val)
        got = lo.aggregate(N, idx, val)
        s = np.zeros(N, dtype=np.float64)
        for p in range(P):
            loc = idx[p].astype(np.int64)
            s[loc] = (s[loc] + val[p].astype(np.float64)).astype(F32).astype(np.float64)
        exp = (s / np.float64(P)).astype(F32)
        assert np.array_equal(_bits(got), _bits(exp)), P


def check_apply_fp64(lo, seed=3):
    rng = np.random.default_rng(seed)
    w, dns = wide_f32(rng, 5000), wide_f32(rng, 5000)
    got = lo.apply_update(w, dns)
    exp = (w.astype(np.float64) - dns.astype(np.float64)).astype(F32)
    assert np.array_equal(_bits(got), _bits(exp))


# ---------------------------------------------------------------- invariants / closed forms
def random_layers(rng, L, dmax):
    sizes = [int(x) for x in rng.integers(1, dmax, L)]
    dens = [float(x) for x in rng.choice([0.001, 0.01, 0.1, 0.3, 1.0], L)]
    return sizes, dens


def check_invariants(lo, seed=4):
    rng = np.random.default_rng(seed)
    sizes, dens = random_layers(rng, 9, 3000)
    P, lr = 3, 0.1
    N = sum(sizes)
    grads = [wide_f32(rng, N) for _ in range(P)]
    res = [wide_f32(rng, N) for _ in range(P)]
    idx, val, new = lo.sparsify(sizes, dens, grads, res, lr)
    off = koff = 0
    for d, rho in zip(sizes, dens):
        k = max(1, min(d, math.ceil(rho * d)))
        for p in range(P):
            acc = (res[p][off:off + d].astype(np.float64)
                   + (np.float64(F32(lr)) * grads[p][off:off + d]).astype(F32)).astype(F32)
            li = idx[p, koff:koff + k].astype(np.int64)
            assert np.all(np.diff(li) > 0) and li.min() >= off and li.max() < off + d
            loc = li - off
            scat = np.zeros(d, dtype=F32)
            scat[loc] = val[p, koff:koff + k]
            rn = new[p][off:off + d]
            # one of the two terms is exactly zero, so the sum is exact
            assert np.array_equal(_bits(scat + rn), _bits(acc)) or \
                np.array_equal(scat + rn, acc)
            assert np.all((scat == 0) | (rn == 0))
            mask = np.zeros(d, bool)
            mask[loc] = True
            if k < d:
                assert np.abs(acc[mask]).min() >= np.abs(acc[~mask]).max()
        off += d
        koff += k


def check_dense_rho1(lo, seed=5):
    """rho = 1: every entry is sent, residual becomes 0 and the update is the
    plain S-SGD mean of acc over workers (integer data: sums are exact)."""
    rng = np.random.default_rng(seed)
    sizes = [17, 5, 40]
    P, lr = 6, 0.5
    N = sum(sizes)
    grads = [rng.integers(-40, 40, N).astype(F32) for _ in range(P)]
    res = [rng.integers(-40, 40, N).astype(F32) for _ in range(P)]
    idx, val, new = lo.sparsify(sizes, [1.0] * 3, grads, res, lr)
    for p in range(P):
        assert np.all(new[p] == 0) and not np.signbit(new[p]).any()
        assert idx[p].tolist() == list(range(N))
    dense = lo.aggregate(N, idx, val)
    exact = sum(res[p].astype(np.float64) + 0.5 * grads[p].astype(np.float64) for p in range(P))
    assert np.array_equal(dense, (exact / P).astype(F32))


def check_single_worker(lo, seed=6):
    """P = 1: the update is the scatter of the picks."""
    rng = np.random.default_rng(seed)
    sizes, dens = random_layers(rng, 5, 500)
    N = sum(sizes)
    g, r = [wide_f32(rng, N)], [wide_f32(rng, N)]
    idx, val, new = lo.sparsify(sizes, dens, g, r, 0.1)
    dense = lo.aggregate(N, idx, val)
    exp = np.zeros(N, dtype=F32)
    exp[idx[0].astype(np.int64)] = val[0]
    assert np.array_equal(_bits(dense), _bits(exp))


def check_k_rule(lo, workloads):
    """k_l against the exact decimal ceiling of rho*d for every layer of every
    workload (the density is written in decimal in the workload definition)."""
    for w in workloads:
        for d, rho in zip(w.sizes, w.densities):
            exact = math.ceil(Fraction(repr(rho)) * d)
            assert lo.k_of(d, rho) == max(1, min(d, exact)), (w.name, d, rho)


def check_merge_hand(lo):
    """Merged-message planner on the hand-worked four-layer fixture (R9)."""
    from conftest import read_golden
    g = read_golden("merge_four_layers.txt")
    b = [int(x) for x in g["bytes"]]
    t = [float(x) for x in g["backward"]]
    a, beta = float(g["alpha"][0]), float(g["beta"][0])
    f = [int(x) for x in g["first"]] + [len(b)]
    want = [(f[i], f[i + 1]) for i in range(len(f) - 1)]
    assert lo.message_schedule_end([(l, l + 1) for l in range(len(b))], b, t, a, beta) == \
        float(g["singles_end"][0])
    assert lo.merge_layers(b, t, a, beta) == (want, float(g["end"][0]))


def check_merge_bruteforce(lo, seed=7):
    """The planner's cut ends no later than any cut of a small model."""
    rng = np.random.default_rng(seed)
    for _ in range(20):
        n = int(rng.integers(2, 8))
        b = [int(x) for x in rng.integers(0, 1_000_000, n)]
        t = [float(x) for x in rng.exponential(1e-3, n)]
        alpha, beta = float(rng.uniform(0, 1e-3)), float(rng.uniform(0, 1e-9))
        buckets, end = lo.merge_layers(b, t, alpha, beta)
        assert end == lo.message_schedule_end(buckets, b, t, alpha, beta)
        for mask in range(1 << (n - 1)):
            f = [0] + [i + 1 for i in range(n - 1) if mask >> i & 1] + [n]
            cut = [(f[i], f[i + 1]) for i in range(len(f) - 1)]
            assert end <= lo.message_schedule_end(cut, b, t, alpha, beta) * (1 + 1e-12)
