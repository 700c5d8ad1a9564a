"""Plain, slow, obviously correct CPU definition of one LAGS-SGD sparsification
step: error feedback, per-layer top-k by magnitude, residual update,
deterministic sparse aggregation and the weight update.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py`` (its CPU-baseline and reference legs), never by the product
library.  It shares no code with the CUDA path.

Sources.  "Layer-wise Adaptive Gradient Sparsification for Distributed Deep
Learning with Convergence Guarantees" (nubint.ai review), section "proposed
method": every worker picks the top-k gradients of each layer independently by
magnitude; an error-compensation mechanism keeps what was not sent; LAGS is
combined with synchronous SGD (abstract: "sparsified S-SGD").  The pages print
no formula, so the exact arithmetic below is the plainest reading, listed here
and in the design notes:

  R1  acc = fl32(residual + fl32(lr * grad)): two fp32 roundings, no FMA.  The
      buffers are fp32, so the method's arithmetic is fp32 with one rounding per
      written operation (the float32 ufuncs below round once each).
  R2  k_l = min(d_l, max(1, ceil(fl64(rho_l * d_l)))) with rho_l a double.
  R3  "largest |acc|" with equal magnitudes broken by the lower index; +0 and -0
      tie; +-inf are the largest magnitudes.  NaN is not a valid input.
  R4  the emitted value is acc itself, and a picked entry's residual becomes
      +0.0 while every other entry keeps acc (error compensation).
  R5  picks are listed per layer in ascending index order, layers in order;
      indices are global positions in the worker's flattened buffer (uint32).
  R6  dense[j] = fl32( (((+0 + v_0j) + v_1j) + ... + v_(P-1)j) / P ), workers
      in order 0..P-1, a worker that did not pick j contributing nothing, and
      a true IEEE division by P.
  R7  weights <- fl32(weights - dense)  (plain S-SGD, lr already inside acc).
  R8  adaptive densities ("proposed method": each layer's ratio follows its
      communication-to-computation ratio so that communication hides behind
      computation): layers come out of backprop in reverse order; layer l's
      message starts when its gradient exists (sum of the backward times of
      layers >= l) and the previous message has ended, takes alpha + 8 beta k
      seconds, and gets the largest density whose message ends by the end of
      the backward pass (rho_min if none does).
  R9  merged messages ("MG-WFBP: Efficient Data Communication for Distributed
      Synchronous SGD Algorithms" review, "proposed method": merge small
      per-layer messages to save start-up costs, choosing the merge that
      minimises the iteration time, by dynamic programming in O(L^2), once
      before training): the layers are cut into buckets of consecutive layers,
      one message per bucket; with the timing of R8 (a message of B bytes
      takes alpha + beta B and starts once its bucket's first layer, the last
      one backprop produces, exists and the previous message has ended) the
      cut minimises the end of the last message.  Equal end times go to the
      longer bucket, deciding from the last layers towards the first.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

F32 = np.float32


def k_of(d: int, rho: float) -> int:
    """Per-layer pick count (reading R2)."""
    if d <= 0:
        raise ValueError("layer size must be positive")
    if not (0.0 < rho <= 1.0):
        raise ValueError("density must lie in (0, 1]")
    k = math.ceil(float(rho) * float(d))
    return int(min(d, max(1, k)))


def layer_plan(sizes: Sequence[int], densities: Sequence[float]):
    """Offsets of each layer in the flattened buffer, pick counts k_l and the
    offsets koff_l of each layer's picks in a worker's pick list."""
    offs, ks, koffs = [], [], []
    off = koff = 0
    for d, rho in zip(sizes, densities):
        k = k_of(int(d), float(rho))
        offs.append(off)
        ks.append(k)
        koffs.append(koff)
        off += int(d)
        koff += k
    return offs, ks, koffs, off, koff


def error_feedback(residual: np.ndarray, grad: np.ndarray, lr: float) -> np.ndarray:
    """acc = residual + lr * grad, one fp32 rounding per operation (R1)."""
    assert residual.dtype == F32 and grad.dtype == F32
    t = np.multiply(F32(lr), grad, dtype=F32)
    return np.add(residual, t, dtype=F32)


def magnitude_order(acc: np.ndarray) -> np.ndarray:
    """Positions sorted by |acc| descending, lower index first among equals
    (R3).  np.abs maps -0 and +0 to the same value, so they tie."""
    if np.isnan(acc).any():
        raise ValueError("NaN is not a valid accumulated gradient")
    neg_mag = -np.abs(acc).astype(np.float64)
    pos = np.arange(acc.size, dtype=np.int64)
    return np.lexsort((pos, neg_mag))


def select_layer(acc: np.ndarray, k: int) -> np.ndarray:
    """Local positions of the k largest-|acc| entries, ascending (R3, R5)."""
    picked = magnitude_order(acc)[:k]
    return np.sort(picked)


def sparsify_layer(off: int, k: int, grads: Sequence[np.ndarray],
                   residuals: Sequence[np.ndarray], lr: float):
    """One layer for every worker.  grads[p], residuals[p]: that layer's slice.

    Returns (idx [P, k] uint32 global, val [P, k] float32, new residual list).
    """
    P = len(grads)
    idx = np.empty((P, k), dtype=np.uint32)
    val = np.empty((P, k), dtype=F32)
    new_res = []
    for p in range(P):
        acc = error_feedback(residuals[p], grads[p], lr)
        loc = select_layer(acc, k)
        idx[p] = (loc + off).astype(np.uint32)
        val[p] = acc[loc]
        r = acc.copy()
        r[loc] = F32(0.0)
        new_res.append(r)
    return idx, val, new_res


def sparsify(sizes: Sequence[int], densities: Sequence[float],
             grads: Sequence[np.ndarray], residuals: Sequence[np.ndarray], lr: float):
    """All layers, all workers.  grads/residuals: P flattened [N] buffers.

    Returns (out_idx [P, K] uint32, out_val [P, K] float32, residuals_new)."""
    offs, ks, koffs, N, K = layer_plan(sizes, densities)
    P = len(grads)
    out_idx = np.empty((P, K), dtype=np.uint32)
    out_val = np.empty((P, K), dtype=F32)
    res_new = [np.empty(N, dtype=F32) for _ in range(P)]
    for l, d in enumerate(sizes):
        o, k, ko = offs[l], ks[l], koffs[l]
        gi = [g[o:o + d] for g in grads]
        ri = [r[o:o + d] for r in residuals]
        idx, val, nr = sparsify_layer(o, k, gi, ri, lr)
        out_idx[:, ko:ko + k] = idx
        out_val[:, ko:ko + k] = val
        for p in range(P):
            res_new[p][o:o + d] = nr[p]
    return out_idx, out_val, res_new


def aggregate_layer(off: int, d: int, idx: np.ndarray, val: np.ndarray) -> np.ndarray:
    """Dense averaged update of one layer from P workers' picks (R6)."""
    P = idx.shape[0]
    dense = np.zeros(d, dtype=F32)
    for p in range(P):
        loc = idx[p].astype(np.int64) - off
        assert np.unique(loc).size == loc.size
        dense[loc] = np.add(dense[loc], val[p], dtype=F32)
    return np.divide(dense, F32(P), dtype=F32)


def aggregate(N: int, out_idx: np.ndarray, out_val: np.ndarray) -> np.ndarray:
    """Dense averaged update [N] from the [P, K] pick lists (R6)."""
    return aggregate_layer(0, N, out_idx, out_val)


def apply_update(weights: np.ndarray, dense: np.ndarray) -> np.ndarray:
    """weights - dense, one fp32 rounding (R7)."""
    return np.subtract(weights, dense, dtype=F32)


def adaptive_densities(sizes: Sequence[int], backward_seconds: Sequence[float], alpha: float,
                       beta: float, rho_min: float) -> List[float]:
    """Per-layer densities by reading R8, in the order of operations written
    there (double precision)."""
    end = 0.0
    for t in backward_seconds:
        end += float(t)
    out = [0.0] * len(sizes)
    produced, link_free = 0.0, 0.0
    for l in range(len(sizes) - 1, -1, -1):
        produced += float(backward_seconds[l])
        start = max(produced, link_free)
        d = float(sizes[l])
        budget = end - start - alpha
        rho = rho_min
        if budget >= 0.0:
            kmax = math.floor(budget / (8.0 * beta)) if beta > 0.0 else d
            rho = min(1.0, max(rho_min, kmax / d))
        out[l] = rho
        link_free = start + alpha + beta * 8.0 * k_of(int(sizes[l]), rho)
    return out


def dense_sgd_update(grads: Sequence[np.ndarray], lr: float) -> np.ndarray:
    """Dense S-SGD update, the baseline of the LAGS review's comparisons
    ("main findings": LAGS-SGD against dense S-SGD, where every worker sends
    its whole gradient): every worker sends fl32(lr g) at every position (R1
    with a zero residual), aggregated in worker order as in R6."""
    P, N = len(grads), grads[0].size
    vals = np.stack([error_feedback(np.zeros(N, dtype=F32), g, lr) for g in grads])
    idx = np.tile(np.arange(N, dtype=np.uint32), (P, 1))
    return aggregate_layer(0, N, idx, vals)


def message_schedule_end(buckets: Sequence[Tuple[int, int]], message_bytes: Sequence[int],
                         backward_seconds: Sequence[float], alpha: float,
                         beta: float) -> float:
    """End of the last message when the layers are sent as `buckets` (reading
    R9's timing): buckets go out from the last layers to the first."""
    L = len(message_bytes)
    ready = [0.0] * (L + 1)  # ready[l]: layers L-1 .. l have been produced
    for l in range(L - 1, -1, -1):
        ready[l] = ready[l + 1] + float(backward_seconds[l])
    link_free = 0.0
    for first, end in sorted(buckets, reverse=True):
        nbytes = 0.0
        for l in range(first, end):
            nbytes += float(message_bytes[l])
        link_free = max(ready[first], link_free) + alpha + beta * nbytes
    return link_free


def merge_layers(message_bytes: Sequence[int], backward_seconds: Sequence[float], alpha: float,
                 beta: float) -> Tuple[List[Tuple[int, int]], float]:
    """Bucket cut of reading R9 by dynamic programming over suffixes: the best
    cut of layers [i, L) is a first bucket [i, j) after a best cut of [j, L),
    because a bucket's end only grows with the end of the messages before it.
    Returns the buckets in forward order and the end of the last message."""
    L = len(message_bytes)
    ready = [0.0] * (L + 1)
    for l in range(L - 1, -1, -1):
        ready[l] = ready[l + 1] + float(backward_seconds[l])
    best = [0.0] * (L + 1)  # best[L]: nothing to send
    cut = [L] * (L + 1)
    for i in range(L - 1, -1, -1):
        nbytes = 0.0
        for j in range(i + 1, L + 1):
            nbytes += float(message_bytes[j - 1])
            end = max(ready[i], best[j]) + alpha + beta * nbytes
            if j == i + 1 or end <= best[i]:  # ties: the longer bucket
                best[i], cut[i] = end, j
    buckets, i = [], 0
    while i < L:
        buckets.append((i, cut[i]))
        i = cut[i]
    return buckets, best[0]


def run_workload(sizes: Sequence[int], densities: Sequence[float], P: int, lr: float,
                 steps: int, grad_fn) -> List[Tuple[np.ndarray, ...]]:
    """Run `steps` steps from zero residuals and zero weights.

    grad_fn(p, s) -> float32 [N].  Returns per step
    (out_idx, out_val, residuals (list), dense, weights) after that step."""
    N = int(sum(sizes))
    residuals = [np.zeros(N, dtype=F32) for _ in range(P)]
    weights = np.zeros(N, dtype=F32)
    history = []
    for s in range(steps):
        grads = [grad_fn(p, s) for p in range(P)]
        out_idx, out_val, residuals = sparsify(sizes, densities, grads, residuals, lr)
        dense = aggregate(N, out_idx, out_val)
        weights = apply_update(weights, dense)
        history.append((out_idx, out_val, [r.copy() for r in residuals], dense, weights.copy()))
    return history
