"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin,
which shows the pins constrain every step of the definition."""
import math

import numpy as np
import pytest

import oracle.lags_oracle as lo
import oracle_pins as pins
from synth.configs import WORKLOADS

F32 = np.float32


def _ef_fma(residual, grad, lr):
    exact = residual.astype(np.float64) + np.float64(F32(lr)) * grad.astype(np.float64)
    return exact.astype(F32)


def _ef_grad_only(residual, grad, lr):
    return np.multiply(F32(lr), grad, dtype=F32)


def _order_high_index(acc):
    neg = -np.abs(acc).astype(np.float64)
    return np.lexsort((-np.arange(acc.size), neg))


def _order_signed(acc):
    return np.lexsort((np.arange(acc.size), -acc.astype(np.float64)))


def _k_floor(d, rho):
    return int(min(d, max(1, math.floor(rho * d))))


def _k_f32(d, rho):
    return int(min(d, max(1, math.ceil(float(F32(rho)) * float(F32(d))))))


def _agg_reverse(off, d, idx, val):
    P = idx.shape[0]
    dense = np.zeros(d, dtype=F32)
    for p in reversed(range(P)):
        loc = idx[p].astype(np.int64) - off
        dense[loc] = np.add(dense[loc], val[p], dtype=F32)
    return np.divide(dense, F32(P), dtype=F32)


def _agg_reciprocal(off, d, idx, val):
    P = idx.shape[0]
    dense = np.zeros(d, dtype=F32)
    for p in range(P):
        loc = idx[p].astype(np.int64) - off
        dense[loc] = np.add(dense[loc], val[p], dtype=F32)
    return np.multiply(dense, F32(1.0) / F32(P), dtype=F32)


def _agg_fp64_sum(off, d, idx, val):
    P = idx.shape[0]
    dense = np.zeros(d, dtype=np.float64)
    for p in range(P):
        loc = idx[p].astype(np.int64) - off
        dense[loc] += val[p].astype(np.float64)
    return (dense / P).astype(F32)


def _apply_plus(weights, dense):
    return np.add(weights, dense, dtype=F32)


def _sparsify_layer_keep_residual(off, k, grads, residuals, lr):
    P = len(grads)
    idx = np.empty((P, k), dtype=np.uint32)
    val = np.empty((P, k), dtype=F32)
    new = []
    for p in range(P):
        acc = lo.error_feedback(residuals[p], grads[p], lr)
        loc = lo.select_layer(acc, k)
        idx[p] = (loc + off).astype(np.uint32)
        val[p] = acc[loc]
        new.append(acc.copy())          # forgot to zero the picked entries
    return idx, val, new


def _sparsify_layer_emit_grad(off, k, grads, residuals, lr):
    P = len(grads)
    idx = np.empty((P, k), dtype=np.uint32)
    val = np.empty((P, k), dtype=F32)
    new = []
    for p in range(P):
        acc = lo.error_feedback(residuals[p], grads[p], lr)
        loc = lo.select_layer(acc, k)
        idx[p] = (loc + off).astype(np.uint32)
        val[p] = grads[p][loc]          # emits the raw gradient
        r = acc.copy()
        r[loc] = 0
        new.append(r)
    return idx, val, new


def _merge_variant(start_when_first_produced=False, no_start_up=False):
    def merge(message_bytes, backward_seconds, alpha, beta):
        L = len(message_bytes)
        ready = [0.0] * (L + 1)
        for l in range(L - 1, -1, -1):
            ready[l] = ready[l + 1] + float(backward_seconds[l])
        best, cut = [0.0] * (L + 1), [L] * (L + 1)
        for i in range(L - 1, -1, -1):
            nbytes = 0.0
            for j in range(i + 1, L + 1):
                nbytes += float(message_bytes[j - 1])
                start = ready[j - 1] if start_when_first_produced else ready[i]
                end = max(start, best[j]) + (0.0 if no_start_up else alpha) + beta * nbytes
                if j == i + 1 or end <= best[i]:
                    best[i], cut[i] = end, j
        buckets, i = [], 0
        while i < L:
            buckets.append((i, cut[i]))
            i = cut[i]
        return buckets, best[0]
    return merge


def _schedule_forward_order(buckets, message_bytes, backward_seconds, alpha, beta):
    L = len(message_bytes)
    ready = [0.0] * (L + 1)
    for l in range(L - 1, -1, -1):
        ready[l] = ready[l + 1] + float(backward_seconds[l])
    link_free = 0.0
    for first, end in sorted(buckets):  # sends the first layers first
        nbytes = sum(float(message_bytes[l]) for l in range(first, end))
        link_free = max(ready[first], link_free) + alpha + beta * nbytes
    return link_free


MUTANTS = {
    "merge_starts_too_early": ("merge_layers", _merge_variant(start_when_first_produced=True)),
    "merge_without_start_up": ("merge_layers", _merge_variant(no_start_up=True)),
    "schedule_forward_order": ("message_schedule_end", _schedule_forward_order),
    "fma_error_feedback": ("error_feedback", _ef_fma),
    "no_residual_term": ("error_feedback", _ef_grad_only),
    "tie_to_higher_index": ("magnitude_order", _order_high_index),
    "signed_order": ("magnitude_order", _order_signed),
    "k_floor": ("k_of", _k_floor),
    "k_in_float32": ("k_of", _k_f32),
    "aggregate_reverse_order": ("aggregate_layer", _agg_reverse),
    "aggregate_reciprocal": ("aggregate_layer", _agg_reciprocal),
    "aggregate_fp64": ("aggregate_layer", _agg_fp64_sum),
    "apply_sign": ("apply_update", _apply_plus),
    "residual_not_zeroed": ("sparsify_layer", _sparsify_layer_keep_residual),
    "emit_raw_grad": ("sparsify_layer", _sparsify_layer_emit_grad),
}

ALL_PINS = [
    pins.check_bruteforce, pins.check_hand_topk, pins.check_two_worker,
    pins.check_error_feedback_fp64, pins.check_aggregate_fp64, pins.check_apply_fp64,
    pins.check_invariants, pins.check_dense_rho1, pins.check_single_worker,
    lambda m: pins.check_k_rule(m, WORKLOADS.values()),
    pins.check_merge_hand, pins.check_merge_bruteforce,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(lo, attr, fn)
    failed = 0
    for pin in ALL_PINS:
        try:
            pin(lo)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed > 0, f"planted mistake {name} passed every pin"
