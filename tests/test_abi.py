"""The C ABI on the CPU: the library loads, exports every entry point that
include/lags.h declares, and plan creation validates and lays out correctly.
No compute call is made here (no GPU)."""
import ctypes
import os
import re

import pytest

import layer_wise_top_b200 as L
import oracle.lags_oracle as lo
from conftest import ROOT
from synth.configs import WORKLOADS


def declared():
    with open(os.path.join(ROOT, "include", "lags.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"LAGS_API\s+[\w\s\*]+?\b(lags_\w+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared()
    assert len(names) == 23, names
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(L.EXPORTED) == names


def test_error_strings():
    for code in range(10):
        assert L.lags_error_string(code) not in ("", "unknown status")
    assert len({L.lags_error_string(c) for c in range(10)}) == 10
    assert L.lags_error_string(99) == "unknown status"


def test_status_codes_match_header():
    with open(os.path.join(ROOT, "include", "lags.h")) as f:
        text = f.read()
    for name in ("LAGS_ERR_TIMEOUT", "LAGS_ERR_INTERNAL", "LAGS_ERR_WRONG_DEVICE",
                 "LAGS_ERR_BAD_PICKS", "LAGS_ERR_WORKSPACE"):
        m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
        assert m and int(m.group(1)) == getattr(L, name), name
    for name in ("LAGS_FLAG_TIMEOUT", "LAGS_FLAG_INTERNAL", "LAGS_FLAG_BAD_PICKS"):
        m = re.search(rf"#define {name} (0x[0-9a-fA-F]+)u", text)
        assert m and int(m.group(1), 16) == getattr(L, name), name
    m = re.search(r"#define LAGS_STAGE_WAIT_POLLS (\d+)u", text)
    assert m and int(m.group(1)) == L.LAGS_STAGE_WAIT_POLLS


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_aggregate_only_workspace_is_a_smaller_prefix(name):
    # the job-wide plan of a data-parallel rank only aggregates: its workspace
    # leaves out the candidate slots, the bulk of the full workspace
    w = WORKLOADS[name]
    h = L.lags_plan_create(w.sizes, w.densities, w.P)
    try:
        full = L.lags_plan_info(h)[2]
        agg = L.lags_plan_aggregate_workspace_bytes(h)
        assert 0 < agg < full and agg % 256 == 0
        # tiles (16 B each) and the per-(worker, tile) first picks (4 B) fit in it
        tiles = sum((o + d - 1) // 8192 - o // 8192 + 1
                    for o, d in zip(w.offsets, w.sizes))
        assert agg >= 16 * tiles + 4 * w.P * tiles
        if name != "resnet20":
            assert agg < full / 4
    finally:
        L.lags_plan_destroy(h)


def test_index_wait_limit_knob_validates():
    with pytest.raises(L.LagsError):
        L.lags_plan_set_index_wait_limit(None, 0)
    h = L.lags_plan_create([100, 7], [0.1, 1.0], 2)
    try:
        L.lags_plan_set_index_wait_limit(h, 0)
        L.lags_plan_set_index_wait_limit(h, L.LAGS_STAGE_WAIT_POLLS)
    finally:
        L.lags_plan_destroy(h)


def test_stage_wait_limit_knob_validates():
    with pytest.raises(L.LagsError) as e:
        L.lags_plan_set_stage_wait_limit(None, 0)
    assert e.value.status == L.LAGS_ERR_INVALID_ARG
    h = L.lags_plan_create([100], [0.1], 2)
    try:
        L.lags_plan_set_stage_wait_limit(h, 0)
        L.lags_plan_set_stage_wait_limit(h, L.LAGS_STAGE_WAIT_POLLS)
    finally:
        L.lags_plan_destroy(h)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_plan_matches_oracle_layout(name):
    w = WORKLOADS[name]
    h = L.lags_plan_create(w.sizes, w.densities, w.P)
    try:
        offs, ks, koffs, N, K = lo.layer_plan(w.sizes, w.densities)
        assert L.lags_plan_info(h)[:2] == (N, K)
        for l in range(w.L):
            assert L.lags_plan_layer(h, l) == (offs[l], ks[l], koffs[l])
    finally:
        L.lags_plan_destroy(h)


@pytest.mark.parametrize("sizes,dens,P", [
    ([], [], 1),
    ([10], [0.5], 0),
    ([10], [0.5], 257),
    ([0], [0.5], 1),
    ([-3], [0.5], 1),
    ([10], [0.0], 1),
    ([10], [1.5], 1),
    ([10], [float("nan")], 1),
    ([1 << 31, 1 << 31], [0.1, 0.1], 1),   # N >= 2^32
])
def test_plan_rejects(sizes, dens, P):
    with pytest.raises(L.LagsError) as e:
        L.lags_plan_create(sizes, dens, P)
    assert e.value.status == L.LAGS_ERR_INVALID_ARG


def test_calls_reject_null_and_unbound_plan():
    h = L.lags_plan_create([100], [0.1], 2)
    try:
        with pytest.raises(L.LagsError) as e:
            L.lags_sparsify(h, [0, 0], [0, 0], 0.1, 0, 0)
        assert e.value.status == L.LAGS_ERR_INVALID_ARG
        with pytest.raises(L.LagsError) as e:
            L.lags_sparsify(h, [16, 32], [48, 64], 0.1, 16, 32)
        assert e.value.status == L.LAGS_ERR_WORKSPACE   # no workspace bound yet
        with pytest.raises(L.LagsError) as e:
            L.lags_aggregate(h, 16, 16, 16)
        assert e.value.status == L.LAGS_ERR_WORKSPACE
        with pytest.raises(L.LagsError) as e:
            L.lags_apply(h, 8, 16)
        assert e.value.status == L.LAGS_ERR_ALIGNMENT
        with pytest.raises(L.LagsError) as e:
            L.lags_plan_set_workspace(h, 128, 1 << 20)
        assert e.value.status == L.LAGS_ERR_ALIGNMENT
        with pytest.raises(L.LagsError) as e:
            L.lags_plan_set_workspace(h, 256, 16)
        assert e.value.status == L.LAGS_ERR_WORKSPACE
    finally:
        L.lags_plan_destroy(h)


def test_k_rule_uses_double_density():
    h = L.lags_plan_create([18_000_000, 2_048_000], [0.001, 0.001], 1)
    try:
        assert L.lags_plan_layer(h, 0)[1] == 18000
        assert L.lags_plan_layer(h, 1)[1] == 2048
    finally:
        L.lags_plan_destroy(h)


def test_plan_size_limit():
    # N may reach LAGS_MAX_ELEMENTS (2^32 - 65536) and not one element more
    top = L.LAGS_MAX_ELEMENTS
    h = L.lags_plan_create([top - 100_003 - 7, 100_003, 7], [1e-7, 0.001, 0.5], 1)
    N, K, _ = L.lags_plan_info(h)
    assert N == top and L.lags_plan_layer(h, 2)[0] == top - 7
    L.lags_plan_destroy(h)
    with pytest.raises(L.LagsError):
        L.lags_plan_create([top - 6, 7], [0.01, 0.5], 1)
    # a range plan past the limit is rejected too, even if its own layers are small
    with pytest.raises(L.LagsError):
        L.lags_plan_create_range([top, 5], [0.01, 0.5], 1, 1, 2)


def test_kernel_launch_counts():
    # a dense-only plan runs just the fused pass; sparse plans add the
    # estimate and one select launch per cluster size in use
    h = L.lags_plan_create([100, 7], [1.0, 1.0], 2)
    try:
        assert L.lags_plan_kernel_launches(h) == (1, 3, 1)
    finally:
        L.lags_plan_destroy(h)
    w = WORKLOADS["gpt_1_3b"]  # one-CTA, 4-CTA and 16-CTA selects
    h = L.lags_plan_create(w.sizes, w.densities, w.P)
    try:
        assert L.lags_plan_kernel_launches(h) == (5, 3, 1)
    finally:
        L.lags_plan_destroy(h)
