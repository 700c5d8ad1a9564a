"""bench.py's host-side helpers (no GPU): workload selection and slicing."""
import os
import sys

import pytest

from conftest import ROOT


def _bench(argv):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    old = sys.argv
    sys.argv = ["bench.py"] + argv
    try:
        return bench, bench.parse_args()
    finally:
        sys.argv = old


def test_default_workload_is_the_largest_single_gpu_config():
    bench, args = _bench([])
    w = bench.workload(args)
    assert w.name == "gpt_1_3b" and w.P == 8 and w.N == 1_311_178_752
    assert args.steps >= 1 and args.warmup >= 3


def test_oracle_sample_is_bounded():
    bench, _ = _bench([])
    from synth.configs import WORKLOADS
    for name, w in WORKLOADS.items():
        layers, per_worker = bench.oracle_sample_layers(w)
        assert layers == list(range(layers[0], layers[-1] + 1))
        assert per_worker == sum(w.sizes[l] for l in layers)
        assert per_worker <= max(bench.ORACLE_SAMPLE_ELEMS, max(w.sizes[l] for l in layers))
    layers, per_worker = bench.oracle_sample_layers(WORKLOADS["gpt_1_3b"])
    assert layers[:8] == list(range(1, 9))  # a whole transformer block
    assert 50_339_840 <= per_worker <= bench.ORACLE_SAMPLE_ELEMS


def test_traffic_scaling():
    bench, _ = _bench([])
    table = {"vgg16": (2000, 1000), "gpt_1_3b[1:9]": (300, 100)}
    assert bench.traffic_for(table, "vgg16", 1000) == (2000, "ncu capture of this workload (vgg16)")
    b, src = bench.traffic_for(table, "gpt_1_3b", 1000)
    assert b == 3000 and "gpt_1_3b[1:9]" in src      # own tensor range preferred
    b, src = bench.traffic_for(table, "lstm_ptb", 500)
    assert b == 1000 and "vgg16" in src


def test_oracle_timer_on_host_cores():
    bench, _ = _bench([])
    from synth.configs import WORKLOADS
    w = WORKLOADS["resnet20"]
    cpu = bench.cpu_baseline(w)
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] > 0
    assert cpu["single_thread"]["value"] > 0
    timer = bench.OracleTimer(w, procs=2)
    try:
        secs, elems = timer.run([(p, 3) for p in range(w.P)], step=1)
    finally:
        timer.close()
    assert secs > 0 and elems == w.P * w.sizes[3]


def test_tensor_range_slices_the_workload():
    bench, args = _bench(["--config", "gpt_1_3b", "--tensors", "1:9"])
    w = bench.workload(args)
    assert w.L == 8 and w.P == 8 and w.N == 50_339_840
    cfg = bench.workload_config(w)
    assert cfg["workload"] == "gpt_1_3b[1:9]" and cfg["elements_per_step"] == 8 * w.N


@pytest.mark.parametrize("spec", ["0:0", "5:3", "0:999"])
def test_tensor_range_rejects_bad_ranges(spec):
    bench, args = _bench(["--config", "resnet20", "--tensors", spec])
    with pytest.raises(SystemExit):
        bench.workload(args)


def test_pinned_host_buffers_split_across_local_ranks():
    import bench
    N = 1_311_178_752                      # 5.24 GB per buffer
    gb = 1 << 30
    assert bench.pinned_host_buffers(190 * gb, 1, 8, N) == min(8, (190 * gb // 4) // (N * 4))
    # eight ranks on one node: each gets an eighth of the quarter
    assert bench.pinned_host_buffers(190 * gb, 8, 8, N) == 1
    # never fewer than one buffer, never more than the workers
    assert bench.pinned_host_buffers(1 * gb, 8, 8, N) == 1
    assert bench.pinned_host_buffers(10_000 * gb, 1, 8, N) == 8
