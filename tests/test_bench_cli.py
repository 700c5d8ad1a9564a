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


def test_default_workload_is_vgg16():
    bench, args = _bench([])
    w = bench.workload(args)
    assert w.name == "vgg16" and w.P == 16 and w.N == 14_719_818
    assert args.steps >= 1 and args.warmup >= 3


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
