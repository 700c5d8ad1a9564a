"""The seeded input generator: Philox known-answer vectors, the shape of the
distributions, and (GPU) host == device bit for bit."""
import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS


def test_philox_known_answers():
    import os
    from conftest import ROOT
    with open(os.path.join(ROOT, "tests", "golden", "philox4x32_10_kat.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        ctr = [int(x, 16) for x in r[0:4]]
        key = [int(x, 16) for x in r[4:6]]
        exp = [int(x, 16) for x in r[6:10]]
        assert synth.philox4x32_10(ctr, key) == exp


def test_normal_moments():
    x = np.empty(400_000, dtype=np.float32)
    synth.fill_host(x, 0, 7, 0, 0, synth.NORMAL, 1.0)
    assert abs(float(x.mean())) < 0.01
    assert abs(float(x.var()) - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0


def test_student_t_heavy_tail():
    x = np.empty(400_000, dtype=np.float32)
    synth.fill_host(x, 0, 7, 0, 0, synth.STUDENT_T3, 1.0)
    assert np.isfinite(x).all()
    # t(3): P(|T| > 5) ~ 1.5%; a normal would give ~6e-7
    frac = float((np.abs(x) > 5).mean())
    assert 0.008 < frac < 0.025


def test_streams_differ_by_worker_step_and_are_reproducible():
    w = WORKLOADS["resnet20"]
    a = synth.layer_grads_host(w, 0, 0, 3)
    b = synth.layer_grads_host(w, 1, 0, 3)
    c = synth.layer_grads_host(w, 0, 1, 3)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    assert np.array_equal(a, synth.layer_grads_host(w, 0, 0, 3))
    # the worker buffer is the concatenation of its layers
    full = synth.worker_grads_host(w, 0, 0)
    off = w.offsets[3]
    assert np.array_equal(full[off:off + a.size], a)


@pytest.mark.gpu
def test_device_matches_host_bitwise():
    import torch
    for name in ("resnet20", "lstm_ptb"):
        w = WORKLOADS[name]
        for p, s in ((0, 0), (w.P - 1, 3)):
            # sampled layers: all for resnet20, the small ones for the LSTM
            layers = range(w.L) if name == "resnet20" else [2, 3, 8]
            buf = torch.empty(w.N, dtype=torch.float32, device="cuda")
            synth.worker_grads_device(w, p, s, buf, layers=layers)
            torch.cuda.synchronize()
            for l in layers:
                off, d = w.offsets[l], w.sizes[l]
                dev = buf[off:off + d].cpu().numpy()
                host = synth.layer_grads_host(w, p, s, l)
                assert np.array_equal(dev.view(np.uint32), host.view(np.uint32)), (name, l)
