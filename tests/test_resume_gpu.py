"""Checkpoint and resume: the step's state is the caller's residuals and
weights (the library keeps nothing across steps), so 5 steps, torch.save,
a fresh plan in a fresh set of buffers, torch.load, and 5 more steps end bit
for bit where 10 uninterrupted steps end, on ResNet-20 and VGG-16."""
import numpy as np
import pytest

import synth
from synth.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _fresh(w):
    import torch
    from layer_wise_top_b200 import Plan
    dev = torch.device("cuda")
    plan = Plan(w.sizes, w.densities, w.P, device=dev)
    idx, val = plan.empty_picks()
    return {"plan": plan, "idx": idx, "val": val,
            "grads": [torch.empty(w.N, device=dev) for _ in range(w.P)],
            "res": [torch.zeros(w.N, device=dev) for _ in range(w.P)],
            "dense": torch.empty(w.N, device=dev),
            "weights": torch.zeros(w.N, device=dev)}


def _steps(w, st, first, last):
    for s in range(first, last):
        for p in range(w.P):
            synth.worker_grads_device(w, p, s, st["grads"][p])
        st["plan"].sparsify(st["grads"], st["res"], w.lr, st["idx"], st["val"])
        st["plan"].aggregate_apply(st["idx"], st["val"], st["dense"], st["weights"])


@pytest.mark.parametrize("name", ["resnet20", "vgg16"])
def test_resume_equals_uninterrupted(name, tmp_path):
    import torch
    w = WORKLOADS[name]
    straight = _fresh(w)
    _steps(w, straight, 0, 10)

    first = _fresh(w)
    _steps(w, first, 0, 5)
    torch.cuda.synchronize()
    ckpt = tmp_path / "lags_state.pt"
    torch.save({"step": 5, "residuals": [r.cpu() for r in first["res"]],
                "weights": first["weights"].cpu()}, ckpt)
    del first
    torch.cuda.empty_cache()

    resumed = _fresh(w)
    state = torch.load(ckpt)
    for r, saved in zip(resumed["res"], state["residuals"]):
        r.copy_(saved)
    resumed["weights"].copy_(state["weights"])
    _steps(w, resumed, state["step"], 10)
    torch.cuda.synchronize()

    def u(t):
        return t.cpu().numpy().view(np.uint32)
    assert np.array_equal(u(resumed["weights"]), u(straight["weights"]))
    assert np.array_equal(u(resumed["dense"]), u(straight["dense"]))
    assert np.array_equal(u(resumed["idx"]), u(straight["idx"]))
    for a, b in zip(resumed["res"], straight["res"]):
        assert np.array_equal(u(a), u(b))
