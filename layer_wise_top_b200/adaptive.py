"""Adaptive per-layer densities from measured backward times (host planner).

LAGS ("Layer-wise Adaptive Gradient Sparsification ..." review, "proposed
method", second bullet) sets each layer's sparsification ratio from its
communication-to-computation ratio, so that the layer's message hides behind
the rest of the backward pass.  The planning rule itself runs in the library
(``lags_adaptive_densities``: a layer's message starts when its gradient
exists and the link is free, and gets the largest density that still ends by
the end of the backward pass).  This module supplies its inputs:

- the backward time of every layer, measured on the device with CUDA events
  around a synthetic backward pass.  The model's own backward is not part of
  this library, so each layer's stands in as the two GEMMs that produce its
  weight gradient and its input gradient for `rows` rows of activations (the
  batch, times the spatial positions of a convolution), in bf16, or a
  column sum for one-dimensional tensors (biases, norm scales).  Layers run
  from the last to the first, as backpropagation produces them;
- the link's start-up time and per-byte time (alpha, beta).  The pages'
  cluster is 16 GPUs on 10 Gb Ethernet; NVLink 5 through NVSwitch is the link
  of one B200 node.  In an all-gather every worker receives the other
  workers' 8-byte picks, so one layer's message of k picks per worker moves
  8 k (P - 1) bytes: the per-pick time passed to the planner is
  beta (P - 1).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import _binding as B

# link presets: (alpha seconds per message, beta seconds per byte)
LINKS: Dict[str, Tuple[float, float]] = {
    "10gbe": (50e-6, 8.0 / 10e9),      # the pages' cluster network
    "nvlink": (20e-6, 1.0 / 770e9),    # measured peer bandwidth per direction, one node
}


def _gemm_dims(shape: Sequence[int]) -> Tuple[int, int]:
    out = int(shape[0])
    fan_in = 1
    for s in shape[1:]:
        fan_in *= int(s)
    return out, fan_in


def measure_backward_seconds(shapes: Sequence[Sequence[int]], rows: int = 4096,
                             repeats: int = 5, device: Optional[torch.device] = None
                             ) -> List[float]:
    """Device time (seconds) of a synthetic backward of every layer, in the
    layers' forward order.  Each layer is timed on its own (CUDA events on
    the current stream, after one untimed run), from the last layer to the
    first; `repeats` runs are averaged."""
    dev = torch.device(device if device is not None else "cuda")
    times = [0.0] * len(shapes)
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev)
        for l in range(len(shapes) - 1, -1, -1):
            shape = shapes[l]
            if len(shape) >= 2:
                out, fan_in = _gemm_dims(shape)
                gen = torch.Generator(device=dev).manual_seed(l)
                dy = torch.randn(rows, out, device=dev, dtype=torch.bfloat16, generator=gen)
                x = torch.randn(rows, fan_in, device=dev, dtype=torch.bfloat16, generator=gen)
                w = torch.randn(out, fan_in, device=dev, dtype=torch.bfloat16, generator=gen)

                def run():
                    torch.mm(dy.t(), x)   # weight gradient [out, fan_in]
                    torch.mm(dy, w)       # input gradient [rows, fan_in]
            else:
                d = int(shape[0])
                gen = torch.Generator(device=dev).manual_seed(l)
                dy = torch.randn(rows, d, device=dev, dtype=torch.bfloat16, generator=gen)

                def run():
                    dy.sum(dim=0)         # bias / norm-scale gradient
            run()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(repeats):
                run()
            b.record(stream)
            b.synchronize()
            times[l] = a.elapsed_time(b) / 1e3 / repeats
            del run
    return times


def adaptive_densities(sizes: Sequence[int], backward_seconds: Sequence[float],
                       workers: int, link: str = "10gbe", rho_min: float = 0.001) -> List[float]:
    """Densities from the library's planner for `workers` workers exchanging
    picks over `link` (a key of LINKS)."""
    alpha, beta = LINKS[link]
    return B.lags_adaptive_densities(sizes, backward_seconds, alpha,
                                     beta * max(1, int(workers) - 1), rho_min)


def plan_densities(shapes: Sequence[Sequence[int]], workers: int, link: str = "10gbe",
                   rho_min: float = 0.001, rows: int = 4096,
                   device: Optional[torch.device] = None) -> Tuple[List[float], List[float]]:
    """Measure the layers' backward times, then plan: (densities, seconds)."""
    secs = measure_backward_seconds(shapes, rows=rows, device=device)
    sizes = []
    for s in shapes:
        n = 1
        for x in s:
            n *= int(x)
        sizes.append(n)
    return adaptive_densities(sizes, secs, workers, link, rho_min), secs
