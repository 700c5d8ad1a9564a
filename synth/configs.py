"""Workload tables: the gradient tensor lists of the five synthetic workloads.

These shapes stand in for the models the LAGS-SGD review reports on (ResNet-20,
VGG-16, ResNet-50, LSTM-PTB; "Layer-wise Adaptive Gradient Sparsification ...",
main findings) plus a 1.3B-parameter transformer.  No dataset or trained weight
is involved: gradients come from the seeded generator in ``synth.gen``.

A workload fixes: the ordered tensor list (name, shape), the number of
simulated workers P, the learning rate, the per-layer density rule, the number
of steps, the gradient distribution and the seed.  Nothing here computes a step
of the method.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Sequence, Tuple

import numpy as np

NORMAL = 0      # N(0, 1/fan_in), Irwin-Hall normal
STUDENT_T3 = 1  # Student-t (nu = 3) scaled by 1/sqrt(fan_in)


@dataclass(frozen=True)
class Tensor:
    name: str
    shape: Tuple[int, ...]

    @property
    def size(self) -> int:
        return int(np.prod(self.shape, dtype=np.int64))

    @property
    def fan_in(self) -> int:
        # 2-D and higher: product of all dims but the first; 1-D: its length.
        if len(self.shape) >= 2:
            return int(np.prod(self.shape[1:], dtype=np.int64))
        return int(self.shape[0])

    @property
    def scale(self) -> np.float32:
        """1/sqrt(fan_in), rounded once to float32 (host double arithmetic)."""
        return np.float32(1.0 / math.sqrt(self.fan_in))


@dataclass(frozen=True)
class Workload:
    name: str
    tensors: Tuple[Tensor, ...]
    P: int
    lr: float
    steps: int
    dist: int
    seed: int
    density_rule: Callable[[int], float] = field(compare=False)

    @property
    def sizes(self) -> List[int]:
        return [t.size for t in self.tensors]

    @property
    def densities(self) -> List[float]:
        return [self.density_rule(t.size) for t in self.tensors]

    @property
    def offsets(self) -> List[int]:
        out, acc = [], 0
        for t in self.tensors:
            out.append(acc)
            acc += t.size
        return out

    @property
    def N(self) -> int:
        return int(sum(self.sizes))

    @property
    def L(self) -> int:
        return len(self.tensors)

    def scaled(self, name: str, P: int | None = None, steps: int | None = None,
               tensors: Sequence[Tensor] | None = None,
               density_rule: Callable[[int], float] | None = None) -> "Workload":
        """A smaller variant (for tests): same distribution, lr and seed."""
        return Workload(name, tuple(tensors) if tensors is not None else self.tensors,
                        P if P is not None else self.P, self.lr,
                        steps if steps is not None else self.steps, self.dist, self.seed,
                        density_rule if density_rule is not None else self.density_rule)


def _const(rho: float) -> Callable[[int], float]:
    return lambda d: rho


def adaptive_resnet50(d: int) -> float:
    """Per-layer density of the ResNet-50 workload: dense below 1e4 elements,
    0.01 up to 1e6, 0.001 above."""
    if d < 10_000:
        return 1.0
    if d <= 1_000_000:
        return 0.01
    return 0.001


def _resnet20() -> Tuple[Tensor, ...]:
    t = [Tensor("conv1", (16, 3, 3, 3))]
    t += [Tensor(f"stage1.conv{i}", (16, 16, 3, 3)) for i in range(6)]
    t += [Tensor("stage2.conv0", (32, 16, 3, 3))]
    t += [Tensor(f"stage2.conv{i}", (32, 32, 3, 3)) for i in range(1, 6)]
    t += [Tensor("stage3.conv0", (64, 32, 3, 3))]
    t += [Tensor(f"stage3.conv{i}", (64, 64, 3, 3)) for i in range(1, 6)]
    t += [Tensor("fc.weight", (10, 64)), Tensor("fc.bias", (10,))]
    return tuple(t)


def _vgg16() -> Tuple[Tensor, ...]:
    chans = [64, 64, 128, 128, 256, 256, 256, 512, 512, 512, 512, 512, 512]
    t, cin = [], 3
    for i, c in enumerate(chans):
        t.append(Tensor(f"conv{i}.weight", (c, cin, 3, 3)))
        t.append(Tensor(f"conv{i}.bias", (c,)))
        cin = c
    t += [Tensor("fc.weight", (10, 512)), Tensor("fc.bias", (10,))]
    return tuple(t)


def _resnet50() -> Tuple[Tensor, ...]:
    t = [Tensor("conv1.weight", (64, 3, 7, 7)), Tensor("bn1.weight", (64,)),
         Tensor("bn1.bias", (64,))]
    inplanes = 64
    for li, (planes, blocks) in enumerate([(64, 3), (128, 4), (256, 6), (512, 3)], start=1):
        for b in range(blocks):
            pre = f"layer{li}.{b}"
            t.append(Tensor(f"{pre}.conv1.weight", (planes, inplanes, 1, 1)))
            t += [Tensor(f"{pre}.bn1.weight", (planes,)), Tensor(f"{pre}.bn1.bias", (planes,))]
            t.append(Tensor(f"{pre}.conv2.weight", (planes, planes, 3, 3)))
            t += [Tensor(f"{pre}.bn2.weight", (planes,)), Tensor(f"{pre}.bn2.bias", (planes,))]
            t.append(Tensor(f"{pre}.conv3.weight", (planes * 4, planes, 1, 1)))
            t += [Tensor(f"{pre}.bn3.weight", (planes * 4,)),
                  Tensor(f"{pre}.bn3.bias", (planes * 4,))]
            if b == 0:
                t.append(Tensor(f"{pre}.downsample.0.weight", (planes * 4, inplanes, 1, 1)))
                t += [Tensor(f"{pre}.downsample.1.weight", (planes * 4,)),
                      Tensor(f"{pre}.downsample.1.bias", (planes * 4,))]
            inplanes = planes * 4
    t += [Tensor("fc.weight", (1000, 2048)), Tensor("fc.bias", (1000,))]
    return tuple(t)


def _lstm_ptb() -> Tuple[Tensor, ...]:
    # One (4*hidden) x (input + hidden) weight tensor per LSTM layer plus the
    # input-side and hidden-side bias vectors.
    t = [Tensor("embedding", (10000, 1500))]
    for layer in range(2):
        t += [Tensor(f"lstm{layer}.weight", (4 * 1500, 3000)),
              Tensor(f"lstm{layer}.bias_ih", (6000,)), Tensor(f"lstm{layer}.bias_hh", (6000,))]
    t += [Tensor("decoder.weight", (10000, 1500)), Tensor("decoder.bias", (10000,))]
    return tuple(t)


def _gpt_1_3b() -> Tuple[Tensor, ...]:
    d = 2048
    t = [Tensor("wte", (50304, d))]
    for i in range(24):
        t += [Tensor(f"h{i}.ln1.weight", (d,)), Tensor(f"h{i}.ln1.bias", (d,)),
              Tensor(f"h{i}.attn.qkv", (3 * d, d)), Tensor(f"h{i}.attn.out", (d, d)),
              Tensor(f"h{i}.ln2.weight", (d,)), Tensor(f"h{i}.ln2.bias", (d,)),
              Tensor(f"h{i}.mlp.fc1", (4 * d, d)), Tensor(f"h{i}.mlp.fc2", (d, 4 * d))]
    return tuple(t)


RESNET20 = Workload("resnet20", _resnet20(), P=4, lr=0.1, steps=10, dist=NORMAL, seed=1,
                    density_rule=_const(0.001))
VGG16 = Workload("vgg16", _vgg16(), P=16, lr=0.1, steps=10, dist=NORMAL, seed=2,
                 density_rule=_const(0.001))
RESNET50 = Workload("resnet50", _resnet50(), P=16, lr=0.1, steps=10, dist=NORMAL, seed=3,
                    density_rule=adaptive_resnet50)
LSTM_PTB = Workload("lstm_ptb", _lstm_ptb(), P=16, lr=1.0, steps=10, dist=STUDENT_T3, seed=4,
                    density_rule=_const(0.001))
GPT_1_3B = Workload("gpt_1_3b", _gpt_1_3b(), P=8, lr=0.01, steps=5, dist=STUDENT_T3, seed=5,
                    density_rule=_const(0.001))

WORKLOADS = {w.name: w for w in (RESNET20, VGG16, RESNET50, LSTM_PTB, GPT_1_3B)}
