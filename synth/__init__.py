"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

Only input generation lives here (Philox4x32-10 gradients and the workload
tables); no step of the sparsification method does.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Optional

import numpy as np

from . import build as _build
from .configs import NORMAL, STUDENT_T3, WORKLOADS, Tensor, Workload  # noqa: F401

_HOST = None
_DEV = None


def _host_lib():
    global _HOST
    if _HOST is None:
        if not os.path.exists(_build.HOST_SO):
            _build.build()
        lib = ctypes.CDLL(_build.HOST_SO)
        lib.synth_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                        ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                        ctypes.c_int, ctypes.c_float]
        lib.synth_fill_host.restype = None
        lib.synth_philox_block.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_uint32,
                                           ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32)]
        lib.synth_philox_block.restype = None
        _HOST = lib
    return _HOST


def _dev_lib():
    global _DEV
    if _DEV is None:
        if not os.path.exists(_build.DEV_SO):
            _build.build()
        lib = ctypes.CDLL(_build.DEV_SO)
        lib.synth_fill_device.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
        lib.synth_fill_device.restype = ctypes.c_int
        _DEV = lib
    return _DEV


def philox4x32_10(ctr, key) -> list:
    """One raw Philox4x32-10 block (for known-answer tests)."""
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    o = (ctypes.c_uint32 * 4)()
    _host_lib().synth_philox_block(c, int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF, o)
    return [int(x) for x in o]


def fill_host(out: np.ndarray, first: int, seed: int, worker: int, step: int, dist: int,
              scale: float) -> np.ndarray:
    assert out.dtype == np.float32 and out.flags.c_contiguous
    _host_lib().synth_fill_host(out.ctypes.data, first, out.size, seed, worker, step, dist,
                                float(np.float32(scale)))
    return out


def layer_grads_host(w: Workload, worker: int, step: int, layer: int) -> np.ndarray:
    """Gradient of one tensor of worker `worker` at step `step` (host, float32)."""
    t = w.tensors[layer]
    out = np.empty(t.size, dtype=np.float32)
    return fill_host(out, w.offsets[layer], w.seed, worker, step, w.dist, t.scale)


def worker_grads_host(w: Workload, worker: int, step: int) -> np.ndarray:
    """Flattened gradient buffer [N] of one worker at one step (host)."""
    out = np.empty(w.N, dtype=np.float32)
    for l, (t, off) in enumerate(zip(w.tensors, w.offsets)):
        fill_host(out[off:off + t.size], off, w.seed, worker, step, w.dist, t.scale)
    return out


def fill_device(ptr: int, first: int, count: int, seed: int, worker: int, step: int, dist: int,
                scale: float, stream: int = 0) -> None:
    rc = _dev_lib().synth_fill_device(ctypes.c_void_p(ptr), first, count, seed, worker, step,
                                      dist, float(np.float32(scale)), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_device failed: cuda error {rc}")


def worker_grads_device(w: Workload, worker: int, step: int, out,
                        layers: Optional[Iterable[int]] = None) -> None:
    """Fill a float32 CUDA tensor [N] with one worker's gradients at one step."""
    import torch
    assert out.dtype == torch.float32 and out.is_cuda and out.numel() >= w.N
    stream = torch.cuda.current_stream(out.device).cuda_stream
    base = out.data_ptr()
    ids = range(w.L) if layers is None else layers
    offs = w.offsets
    for l in ids:
        t = w.tensors[l]
        fill_device(base + 4 * offs[l], offs[l], t.size, w.seed, worker, step, w.dist, t.scale,
                    stream)
