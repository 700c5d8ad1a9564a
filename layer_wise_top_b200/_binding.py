"""ctypes binding of liblags.so: one Python function per C entry point, same
names, argument marshalling only.  Every step of the computation runs in the
library's CUDA kernels; there is no Python or CPU fallback, and importing this
module fails if the library has not been built."""
from __future__ import annotations

import ctypes
import os
from typing import Sequence, Tuple

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblags.so")

LAGS_OK = 0
LAGS_ERR_INVALID_ARG = 1
LAGS_ERR_ALIGNMENT = 2
LAGS_ERR_CUDA = 3
LAGS_ERR_UNSUPPORTED_DEVICE = 4
LAGS_ERR_WORKSPACE = 5
LAGS_ERR_BAD_PICKS = 6
LAGS_ERR_TIMEOUT = 7
LAGS_ERR_INTERNAL = 8
LAGS_ERR_WRONG_DEVICE = 9
LAGS_STAGE_WAIT_POLLS = 4194304
LAGS_MAX_WORKERS = 256
LAGS_MAX_ELEMENTS = (1 << 32) - 65536
LAGS_FLAG_BAD_PICKS = 0x1
LAGS_FLAG_INTERNAL = 0x2
LAGS_FLAG_TIMEOUT = 0x4

EXPORTED = ("lags_plan_create", "lags_plan_destroy", "lags_plan_info", "lags_plan_layer",
            "lags_plan_set_workspace", "lags_sparsify", "lags_aggregate", "lags_apply",
            "lags_status_poll", "lags_plan_set_events", "lags_sparsify_static",
            "lags_aggregate_apply", "lags_plan_kernel_launches", "lags_adaptive_densities",
            "lags_plan_create_range", "lags_merge_layers", "lags_dense_sum",
            "lags_dense_finish", "lags_plan_aggregate_workspace_bytes",
            "lags_plan_set_stage_wait_limit", "lags_plan_set_index_wait_limit",
            "lags_static_status_poll", "lags_error_string")


class LagsError(RuntimeError):
    """A non-OK lags_status.  A status poll that fails also carries the
    flags and exhaustive-path count it read."""

    def __init__(self, status: int, where: str, flags: int = 0, fallbacks: int = 0):
        self.status = status
        self.flags = flags
        self.fallbacks = fallbacks
        extra = f", flags {flags:#x}" if flags else ""
        super().__init__(f"{where}: {lags_error_string(status)} (status {status}{extra})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python layer_wise_top_b200/build.py` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64)
    st = ctypes.c_int
    lib.lags_plan_create.argtypes = [i64p, ctypes.POINTER(ctypes.c_double), i32, i32,
                                     ctypes.POINTER(vp)]
    lib.lags_plan_create_range.argtypes = [i64p, ctypes.POINTER(ctypes.c_double), i32, i32,
                                           i32, i32, ctypes.POINTER(vp)]
    lib.lags_plan_destroy.argtypes = [vp]
    lib.lags_plan_info.argtypes = [vp, i64p, i64p, ctypes.POINTER(ctypes.c_size_t)]
    lib.lags_plan_layer.argtypes = [vp, i32, i64p, i64p, i64p]
    lib.lags_plan_set_workspace.argtypes = [vp, vp, ctypes.c_size_t, vp]
    lib.lags_sparsify.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.c_float,
                                  vp, vp, vp]
    lib.lags_aggregate.argtypes = [vp, vp, vp, vp, vp]
    lib.lags_apply.argtypes = [vp, vp, vp, vp]
    lib.lags_aggregate_apply.argtypes = [vp, vp, vp, vp, vp, vp]
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.lags_plan_kernel_launches.argtypes = [vp, i32p, i32p, i32p]
    dp_ = ctypes.POINTER(ctypes.c_double)
    lib.lags_adaptive_densities.argtypes = [i64p, dp_, i32, ctypes.c_double, ctypes.c_double,
                                            ctypes.c_double, dp_]
    lib.lags_merge_layers.argtypes = [i64p, dp_, i32, ctypes.c_double, ctypes.c_double, i32p,
                                      i32p, dp_]
    lib.lags_dense_sum.argtypes = [ctypes.POINTER(vp), i32, ctypes.c_int64, ctypes.c_float, vp,
                                   vp]
    lib.lags_dense_finish.argtypes = [vp, ctypes.c_int64, i32, vp, vp, vp]
    lib.lags_status_poll.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32),
                                     ctypes.POINTER(ctypes.c_uint32), vp]
    lib.lags_plan_set_events.argtypes = [vp, vp, vp]
    lib.lags_sparsify_static.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                         ctypes.c_float, vp, vp, vp]
    lib.lags_static_status_poll.argtypes = [ctypes.POINTER(ctypes.c_uint32),
                                            ctypes.POINTER(ctypes.c_uint32), vp]
    lib.lags_plan_aggregate_workspace_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
    lib.lags_plan_set_stage_wait_limit.argtypes = [vp, ctypes.c_uint32]
    lib.lags_plan_set_index_wait_limit.argtypes = [vp, ctypes.c_uint32]
    lib.lags_error_string.argtypes = [st]
    lib.lags_error_string.restype = ctypes.c_char_p
    for name in EXPORTED[:-1]:
        getattr(lib, name).restype = st
    return lib


_LIB = _load()


def library() -> ctypes.CDLL:
    return _LIB


def _check(status: int, where: str) -> None:
    if status != LAGS_OK:
        raise LagsError(status, where)


def lags_error_string(status: int) -> str:
    return _LIB.lags_error_string(int(status)).decode()


def lags_plan_create(layer_sizes: Sequence[int], densities: Sequence[float],
                     num_workers: int) -> ctypes.c_void_p:
    L = len(layer_sizes)
    if len(densities) != L:
        raise ValueError("layer_sizes and densities differ in length")
    sizes = (ctypes.c_int64 * max(L, 1))(*[int(x) for x in layer_sizes])
    dens = (ctypes.c_double * max(L, 1))(*[float(x) for x in densities])
    out = ctypes.c_void_p()
    _check(_LIB.lags_plan_create(sizes, dens, L, int(num_workers), ctypes.byref(out)),
           "lags_plan_create")
    return out


def lags_plan_create_range(layer_sizes: Sequence[int], densities: Sequence[float],
                           num_workers: int, layer_begin: int, layer_end: int) -> ctypes.c_void_p:
    L = len(layer_sizes)
    if len(densities) != L:
        raise ValueError("layer_sizes and densities differ in length")
    sizes = (ctypes.c_int64 * max(L, 1))(*[int(x) for x in layer_sizes])
    dens = (ctypes.c_double * max(L, 1))(*[float(x) for x in densities])
    out = ctypes.c_void_p()
    _check(_LIB.lags_plan_create_range(sizes, dens, L, int(num_workers), int(layer_begin),
                                       int(layer_end), ctypes.byref(out)),
           "lags_plan_create_range")
    return out


def lags_plan_destroy(plan) -> None:
    _check(_LIB.lags_plan_destroy(plan), "lags_plan_destroy")


def raw_plan_destroy():
    """The C entry point itself, for destructors that may run at interpreter
    exit (after this module's globals are cleared); its status is ignored."""
    return _LIB.lags_plan_destroy


def lags_plan_info(plan) -> Tuple[int, int, int]:
    n, k, ws = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_size_t()
    _check(_LIB.lags_plan_info(plan, ctypes.byref(n), ctypes.byref(k), ctypes.byref(ws)),
           "lags_plan_info")
    return n.value, k.value, ws.value


def lags_plan_aggregate_workspace_bytes(plan) -> int:
    n = ctypes.c_size_t()
    _check(_LIB.lags_plan_aggregate_workspace_bytes(plan, ctypes.byref(n)),
           "lags_plan_aggregate_workspace_bytes")
    return n.value


def lags_plan_set_stage_wait_limit(plan, polls: int) -> None:
    _check(_LIB.lags_plan_set_stage_wait_limit(plan, int(polls)),
           "lags_plan_set_stage_wait_limit")


def lags_plan_set_index_wait_limit(plan, polls: int) -> None:
    _check(_LIB.lags_plan_set_index_wait_limit(plan, int(polls)),
           "lags_plan_set_index_wait_limit")


def lags_plan_layer(plan, l: int) -> Tuple[int, int, int]:
    o, k, ko = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(_LIB.lags_plan_layer(plan, int(l), ctypes.byref(o), ctypes.byref(k),
                                ctypes.byref(ko)), "lags_plan_layer")
    return o.value, k.value, ko.value


def lags_plan_set_workspace(plan, workspace: int, nbytes: int, stream: int = 0) -> None:
    _check(_LIB.lags_plan_set_workspace(plan, ctypes.c_void_p(workspace), int(nbytes),
                                        ctypes.c_void_p(stream)), "lags_plan_set_workspace")


def lags_sparsify(plan, grads: Sequence[int], residuals: Sequence[int], lr: float,
                  out_idx: int, out_val: int, stream: int = 0) -> None:
    P = len(grads)
    g = (ctypes.c_void_p * max(P, 1))(*[ctypes.c_void_p(x) for x in grads])
    r = (ctypes.c_void_p * max(len(residuals), 1))(*[ctypes.c_void_p(x) for x in residuals])
    _check(_LIB.lags_sparsify(plan, g, r, ctypes.c_float(lr), ctypes.c_void_p(out_idx),
                              ctypes.c_void_p(out_val), ctypes.c_void_p(stream)),
           "lags_sparsify")


def lags_sparsify_static(plan, grads: Sequence[int], residuals: Sequence[int], lr: float,
                         out_idx: int, out_val: int, stream: int = 0) -> None:
    """lags_sparsify with the library's static scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/lags.h)."""
    P = len(grads)
    g = (ctypes.c_void_p * max(P, 1))(*[ctypes.c_void_p(x) for x in grads])
    r = (ctypes.c_void_p * max(len(residuals), 1))(*[ctypes.c_void_p(x) for x in residuals])
    _check(_LIB.lags_sparsify_static(plan, g, r, ctypes.c_float(lr), ctypes.c_void_p(out_idx),
                                     ctypes.c_void_p(out_val), ctypes.c_void_p(stream)),
           "lags_sparsify_static")


def lags_aggregate(plan, idx: int, val: int, dense_out: int, stream: int = 0) -> None:
    _check(_LIB.lags_aggregate(plan, ctypes.c_void_p(idx), ctypes.c_void_p(val),
                               ctypes.c_void_p(dense_out), ctypes.c_void_p(stream)),
           "lags_aggregate")


def lags_aggregate_apply(plan, idx: int, val: int, dense_out: int, weights: int,
                         stream: int = 0) -> None:
    _check(_LIB.lags_aggregate_apply(plan, ctypes.c_void_p(idx), ctypes.c_void_p(val),
                                     ctypes.c_void_p(dense_out), ctypes.c_void_p(weights),
                                     ctypes.c_void_p(stream)), "lags_aggregate_apply")


def lags_plan_kernel_launches(plan) -> Tuple[int, int, int]:
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_LIB.lags_plan_kernel_launches(plan, ctypes.byref(a), ctypes.byref(b),
                                          ctypes.byref(c)), "lags_plan_kernel_launches")
    return a.value, b.value, c.value


def lags_adaptive_densities(layer_sizes: Sequence[int], backward_seconds: Sequence[float],
                            alpha: float, beta: float, rho_min: float) -> list:
    """Per-layer densities from each layer's communication-to-computation
    ratio (see include/lags.h for the rule)."""
    L = len(layer_sizes)
    if len(backward_seconds) != L:
        raise ValueError("layer_sizes and backward_seconds differ in length")
    sizes = (ctypes.c_int64 * max(L, 1))(*[int(x) for x in layer_sizes])
    t = (ctypes.c_double * max(L, 1))(*[float(x) for x in backward_seconds])
    out = (ctypes.c_double * max(L, 1))()
    _check(_LIB.lags_adaptive_densities(sizes, t, L, float(alpha), float(beta), float(rho_min),
                                        out), "lags_adaptive_densities")
    return [out[i] for i in range(L)]


def lags_merge_layers(message_bytes: Sequence[int], backward_seconds: Sequence[float],
                      alpha: float, beta: float) -> Tuple[list, float]:
    """Buckets of consecutive layers, one message each, whose last message
    ends earliest (see include/lags.h for the model).  Returns the list of
    (first layer, end layer) pairs in forward order and that end time."""
    L = len(message_bytes)
    if len(backward_seconds) != L:
        raise ValueError("message_bytes and backward_seconds differ in length")
    b = (ctypes.c_int64 * max(L, 1))(*[int(x) for x in message_bytes])
    t = (ctypes.c_double * max(L, 1))(*[float(x) for x in backward_seconds])
    first = (ctypes.c_int32 * max(L, 1))()
    nb, end = ctypes.c_int32(), ctypes.c_double()
    _check(_LIB.lags_merge_layers(b, t, L, float(alpha), float(beta), first, ctypes.byref(nb),
                                  ctypes.byref(end)), "lags_merge_layers")
    f = [first[i] for i in range(nb.value)] + [L]
    return [(f[i], f[i + 1]) for i in range(nb.value)], end.value


def lags_dense_sum(grads: Sequence[int], N: int, lr: float, sum_out: int,
                   stream: int = 0) -> None:
    P = len(grads)
    g = (ctypes.c_void_p * max(P, 1))(*[ctypes.c_void_p(x) for x in grads])
    _check(_LIB.lags_dense_sum(g, P, int(N), ctypes.c_float(lr), ctypes.c_void_p(sum_out),
                               ctypes.c_void_p(stream)), "lags_dense_sum")


def lags_dense_finish(sum_in: int, N: int, num_workers_total: int, dense_out: int,
                      weights: int = 0, stream: int = 0) -> None:
    _check(_LIB.lags_dense_finish(ctypes.c_void_p(sum_in), int(N), int(num_workers_total),
                                  ctypes.c_void_p(dense_out), ctypes.c_void_p(weights),
                                  ctypes.c_void_p(stream)), "lags_dense_finish")


def lags_apply(plan, weights: int, dense_out: int, stream: int = 0) -> None:
    _check(_LIB.lags_apply(plan, ctypes.c_void_p(weights), ctypes.c_void_p(dense_out),
                           ctypes.c_void_p(stream)), "lags_apply")


def lags_plan_set_events(plan, before: int, after: int) -> None:
    _check(_LIB.lags_plan_set_events(plan, ctypes.c_void_p(before), ctypes.c_void_p(after)),
           "lags_plan_set_events")


def _poll_result(status: int, f, fb, where: str) -> Tuple[int, int]:
    if status != LAGS_OK:
        raise LagsError(status, where, f.value, fb.value)
    return f.value, fb.value


def lags_status_poll(plan, stream: int = 0) -> Tuple[int, int]:
    """Returns (flags, exact_fallbacks); raises LagsError (with .flags) when a
    flag reports a timeout, a failed self-check or malformed pick lists."""
    f, fb = ctypes.c_uint32(), ctypes.c_uint32()
    st = _LIB.lags_status_poll(plan, ctypes.byref(f), ctypes.byref(fb), ctypes.c_void_p(stream))
    return _poll_result(st, f, fb, "lags_status_poll")


def lags_static_status_poll(stream: int = 0) -> Tuple[int, int]:
    """lags_status_poll for lags_sparsify_static (the current device's static
    status words)."""
    f, fb = ctypes.c_uint32(), ctypes.c_uint32()
    st = _LIB.lags_static_status_poll(ctypes.byref(f), ctypes.byref(fb), ctypes.c_void_p(stream))
    return _poll_result(st, f, fb, "lags_static_status_poll")
