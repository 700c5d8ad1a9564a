"""A plan bound to torch-owned device memory: the convenience layer the tests
and the benchmark use.  It only checks tensors and passes their pointers and
the current CUDA stream to the C entry points."""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import _binding as B


def _stream(stream: Optional[torch.cuda.Stream], device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _need(t: torch.Tensor, dtype, numel: int, what: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous() or t.numel() < numel:
        raise ValueError(f"{what} must be contiguous with at least {numel} elements")


class Plan:
    """Layer table of one flattened gradient buffer shared by P workers.

    With `layer_range=(begin, end)` the plan covers only model layers
    [begin, end): buffers stay the whole model's (N is one past the range's
    last element), indices stay global, and the pick lists hold only the
    range's K picks per worker."""

    def __init__(self, layer_sizes: Sequence[int], densities: Sequence[float], P: int,
                 device: Optional[torch.device] = None,
                 layer_range: Optional[Tuple[int, int]] = None,
                 aggregate_only: bool = False):
        self.device = torch.device(device if device is not None else "cuda")
        self._destroy = B.raw_plan_destroy()
        if layer_range is None:
            lb, le = 0, len(layer_sizes)
            self.handle = B.lags_plan_create(layer_sizes, densities, P)
        else:
            lb, le = int(layer_range[0]), int(layer_range[1])
            self.handle = B.lags_plan_create_range(layer_sizes, densities, P, lb, le)
        self.layer_range = (lb, le)
        self.P = int(P)
        self.L = le - lb
        self.N, self.K, self.workspace_bytes = B.lags_plan_info(self.handle)
        self.layers = [B.lags_plan_layer(self.handle, l) for l in range(self.L)]
        self.sizes = [int(x) for x in layer_sizes[lb:le]]
        self.first = self.layers[0][0]  # first element of the plan's layers
        # a plan that only aggregates binds the smaller workspace without the
        # selection's candidate slots (sparsify then fails with LAGS_ERR_WORKSPACE)
        self.aggregate_only = bool(aggregate_only)
        if self.aggregate_only:
            self.workspace_bytes = B.lags_plan_aggregate_workspace_bytes(self.handle)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8,
                                         device=self.device)
            B.lags_plan_set_workspace(self.handle, self.workspace.data_ptr(),
                                      self.workspace.numel(), _stream(None, self.device))

    def __del__(self):
        # the raw C entry point, held by the instance: at interpreter exit the
        # binding module's globals may already be gone
        h = getattr(self, "handle", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self.handle = None

    # ---------------------------------------------------------------- buffers
    def empty_picks(self):
        idx = torch.empty(self.P * self.K, dtype=torch.int32, device=self.device)
        val = torch.empty(self.P * self.K, dtype=torch.float32, device=self.device)
        return idx, val

    # ---------------------------------------------------------------- calls
    def sparsify(self, grads: List[torch.Tensor], residuals: List[torch.Tensor], lr: float,
                 out_idx: torch.Tensor, out_val: torch.Tensor,
                 stream: Optional[torch.cuda.Stream] = None) -> None:
        if len(grads) != self.P or len(residuals) != self.P:
            raise ValueError(f"need {self.P} gradient and residual buffers")
        for i, (g, r) in enumerate(zip(grads, residuals)):
            _need(g, torch.float32, self.N, f"grads[{i}]")
            _need(r, torch.float32, self.N, f"residuals[{i}]")
        _need(out_idx, torch.int32, self.P * self.K, "out_idx")
        _need(out_val, torch.float32, self.P * self.K, "out_val")
        B.lags_sparsify(self.handle, [g.data_ptr() for g in grads],
                        [r.data_ptr() for r in residuals], lr, out_idx.data_ptr(),
                        out_val.data_ptr(), _stream(stream, self.device))

    def aggregate(self, idx: torch.Tensor, val: torch.Tensor, dense_out: torch.Tensor,
                  stream: Optional[torch.cuda.Stream] = None) -> None:
        _need(idx, torch.int32, self.P * self.K, "idx")
        _need(val, torch.float32, self.P * self.K, "val")
        _need(dense_out, torch.float32, self.N, "dense_out")
        B.lags_aggregate(self.handle, idx.data_ptr(), val.data_ptr(), dense_out.data_ptr(),
                         _stream(stream, self.device))

    def aggregate_apply(self, idx: torch.Tensor, val: torch.Tensor, dense_out: torch.Tensor,
                        weights: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
        _need(idx, torch.int32, self.P * self.K, "idx")
        _need(val, torch.float32, self.P * self.K, "val")
        _need(dense_out, torch.float32, self.N, "dense_out")
        _need(weights, torch.float32, self.N, "weights")
        B.lags_aggregate_apply(self.handle, idx.data_ptr(), val.data_ptr(), dense_out.data_ptr(),
                               weights.data_ptr(), _stream(stream, self.device))

    def kernel_launches(self):
        """Kernels enqueued by one sparsify, aggregate and apply call."""
        return B.lags_plan_kernel_launches(self.handle)

    def apply(self, weights: torch.Tensor, dense_out: torch.Tensor,
              stream: Optional[torch.cuda.Stream] = None) -> None:
        _need(weights, torch.float32, self.N, "weights")
        _need(dense_out, torch.float32, self.N, "dense_out")
        B.lags_apply(self.handle, weights.data_ptr(), dense_out.data_ptr(),
                     _stream(stream, self.device))

    def set_events(self, before: Optional[torch.cuda.Event],
                   after: Optional[torch.cuda.Event]) -> None:
        """Record `before`/`after` around the fused pass of later sparsify calls."""
        if before is None or after is None:
            B.lags_plan_set_events(self.handle, 0, 0)
            return
        for ev in (before, after):
            if not ev.cuda_event:  # torch creates the event on first record
                ev.record()
        B.lags_plan_set_events(self.handle, before.cuda_event, after.cuda_event)

    def poll(self, stream: Optional[torch.cuda.Stream] = None):
        """(flags, exact_fallbacks) since the last poll; synchronises the stream.
        Raises LagsError (carrying the flags) when a flag reports an error."""
        return B.lags_status_poll(self.handle, _stream(stream, self.device))

    def set_stage_wait_limit(self, polls: int) -> None:
        """Failure-injection knob: polls of the selection's first staging wait."""
        B.lags_plan_set_stage_wait_limit(self.handle, polls)

    def set_index_wait_limit(self, polls: int) -> None:
        """Failure-injection knob: polls of the values-only selection's wait for
        its index copies."""
        B.lags_plan_set_index_wait_limit(self.handle, polls)


class DenseKernels:
    """The dense S-SGD baseline's two kernels on torch tensors (no plan)."""

    def __init__(self, N: int, device: Optional[torch.device] = None):
        self.N = int(N)
        self.device = torch.device(device if device is not None else "cuda")

    def sum(self, grads: List[torch.Tensor], lr: float, out: torch.Tensor,
            stream: Optional[torch.cuda.Stream] = None) -> None:
        """out = worker-ordered sum of fl(lr * g_p)."""
        for i, g in enumerate(grads):
            _need(g, torch.float32, self.N, f"grads[{i}]")
        _need(out, torch.float32, self.N, "sum_out")
        B.lags_dense_sum([g.data_ptr() for g in grads], self.N, lr, out.data_ptr(),
                         _stream(stream, self.device))

    def finish(self, sum_in: torch.Tensor, P_total: int, dense_out: torch.Tensor,
               weights: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> None:
        """dense_out = sum / P_total; weights -= dense_out when given."""
        _need(sum_in, torch.float32, self.N, "sum")
        _need(dense_out, torch.float32, self.N, "dense_out")
        if weights is not None:
            _need(weights, torch.float32, self.N, "weights")
        B.lags_dense_finish(sum_in.data_ptr(), self.N, P_total, dense_out.data_ptr(),
                            weights.data_ptr() if weights is not None else 0,
                            _stream(stream, self.device))
