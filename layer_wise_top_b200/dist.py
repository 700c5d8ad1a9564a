"""Data-parallel LAGS across processes (one per GPU).

Every rank holds `workers_per_rank` workers of one job.  A step is:

1. local sparsify: error feedback and layer-wise top-k of the rank's own
   workers (``lags_sparsify``);
2. exchange: one all-gather of the fixed-size pick lists (indices and values,
   ``[workers_per_rank, K]`` each) over the process group.  The lists have a
   fixed size because every k_l is fixed, so no sizes are exchanged; the
   gathered lists are in rank-major order, i.e. global worker
   ``rank * workers_per_rank + p``;
3. aggregation of all workers' picks in global worker order and the weight
   update (``lags_aggregate_apply``), identically on every rank, so all ranks
   hold bit-identical updates and weights.

This is the synchronous, sparsified S-SGD step of the LAGS review (abstract:
workers exchange their significant gradients, then every worker applies the
same averaged update), with NCCL over NVLink as the transport.

The compute objects are the library's plans; tests may pass other objects with
the same methods (``sparsify``, ``aggregate_apply``) to exercise the exchange
on CPU ranks.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


class DataParallelLags:
    """One LAGS step over `world` ranks x `workers_per_rank` workers."""

    def __init__(self, local_plan, total_plan, workers_per_rank: int, K: int,
                 device: torch.device, group: Optional[dist.ProcessGroup] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.local = local_plan
        self.total = total_plan
        self.P_local = int(workers_per_rank)
        self.P_total = self.P_local * self.world
        self.K = int(K)
        n_local = self.P_local * self.K
        self.idx_local = torch.empty(n_local, dtype=torch.int32, device=device)
        self.val_local = torch.empty(n_local, dtype=torch.float32, device=device)
        self.idx_all = torch.empty(n_local * self.world, dtype=torch.int32, device=device)
        self.val_all = torch.empty(n_local * self.world, dtype=torch.float32, device=device)

    @classmethod
    def create(cls, layer_sizes: Sequence[int], densities: Sequence[float],
               workers_per_rank: int, device: torch.device,
               group: Optional[dist.ProcessGroup] = None) -> "DataParallelLags":
        """Plans on `device`: one for the rank's workers (sparsify) and one for
        all workers of the job (aggregation only, so it binds the smaller
        workspace without candidate slots)."""
        from .plan import Plan
        world = dist.get_world_size(group)
        local = Plan(layer_sizes, densities, workers_per_rank, device=device)
        total = Plan(layer_sizes, densities, workers_per_rank * world, device=device,
                     aggregate_only=True)
        return cls(local, total, workers_per_rank, local.K, device, group)

    def exchange(self) -> None:
        """All-gather the local pick lists into rank-major global lists."""
        dist.all_gather_into_tensor(self.idx_all, self.idx_local, group=self.group)
        dist.all_gather_into_tensor(self.val_all, self.val_local, group=self.group)

    def step(self, grads: List[torch.Tensor], residuals: List[torch.Tensor], lr: float,
             dense_out: torch.Tensor, weights: torch.Tensor) -> None:
        """grads/residuals: this rank's `workers_per_rank` buffers of N."""
        if len(grads) != self.P_local or len(residuals) != self.P_local:
            raise ValueError(f"need {self.P_local} gradient and residual buffers per rank")
        self.local.sparsify(grads, residuals, lr, self.idx_local, self.val_local)
        self.exchange()
        self.total.aggregate_apply(self.idx_all, self.val_all, dense_out, weights)


class LayerwiseLags:
    """LAGS-SGD step with layer-wise pipelining.

    The layers are cut into buckets of consecutive layers (for instance by
    ``lags_merge_layers``).  The backward pass produces the last layers first,
    so the buckets are processed from the last to the first, each as soon as
    its gradients exist (``ready[b]``, an event the caller records after
    producing bucket b): sparsify the bucket (consecutive buckets on two
    alternating streams), start the all-gather of its pick lists without
    waiting, and aggregate + apply it on a third stream once the gather has
    landed.  A bucket's selection overlaps the next bucket's fused pass, its
    exchange overlaps the next buckets' sparsification, and all of it
    overlaps the rest of the backward pass ("Layer-wise Adaptive
    Gradient Sparsification ..." review, "proposed method": layer-wise
    selection lets communication start before back-propagation ends).

    Every layer is selected and aggregated exactly as by one whole-model plan,
    so the results equal ``DataParallelLags.step`` bit for bit, whatever the
    buckets.
    """

    def __init__(self, local_plans, total_plans, buckets, workers_per_rank: int,
                 device: torch.device, group: Optional[dist.ProcessGroup] = None):
        if len(local_plans) != len(buckets) or len(total_plans) != len(buckets):
            raise ValueError("one local and one total plan per bucket")
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = torch.device(device)
        self.buckets = [(int(a), int(b)) for a, b in buckets]
        self.local = list(local_plans)
        self.total = list(total_plans)
        self.P_local = int(workers_per_rank)
        self.P_total = self.P_local * self.world
        self.idx_local, self.val_local, self.idx_all, self.val_all = [], [], [], []
        for plan in self.local:
            n = self.P_local * plan.K
            self.idx_local.append(torch.empty(n, dtype=torch.int32, device=device))
            self.val_local.append(torch.empty(n, dtype=torch.float32, device=device))
            self.idx_all.append(torch.empty(n * self.world, dtype=torch.int32, device=device))
            self.val_all.append(torch.empty(n * self.world, dtype=torch.float32, device=device))
        cuda = self.device.type == "cuda"
        self.agg_stream = torch.cuda.Stream(device=self.device) if cuda else None
        # consecutive buckets sparsify on alternating streams, so one bucket's
        # (latency-bound) selection overlaps the next bucket's fused pass
        self.sp_streams = ([torch.cuda.Stream(device=self.device) for _ in range(2)]
                           if cuda else None)

    @classmethod
    def create(cls, layer_sizes: Sequence[int], densities: Sequence[float],
               workers_per_rank: int, buckets: Sequence[Tuple[int, int]],
               device: torch.device,
               group: Optional[dist.ProcessGroup] = None) -> "LayerwiseLags":
        """Range plans on `device`, one pair per bucket of layers."""
        from .plan import Plan
        world = dist.get_world_size(group)
        check_buckets(buckets, len(layer_sizes))
        local = [Plan(layer_sizes, densities, workers_per_rank, device=device, layer_range=b)
                 for b in buckets]
        total = [Plan(layer_sizes, densities, workers_per_rank * world, device=device,
                      layer_range=b, aggregate_only=True) for b in buckets]
        return cls(local, total, buckets, workers_per_rank, device, group)

    def step(self, grads: List[torch.Tensor], residuals: List[torch.Tensor], lr: float,
             dense_out: torch.Tensor, weights: torch.Tensor, ready=None) -> None:
        """grads/residuals: this rank's `workers_per_rank` whole-model buffers.
        ready: None, or one CUDA event per bucket (forward order) after which
        that bucket's gradients are complete."""
        if len(grads) != self.P_local or len(residuals) != self.P_local:
            raise ValueError(f"need {self.P_local} gradient and residual buffers per rank")
        if ready is not None and len(ready) != len(self.buckets):
            raise ValueError("one ready event per bucket")
        cuda = self.agg_stream is not None
        main = torch.cuda.current_stream(self.device) if cuda else None
        if cuda:
            # inputs, dense and weights are written on `main` before this step
            for st in (self.agg_stream, *self.sp_streams):
                st.wait_stream(main)
        for n, b in enumerate(reversed(range(len(self.buckets)))):
            sp = self.sp_streams[n % 2] if cuda else None
            if ready is not None and ready[b] is not None:
                sp.wait_event(ready[b])
            with torch.cuda.stream(sp) if cuda else _nullctx():
                self.local[b].sparsify(grads, residuals, lr, self.idx_local[b],
                                       self.val_local[b])
                # NCCL orders the gathers by issue order and waits for `sp`
                works = [dist.all_gather_into_tensor(self.idx_all[b], self.idx_local[b],
                                                     group=self.group, async_op=True),
                         dist.all_gather_into_tensor(self.val_all[b], self.val_local[b],
                                                     group=self.group, async_op=True)]
            if cuda:
                with torch.cuda.stream(self.agg_stream):
                    for w in works:
                        w.wait()  # the aggregation stream waits; the host does not
                    self.total[b].aggregate_apply(self.idx_all[b], self.val_all[b],
                                                  dense_out, weights)
            else:
                for w in works:
                    w.wait()
                self.total[b].aggregate_apply(self.idx_all[b], self.val_all[b], dense_out,
                                              weights)
        if cuda:
            # the next step reuses the pick buffers and reads dense/weights
            for st in (self.agg_stream, *self.sp_streams):
                main.wait_stream(st)


class DenseSgd:
    """Dense S-SGD over `world` ranks x `workers_per_rank` workers, the
    baseline of the LAGS review's comparisons: every rank sums its workers'
    fl(lr g) in worker order (``lags_dense_sum``), the ranks all-reduce the
    sums (NCCL, over NVLink), and every rank divides by the job's worker count
    and updates its weights (``lags_dense_finish``).  With one rank the result
    is the LAGS step at density 1, bit for bit; with more, the all-reduce adds
    the ranks' sums in its own order.  The message is the whole gradient,
    4 N bytes per rank, against 8 K bytes per worker for LAGS."""

    def __init__(self, kernels, N: int, workers_per_rank: int, device: torch.device,
                 group: Optional[dist.ProcessGroup] = None):
        self.kernels = kernels
        self.group = group
        self.world = dist.get_world_size(group)
        self.N = int(N)
        self.P_local = int(workers_per_rank)
        self.P_total = self.P_local * self.world
        self.sum = torch.empty(self.N, dtype=torch.float32, device=device)

    @classmethod
    def create(cls, N: int, workers_per_rank: int, device: torch.device,
               group: Optional[dist.ProcessGroup] = None) -> "DenseSgd":
        from .plan import DenseKernels
        return cls(DenseKernels(N, device), N, workers_per_rank, device, group)

    def step(self, grads: List[torch.Tensor], lr: float, dense_out: torch.Tensor,
             weights: torch.Tensor) -> None:
        if len(grads) != self.P_local:
            raise ValueError(f"need {self.P_local} gradient buffers per rank")
        self.kernels.sum(grads, lr, self.sum)
        if self.world > 1:
            dist.all_reduce(self.sum, op=dist.ReduceOp.SUM, group=self.group)
        self.kernels.finish(self.sum, self.P_total, dense_out, weights)


class _nullctx:
    def __enter__(self):
        return None

    def __exit__(self, *exc):
        return False


def capture_step(step, *args, **kwargs):
    """Capture one call of ``step(*args, **kwargs)`` (a LAGS step on fixed
    buffers: ``DataParallelLags.step`` or ``LayerwiseLags.step``) in a CUDA
    graph and return it; ``graph.replay()`` then runs the same step without
    host work per kernel or per bucket.  Run one eager step first, so that the
    NCCL communicators exist.  Release the graphs before destroying the
    process group."""
    dev = torch.cuda.current_device()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(graph, stream=side):
        step(*args, **kwargs)
    torch.cuda.current_stream(dev).wait_stream(side)
    return graph


def check_buckets(buckets: Sequence[Tuple[int, int]], num_layers: int) -> None:
    """Buckets must cover layers 0..num_layers-1 in order, without gaps."""
    at = 0
    for a, b in buckets:
        if a != at or b <= a:
            raise ValueError(f"buckets must partition the layers in order, got {list(buckets)}")
        at = b
    if at != num_layers:
        raise ValueError(f"buckets cover {at} of {num_layers} layers")
