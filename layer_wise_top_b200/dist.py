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

from typing import List, Optional, Sequence

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
        all workers of the job (aggregation)."""
        from .plan import Plan
        world = dist.get_world_size(group)
        local = Plan(layer_sizes, densities, workers_per_rank, device=device)
        total = Plan(layer_sizes, densities, workers_per_rank * world, device=device)
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
