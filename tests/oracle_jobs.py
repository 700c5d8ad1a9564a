"""Oracle replays of single large layers, run in worker processes (test
infrastructure).  Each job generates one worker's gradients of one layer on
the host and runs the oracle over the first steps of the workload, carrying
the residual; layers are independent, so this is exact.  The pool uses the
spawn start method: a process forked after the parent touched the GPU could
hang."""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os
from typing import Dict, List, Sequence, Tuple

import numpy as np

F32 = np.float32


def worker_layer_steps(wname: str, layer: int, p: int, steps: int):
    """[(idx[k] uint32, val[k] f32, residual[d] f32)] for steps 0..steps-1 of
    worker p on one layer of the named workload, from a zero residual."""
    import oracle.lags_oracle as lo
    import synth
    from synth.configs import WORKLOADS
    w = WORKLOADS[wname]
    off, d = w.offsets[layer], w.sizes[layer]
    k = lo.k_of(d, w.densities[layer])
    res = np.zeros(d, dtype=F32)
    out = []
    for s in range(steps):
        g = synth.layer_grads_host(w, p, s, layer)
        idx, val, new = lo.sparsify_layer(off, k, [g], [res], w.lr)
        res = new[0]
        out.append((idx[0].copy(), val[0].copy(), res.copy()))
    return out


def pool(jobs: int, bytes_per_job: int) -> cf.ProcessPoolExecutor:
    """A spawn pool of at most `jobs` processes, fewer when host memory or
    cores are short (each job holds about bytes_per_job)."""
    n = min(jobs, os.cpu_count() or 1)
    try:
        import psutil
        n = min(n, max(1, int(psutil.virtual_memory().available * 0.6) // max(bytes_per_job, 1)))
    except Exception:  # pragma: no cover
        pass
    return cf.ProcessPoolExecutor(max_workers=max(1, n), mp_context=mp.get_context("spawn"))


def submit_layers(ex: cf.ProcessPoolExecutor, wname: str, layers: Sequence[int],
                  workers: Sequence[int], steps: int) -> Dict[Tuple[int, int], cf.Future]:
    """One job per (layer, worker); largest layers first."""
    from synth.configs import WORKLOADS
    w = WORKLOADS[wname]
    order = sorted(layers, key=lambda l: -w.sizes[l])
    return {(l, p): ex.submit(worker_layer_steps, wname, l, p, steps)
            for l in order for p in workers}


def layer_history(futures: Dict[Tuple[int, int], cf.Future], wname: str, layer: int,
                  P: int) -> List[tuple]:
    """Per step (idx [P,k], val [P,k], residuals [P] list, dense [d], weights
    [d]) of one layer, all P workers' jobs combined (weights start at +0)."""
    import oracle.lags_oracle as lo
    from synth.configs import WORKLOADS
    w = WORKLOADS[wname]
    off, d = w.offsets[layer], w.sizes[layer]
    per = [futures[(layer, p)].result() for p in range(P)]
    wt = np.zeros(d, dtype=F32)
    hist = []
    for s in range(len(per[0])):
        idx = np.stack([per[p][s][0] for p in range(P)])
        val = np.stack([per[p][s][1] for p in range(P)])
        dense = lo.aggregate_layer(off, d, idx, val)
        wt = lo.apply_update(wt, dense)
        hist.append((idx, val, [per[p][s][2] for p in range(P)], dense, wt.copy()))
    return hist
