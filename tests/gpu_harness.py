"""Drives the CUDA path through the C ABI (via layer_wise_top_b200.Plan) and
checks it against the oracle and against full-size invariants (torch on the
GPU as an independent checker).  Test infrastructure."""
from __future__ import annotations

from typing import Callable, Iterable, List, Optional, Sequence

import numpy as np
import torch

import oracle.lags_oracle as lo

F32 = np.float32


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


class GpuRun:
    """Runs steps of sparsify -> aggregate -> apply on the GPU."""

    def __init__(self, sizes: Sequence[int], densities: Sequence[float], P: int, lr: float,
                 keep_prev: bool = False):
        from layer_wise_top_b200 import Plan
        self.plan = Plan(sizes, densities, P)
        self.P, self.lr = P, lr
        N, K = self.plan.N, self.plan.K
        dev = torch.device("cuda")
        self.grads = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(P)]
        self.res = [torch.zeros(N, dtype=torch.float32, device=dev) for _ in range(P)]
        self.idx, self.val = self.plan.empty_picks()
        self.dense = torch.empty(N, dtype=torch.float32, device=dev)
        self.weights = torch.zeros(N, dtype=torch.float32, device=dev)
        self.keep_prev = keep_prev
        self.prev: Optional[List[torch.Tensor]] = None

    def step(self, fused: bool = False) -> None:
        """One step; `fused` uses lags_aggregate_apply instead of
        lags_aggregate + lags_apply (the results must be identical)."""
        if self.keep_prev:
            self.prev = None  # drop the old copy first: full-size workloads fill the device
            self.prev = [r.clone() for r in self.res]
        self.plan.sparsify(self.grads, self.res, self.lr, self.idx, self.val)
        if fused:
            self.plan.aggregate_apply(self.idx, self.val, self.dense, self.weights)
        else:
            self.plan.aggregate(self.idx, self.val, self.dense)
            self.plan.apply(self.weights, self.dense)


def oracle_layer_steps(off: int, d: int, k: int, P: int, lr: float, steps: int,
                       grad_fn: Callable[[int, int], np.ndarray]):
    """Oracle history of one layer: grad_fn(p, s) -> that layer's gradient."""
    res = [np.zeros(d, dtype=F32) for _ in range(P)]
    w = np.zeros(d, dtype=F32)
    out = []
    for s in range(steps):
        grads = [grad_fn(p, s) for p in range(P)]
        idx, val, res = lo.sparsify_layer(off, k, grads, res, lr)
        dense = lo.aggregate_layer(off, d, idx, val)
        w = lo.apply_update(w, dense)
        out.append((idx, val, [r.copy() for r in res], dense, w.copy()))
    return out


def compare_layer(run: GpuRun, l: int, exp, where: str) -> None:
    """Bit-exact comparison of one layer's slices with an oracle step."""
    off, k, koff = run.plan.layers[l]
    d = run.plan.sizes[l]
    e_idx, e_val, e_res, e_dense, e_w = exp
    K = run.plan.K
    idx = u32(run.idx).reshape(run.P, K)[:, koff:koff + k]
    val = u32(run.val).reshape(run.P, K)[:, koff:koff + k]
    assert np.array_equal(idx, e_idx), f"{where}: indices differ"
    assert np.array_equal(val, e_val.view(np.uint32)), f"{where}: values differ"
    for p in range(run.P):
        r = u32(run.res[p][off:off + d])
        assert np.array_equal(r, e_res[p].view(np.uint32)), f"{where}: residual p={p}"
    assert np.array_equal(u32(run.dense[off:off + d]), e_dense.view(np.uint32)), \
        f"{where}: dense update"
    assert np.array_equal(u32(run.weights[off:off + d]), e_w.view(np.uint32)), \
        f"{where}: weights"


def check_invariants(run: GpuRun, workers: Iterable[int], check_dense: bool = True,
                     max_elems: int = 1 << 27) -> None:
    """Full-size properties that determine the result uniquely, checked for
    the given workers of every layer (workers in groups of up to `max_elems`
    layer elements, so whole layers are checked at once): the picks are
    ascending and inside the layer, each value is acc at its index, picked
    residuals are +0 and the others keep acc, every picked magnitude is >=
    every unpicked one, and among entries tied at the smallest picked
    magnitude the picked ones have the lowest indices.  The dense update is
    recomputed in worker order with one rounding per add."""
    assert run.prev is not None, "run with keep_prev=True"
    lr = torch.tensor(run.lr, dtype=torch.float32, device="cuda")
    K = run.plan.K
    idx_all = run.idx.view(run.P, K)
    val_all = run.val.view(run.P, K)
    workers = list(workers)
    i32 = torch.int32
    for l, (off, k, koff) in enumerate(run.plan.layers):
        d = run.plan.sizes[l]
        per = max(1, min(len(workers), max_elems // d))
        for g0 in range(0, len(workers), per):
            ws = workers[g0:g0 + per]
            # acc = prev + lr * g: two separate fp32 roundings
            a = torch.stack([run.prev[p][off:off + d] + lr * run.grads[p][off:off + d]
                             for p in ws])
            res = torch.stack([run.res[p][off:off + d] for p in ws])
            li = idx_all[ws, koff:koff + k].to(torch.int64) & 0xFFFFFFFF
            lv = val_all[ws, koff:koff + k]
            where = (l, ws)
            assert bool((li >= off).all() and (li < off + d).all()), (where, "range")
            if k > 1:
                assert bool((li[:, 1:] > li[:, :-1]).all()), (where, "ascending")
            loc = li - off
            assert torch.equal(lv.view(i32), torch.gather(a, 1, loc).view(i32)), (where, "val")
            mask = torch.zeros_like(a, dtype=torch.bool)
            mask.scatter_(1, loc, True)
            assert bool((res.view(i32)[mask] == 0).all()), (where, "zeroed")
            assert torch.equal(res.view(i32)[~mask], a.view(i32)[~mask]), (where, "residual")
            if k < d:
                mag = a.abs()
                inf = torch.tensor(float("inf"), device="cuda")
                tmin = torch.where(mask, mag, inf).amin(1, keepdim=True)
                umax = torch.where(mask, -inf, mag).amax(1, keepdim=True)
                assert bool((tmin >= umax).all()), (where, "magnitude")
                pos = torch.arange(d, device="cuda", dtype=torch.int64).expand_as(a)
                at_min = mag == tmin
                first_unpicked = torch.where(at_min & ~mask, pos, d).amin(1)
                last_picked = torch.where(at_min & mask, pos, -1).amax(1)
                assert bool((last_picked < first_unpicked).all()), (where, "tie order")
            del a, res, mask
    if check_dense:
        dense = torch.zeros(run.plan.N, dtype=torch.float32, device="cuda")
        for p in range(run.P):
            li = idx_all[p].to(torch.int64) & 0xFFFFFFFF
            dense[li] = dense[li] + val_all[p]
        dense = dense / torch.tensor(float(run.P), dtype=torch.float32, device="cuda")
        assert torch.equal(dense.view(torch.int32), run.dense.view(torch.int32)), "dense"


def check_layer_chunked(run: GpuRun, l: int, lr: float, chunk: int = 1 << 28) -> None:
    """The properties that fix layer l's top-k, checked on the GPU in chunks
    (for layers too large for the oracle or for whole-layer temporaries),
    for every worker: picks ascending and inside the layer, each value equal
    to acc at its index, picked residuals +0 and all others acc, every picked
    magnitude at least every unpicked one, ties to the lower index; and the
    dense update recomputed from the picks in worker order.  Needs
    keep_prev=True."""
    assert run.prev is not None, "run with keep_prev=True"
    off, k, koff = run.plan.layers[l]
    d = run.plan.sizes[l]
    K = run.plan.K
    lr_t = torch.tensor(lr, dtype=torch.float32, device="cuda")

    def bits(t):
        return t.view(torch.int32)

    for p in range(run.P):
        idx = run.idx[p * K + koff:p * K + koff + k].to(torch.int64) & 0xFFFFFFFF
        val = run.val[p * K + koff:p * K + koff + k]
        assert bool((idx[1:] > idx[:-1]).all()) and int(idx[0]) >= off
        assert int(idx[-1]) < off + d
        g, prev, res = run.grads[p], run.prev[p], run.res[p]
        assert torch.equal(bits(val), bits(prev[idx] + lr_t * g[idx])), f"values p={p}"
        assert int(bits(res[idx]).abs().max()) == 0, f"picked residuals p={p}"
        vmin = float(val.abs().min())
        top_unpicked, first_tie = 0.0, None
        for a in range(off, off + d, chunk):
            b = min(a + chunk, off + d)
            inside = (idx >= a) & (idx < b)
            sel = idx[inside] - a
            want = prev[a:b] + lr_t * g[a:b]
            want[sel] = 0.0
            assert torch.equal(bits(res[a:b]), bits(want)), f"residual p={p} chunk {a}"
            mag = want.abs()
            mag[sel] = -1.0
            top_unpicked = max(top_unpicked, float(mag.max()))
            ties = torch.nonzero(mag == vmin)
            if first_tie is None and ties.numel():
                first_tie = a + int(ties[0])
        assert vmin >= top_unpicked, f"p={p}: a picked magnitude is below an unpicked one"
        if first_tie is not None:
            assert first_tie > int(idx[val.abs() == vmin].max()), f"p={p}: tie order"
    # dense update: the workers' picks added in worker order from +0, one
    # rounding per add, then divided by P (positions nobody picked: +0)
    picks = []
    for p in range(run.P):
        picks.append((run.idx[p * K + koff:p * K + koff + k].to(torch.int64) & 0xFFFFFFFF,
                      run.val[p * K + koff:p * K + koff + k]))
    fP = torch.tensor(float(run.P), dtype=torch.float32, device="cuda")
    for a in range(off, off + d, chunk):
        b = min(a + chunk, off + d)
        acc = torch.zeros(b - a, dtype=torch.float32, device="cuda")
        for idx, val in picks:
            inside = (idx >= a) & (idx < b)
            sel = idx[inside] - a
            acc[sel] = acc[sel] + val[inside]
        assert torch.equal(bits(run.dense[a:b]), bits(acc / fP)), f"dense chunk {a}"


def same_bits_or_nan(got_u32, exp_f32):
    """Bitwise equality, except that a NaN matches any NaN: IEEE 754 leaves the
    payload and sign of an invalid operation's NaN (inf - inf) unspecified."""
    exp_u32 = exp_f32.view(np.uint32)
    got_f = got_u32.view(np.float32)
    both_nan = np.isnan(got_f) & np.isnan(exp_f32)
    return bool(np.all((got_u32 == exp_u32) | both_nan))


def run_full_compare(sizes, densities, P, lr, steps, grad_fn, expect_fallbacks=None):
    """Element-by-element parity of every output for `steps` steps."""
    run = GpuRun(sizes, densities, P, lr)
    hist = lo.run_workload(sizes, densities, P, lr, steps, grad_fn)
    total_fb = 0
    for s in range(steps):
        for p in range(P):
            run.grads[p].copy_(torch.from_numpy(grad_fn(p, s)))
        run.step(fused=s % 2 == 1)  # odd steps: lags_aggregate_apply
        flags, fb = run.plan.poll()
        assert flags == 0
        total_fb += fb
        e_idx, e_val, e_res, e_dense, e_w = hist[s]
        K = run.plan.K
        assert np.array_equal(u32(run.idx).reshape(P, K), e_idx), f"step {s}: idx"
        assert np.array_equal(u32(run.val).reshape(P, K), e_val.view(np.uint32)), f"step {s}: val"
        for p in range(P):
            assert np.array_equal(u32(run.res[p]), e_res[p].view(np.uint32)), f"step {s}: res {p}"
        assert same_bits_or_nan(u32(run.dense), e_dense), f"step {s}: dense"
        assert same_bits_or_nan(u32(run.weights), e_w), f"step {s}: weights"
    if expect_fallbacks is not None:
        assert expect_fallbacks(total_fb), total_fb
    return total_fb


def synth_grad_fn(w):
    """grad_fn(p, s) of a workload: host gradients, generated once each."""
    import synth
    cache = {}

    def fn(p, s):
        if (p, s) not in cache:
            cache[(p, s)] = synth.worker_grads_host(w, p, s)
        return cache[(p, s)]
    return fn
