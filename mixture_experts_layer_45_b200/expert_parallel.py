"""Expert parallelism across GPUs: G ranks, each holding E/G of the experts.

The pages' serving setting: the experts are spread over the GPUs and each
token's hidden vector travels to the GPUs of its chosen experts and back
(blog "MoE Parallelism for Inference", sections "Expert Parallelism" and
"Communication Overhead"; notebook "Mixture-of-experts and expert
parallelism", section "What", the all-to-all of dispatch and combine).

Rank r holds the experts [r*E/G, (r+1)*E/G) (contiguous blocks), the router
weight (replicated) and its own batch of tokens.  One forward pass:

  1. route its tokens and dispatch them by expert with its own capacity
     (the per-batch slot budget applies to each rank's batch, as in GShard's
     per-group capacity); the grouped rows are expert-major, so the rows
     for rank q are one contiguous block;
  2. exchange the per-(rank, expert) kept counts (all-to-all), then the
     rows and their gates (all-to-all-v);
  3. regroup the received rows by local expert (a stable dispatch keyed by
     the local expert: source rank, then the sender's row order), run the
     grouped FFN with the received gates, and put the rows back in receive
     order;
  4. send the rows back (all-to-all-v) and sum each token's rows (combine,
     gates already applied by the owning rank).

Every row sees the arithmetic it would see on one GPU that holds all the
experts and runs the same rank's batch, so each rank's output equals the
single-GPU layer on its own tokens (routing, drops and gates exactly; the
expert rows up to the grouped FFN's tiling).  The collectives are
torch.distributed all-to-alls (NCCL on GPUs); the split sizes are host
lists, so a pass reads the offsets and the received counts back to the
host once each.  Shared experts and overflow rerouting are not part of
this path.

A second form, `ShardedExpertsMoE`, splits every expert instead of the
set of experts (the MoEShard pages, abstract: each expert's weight matrices
cut by rows and by columns across the GPUs, so that every GPU does an
equal share of every expert whatever the routing skew and no token is
dropped for balance).  Rank g holds the hidden
units [g*ff/G, (g+1)*ff/G) of every expert: those columns of fc1 (rows of
W1 and b1) and the matching rows of fc2 (columns of W2); b2 lives on rank
0.  Every rank routes and dispatches the same replicated batch, runs the
grouped FFN on its slice (GELU acts on each hidden unit alone, so the
slices' fc2 partial products sum exactly to the full one), and one
all-reduce sums the gated partial rows before the combine.

`ep_forward` / `sharded_forward` are the choreographies over four step
operations; the product binds them to libmoe's kernels (`LibmoeSteps`),
and the CPU tests bind the same choreographies to the float64 oracle to
check the exchanges with gloo.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import _lib
from .layer import TORCH_DTYPE


# ---------------------------------------------------------------------------
# the exchange plan (host side, pure)
# ---------------------------------------------------------------------------

def expert_range(E: int, G: int, rank: int) -> Tuple[int, int]:
    """[first, last) expert of `rank` when E experts are split over G ranks."""
    if G < 1 or E % G != 0:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    el = E // G
    return rank * el, (rank + 1) * el


def dest_counts(offsets: np.ndarray, E: int, G: int) -> np.ndarray:
    """Kept rows per (destination rank, its local expert), [G, E/G], from
    the expert-major grouped-row offsets [E+1]."""
    expert_range(E, G, 0)
    offsets = np.asarray(offsets, np.int64)
    return np.diff(offsets).reshape(G, E // G).astype(np.int32)


def send_splits(offsets: np.ndarray, E: int, G: int) -> List[int]:
    """Rows for each destination rank: the contiguous blocks of the
    expert-major grouped rows."""
    return [int(v) for v in dest_counts(offsets, E, G).sum(axis=1)]


def hidden_range(ff: int, G: int, rank: int) -> Tuple[int, int]:
    """[first, last) hidden unit of every expert held by `rank` when each
    expert's ff hidden units are split over G ranks (each slice a multiple
    of 8, the grouped FFN's granularity)."""
    if G < 1 or ff % G != 0 or (ff // G) % 8 != 0:
        raise ValueError(f"ff = {ff} does not split into {G} slices of a multiple of 8")
    f = ff // G
    return rank * f, (rank + 1) * f


def received_expert_ids(recv_counts: np.ndarray) -> np.ndarray:
    """Local expert of each received row, in receive order (source rank,
    then the sender's expert-major order), from the received counts [G, E/G]."""
    rc = np.asarray(recv_counts, np.int64)
    G, el = rc.shape
    ids = np.repeat(np.tile(np.arange(el, dtype=np.int32), G), rc.reshape(-1))
    return ids.astype(np.int32)


# ---------------------------------------------------------------------------
# the collectives
# ---------------------------------------------------------------------------

class Exchange:
    """The two collectives of the multi-GPU forms on a torch.distributed
    group: all-to-all(-v) and a sum all-reduce.

    A backend that moves device tensors (NCCL) gets them as they are.  A
    backend that moves host tensors only (gloo) gets each exchanged tensor
    copied to host memory and the result copied back, so the same forms run
    over gloo, e.g. several processes sharing one GPU."""

    def __init__(self, group=None, host_staged=None):
        self.group = group
        if host_staged is None:
            host_staged = dist.get_backend(group) == "gloo"
        self.host_staged = host_staged

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits=None, in_splits=None) -> None:
        if not (self.host_staged and (out.is_cuda or inp.is_cuda)):
            dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
            return
        h_out = torch.empty(out.shape, dtype=out.dtype)
        dist.all_to_all_single(h_out, inp.cpu(), out_splits, in_splits, group=self.group)
        out.copy_(h_out)

    def all_reduce_sum(self, t: torch.Tensor) -> None:
        if not (self.host_staged and t.is_cuda):
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
            return
        h = t.cpu()
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=self.group)
        t.copy_(h)


# ---------------------------------------------------------------------------
# the choreography
# ---------------------------------------------------------------------------

def ep_forward(x: torch.Tensor, steps, E: int, k: int, capacity: int, group=None,
               exchange: Exchange = None) -> torch.Tensor:
    """One expert-parallel forward pass of this rank's tokens x [T, d].

    `steps` provides route / dispatch / ffn / combine (see LibmoeSteps);
    the collectives run on `group` (default: the world) through `exchange`
    (default: Exchange(group))."""
    G = dist.get_world_size(group)
    xc = exchange if exchange is not None else Exchange(group)
    T, d = x.shape
    dev = x.device
    el = E // G
    expert_range(E, G, 0)

    # 1. route and dispatch this rank's batch (its own capacity)
    idx, gate = steps.route(x)
    dsp = steps.dispatch(idx, gate, T, k, E, capacity, x)
    offs = dsp["offsets"].cpu().numpy()
    R = int(offs[E])
    splits = send_splits(offs, E, G)

    # 2. counts, then rows and gates
    send_c = torch.from_numpy(dest_counts(offs, E, G).reshape(-1)).to(dev)
    recv_c = torch.empty(G * el, dtype=torch.int32, device=dev)
    xc.all_to_all(recv_c, send_c)
    rc = recv_c.cpu().numpy().reshape(G, el)
    recv_splits = [int(v) for v in rc.sum(axis=1)]
    Rr = sum(recv_splits)
    xr = torch.empty((Rr, d), dtype=x.dtype, device=dev)
    gr = torch.empty((Rr,), dtype=torch.float32, device=dev)
    xc.all_to_all(xr, dsp["xp"][:R].contiguous(), recv_splits, splits)
    xc.all_to_all(gr, dsp["row_gate"][:R].contiguous(), recv_splits, splits)

    # 3. the local experts on the received rows
    yr = torch.empty((Rr, d), dtype=x.dtype, device=dev)
    if Rr > 0:
        ids = torch.from_numpy(received_expert_ids(rc)).to(dev).reshape(Rr, 1)
        loc = steps.dispatch(ids, gr.reshape(Rr, 1), Rr, 1, el, -1, xr)
        yp_loc = steps.ffn(loc["xp"], loc["offsets"], loc["row_gate"], Rr)
        yr = steps.combine(yp_loc, loc["slot_of"], Rr, 1)     # back to receive order

    # 4. rows home, then each token's sum (a token whose slots were all
    # dropped sums nothing: 0)
    yb = torch.empty((R, d), dtype=x.dtype, device=dev)
    xc.all_to_all(yb, yr, splits, recv_splits)
    if R == 0:
        yb = torch.zeros((1, d), dtype=x.dtype, device=dev)
    return steps.combine(yb, dsp["slot_of"], T, k)


def sharded_forward(x: torch.Tensor, steps, E: int, k: int, capacity: int, group=None,
                    exchange: Exchange = None) -> torch.Tensor:
    """One forward pass of the replicated batch x [T, d] with every expert's
    hidden units split over the ranks of `group`: each rank's grouped FFN
    gives gated partial rows from its slice, an all-reduce sums them, and
    the combine (gates already applied) gives the replicated output."""
    xc = exchange if exchange is not None else Exchange(group)
    T, d = x.shape
    idx, gate = steps.route(x)
    dsp = steps.dispatch(idx, gate, T, k, E, capacity, x)
    R = int(dsp["offsets"][E].item())
    if R == 0:
        return steps.combine(torch.zeros((1, d), dtype=x.dtype, device=x.device), dsp["slot_of"], T, k)
    yp = steps.ffn(dsp["xp"], dsp["offsets"], dsp["row_gate"], T * k)
    part = yp[:R]
    xc.all_reduce_sum(part)
    return steps.combine(yp, dsp["slot_of"], T, k)


# ---------------------------------------------------------------------------
# the step operations on libmoe's kernels
# ---------------------------------------------------------------------------

class LibmoeSteps:
    """route / dispatch / ffn / combine through the C ABI, on torch's current
    stream.  Holds the router weight (all E experts) and this rank's E/G
    experts' parameters [E/G, ...]."""

    def __init__(self, w_router, logit_bias, w1, b1, w2, b2, dtype: int, k: int):
        self.w_router, self.logit_bias = w_router, logit_bias
        self.w1, self.b1, self.w2, self.b2 = w1, b1, w2, b2
        self.dtype = dtype
        self.k = k
        self.E = w_router.shape[0]
        self.el, self.ff, self.d = w1.shape

    def route(self, x):
        T, d = x.shape
        k = self.k
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        gate = torch.empty((T, k), dtype=torch.float32, device=x.device)
        _lib.moe_router_topk(x, self.w_router, self.logit_bias, T, d, self.E, k, self.dtype, idx, gate, None)
        return idx, gate

    def dispatch(self, idx, gate, T, k, E, capacity, x):
        dev = x.device
        A = T * k
        out = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
               "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
               "perm": torch.empty(max(A, 1), dtype=torch.int32, device=dev),
               "slot_of": torch.empty(max(A, 1), dtype=torch.int32, device=dev),
               "row_gate": torch.empty(max(A, 1), dtype=torch.float32, device=dev),
               "xp": torch.empty((max(A, 1), x.shape[1]), dtype=x.dtype, device=dev)}
        n = _lib.moe_dispatch_workspace_size(T, k, E)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
        _lib.moe_dispatch(idx, gate, T, k, E, capacity, out["counts"], out["offsets"], out["perm"],
                          out["slot_of"], None, out["row_gate"], x, out["xp"], x.shape[1], self.dtype, ws, n)
        return out

    def ffn(self, xp, offsets, row_gate, rows):
        h = torch.empty((rows, self.ff), dtype=xp.dtype, device=xp.device)
        yp = torch.empty((rows, self.d), dtype=xp.dtype, device=xp.device)
        _lib.moe_grouped_ffn(xp, offsets, rows, self.el, self.d, self.ff, self.w1, self.b1, self.w2, self.b2,
                             row_gate, h, yp, self.dtype)
        return yp

    def combine(self, yp, slot_of, T, k):
        out = torch.empty((T, self.d), dtype=yp.dtype, device=yp.device)
        _lib.moe_combine(yp, slot_of, None, T, k, self.d, self.dtype, out)
        return out


class ExpertParallelMoE:
    """One MoE layer whose experts are split over the ranks of `group`.

    w_router [E, d] (and logit_bias [E]) on every rank; w1 [E/G, ff, d],
    b1 [E/G, ff], w2 [E/G, d, ff], b2 [E/G, d]: this rank's experts
    (expert_range(E, G, rank)).  capacity applies to each rank's batch."""

    def __init__(self, w_router, logit_bias, w1, b1, w2, b2, dtype: int, k: int, capacity: int = -1,
                 group=None):
        G = dist.get_world_size(group)
        E = w_router.shape[0]
        expert_range(E, G, 0)
        if w1.shape[0] != E // G:
            raise ValueError(f"rank holds {w1.shape[0]} experts, expected {E // G}")
        if TORCH_DTYPE[dtype] != w1.dtype:
            raise ValueError("parameter dtype does not match `dtype`")
        self.steps = LibmoeSteps(w_router, logit_bias, w1, b1, w2, b2, dtype, k)
        self.E, self.k, self.capacity, self.group = E, k, capacity, group

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if not x.is_cuda:
            raise ValueError("x must be a CUDA tensor")
        return ep_forward(x, self.steps, self.E, self.k, self.capacity, self.group)

    __call__ = forward


class ShardedExpertsMoE:
    """One MoE layer with every expert's hidden units split over the ranks of
    `group` (the same batch on every rank, replicated output).

    w_router [E, d] (and logit_bias [E]) on every rank; this rank's slice
    (hidden_range(ff, G, rank)) of every expert: w1 [E, ff/G, d],
    b1 [E, ff/G], w2 [E, d, ff/G]; b2 [E, d] on rank 0 (zeros elsewhere, so
    the bias is added once)."""

    def __init__(self, w_router, logit_bias, w1, b1, w2, b2, dtype: int, k: int, capacity: int = -1,
                 group=None):
        if TORCH_DTYPE[dtype] != w1.dtype:
            raise ValueError("parameter dtype does not match `dtype`")
        if w1.shape[0] != w_router.shape[0]:
            raise ValueError("every rank holds a slice of every expert")
        self.steps = LibmoeSteps(w_router, logit_bias, w1, b1, w2, b2, dtype, k)
        self.E, self.k, self.capacity, self.group = w_router.shape[0], k, capacity, group

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if not x.is_cuda:
            raise ValueError("x must be a CUDA tensor")
        return sharded_forward(x, self.steps, self.E, self.k, self.capacity, self.group)

    __call__ = forward


def shard_hidden(params, rank: int, G: int):
    """This rank's hidden-unit slice of a full MoEParams' experts:
    (w1, b1, w2, b2), b2 zeroed except on rank 0."""
    f0, f1 = hidden_range(params.ff, G, rank)
    b2 = params.b2 if rank == 0 else torch.zeros_like(params.b2)
    return (params.w1[:, f0:f1].contiguous(), params.b1[:, f0:f1].contiguous(),
            params.w2[:, :, f0:f1].contiguous(), b2.contiguous())


def shard_experts(params, rank: int, G: int):
    """This rank's block of a full MoEParams' experts: (w1, b1, w2, b2)."""
    e0, e1 = expert_range(params.E, G, rank)
    return (params.w1[e0:e1].contiguous(), params.b1[e0:e1].contiguous(), params.w2[e0:e1].contiguous(),
            params.b2[e0:e1].contiguous())

