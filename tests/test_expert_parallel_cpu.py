"""The multi-GPU forms on CPU: the exchange plan, the parameter slicing, and
the whole choreographies (`ep_forward`: experts split over the ranks;
`sharded_forward`: every expert's hidden units split over the ranks) on two
and four gloo ranks, with the float64 oracle standing in for the kernels.
Each rank's output must equal the one-device layer with all experts on the
same tokens (the forms' defining property), through drops, skewed routing
that leaves a rank with no rows to serve, and capacity 0."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_45_b200 import expert_parallel as ep
from mixture_experts_layer_45_b200 import workloads as wl
from oracle import moe_ref


# ---------------------------------------------------------------------------
# the plan
# ---------------------------------------------------------------------------

def test_expert_range_and_splits():
    assert ep.expert_range(8, 2, 1) == (4, 8)
    with pytest.raises(ValueError):
        ep.expert_range(6, 4, 0)
    offsets = np.array([0, 3, 3, 7, 9, 9, 10, 14, 20])          # 8 experts, 20 rows
    np.testing.assert_array_equal(ep.dest_counts(offsets, 8, 4), [[3, 0], [4, 2], [0, 1], [4, 6]])
    assert ep.send_splits(offsets, 8, 4) == [3, 6, 1, 10]
    assert ep.send_splits(offsets, 8, 1) == [20]


def test_received_expert_ids():
    rc = np.array([[2, 0, 1], [0, 3, 1]])                        # from 2 sources, 3 local experts
    np.testing.assert_array_equal(ep.received_expert_ids(rc), [0, 0, 2, 1, 1, 1, 2])
    assert ep.received_expert_ids(np.zeros((2, 3), np.int64)).size == 0


def test_regroup_is_the_stable_dispatch_of_the_received_rows():
    """Grouping the received rows by local expert with the plain dispatch
    keeps, inside each expert, the source-rank order, then the sender's."""
    rng = np.random.default_rng(3)
    rc = rng.integers(0, 5, size=(3, 4))
    ids = ep.received_expert_ids(rc)
    d = moe_ref.dispatch(ids.reshape(-1, 1), 4, -1)
    src = np.repeat(np.repeat(np.arange(3), 4), rc.reshape(-1))
    pos = np.arange(ids.size)
    for e in range(4):
        rows = d["perm"][d["offsets"][e]:d["offsets"][e + 1]]
        assert list(rows) == sorted(rows, key=lambda a: (src[a], pos[a]))
        assert (ids[rows] == e).all()


# ---------------------------------------------------------------------------
# the choreography on gloo ranks, oracle steps
# ---------------------------------------------------------------------------

class OracleSteps:
    """route / dispatch / ffn / combine by the float64 oracle (test only);
    gates are rounded to float32 as the exchanged row gates are."""

    def __init__(self, inp, k, e0, e1):
        self.inp, self.k = inp, k
        self.local = {key: inp[key][e0:e1] for key in ("w1", "b1", "w2", "b2")}

    def route(self, x):
        r = moe_ref.route(x.numpy(), self.inp["w_router"], self.k, self.inp.get("logit_bias"))
        return (torch.from_numpy(r["topk_idx"].astype(np.int32)),
                torch.from_numpy(r["topk_gate"].astype(np.float32)))

    def dispatch(self, idx, gate, T, k, E, capacity, x):
        d = moe_ref.dispatch(idx.numpy(), E, capacity)
        perm = d["perm"]
        return {"offsets": torch.from_numpy(d["offsets"].astype(np.int32)),
                "slot_of": torch.from_numpy(d["slot_of"].astype(np.int32)),
                "row_gate": torch.from_numpy(gate.numpy().reshape(-1)[perm].astype(np.float32)),
                "xp": torch.from_numpy(x.numpy()[perm // k])}

    def ffn(self, xp, offsets, row_gate, rows):
        return torch.from_numpy(moe_ref.grouped_ffn(xp.numpy(), offsets.numpy(), self.local,
                                                    row_gate.numpy().astype(np.float64)))

    def combine(self, yp, slot_of, T, k):
        return torch.from_numpy(moe_ref.combine(yp.numpy(), slot_of.numpy(), T, k, None))


def one_device_reference(x, inp, k, E, capacity):
    r = moe_ref.route(x, inp["w_router"], k, inp.get("logit_bias"))
    gates = r["topk_gate"].astype(np.float32).astype(np.float64)
    d = moe_ref.dispatch(r["topk_idx"], E, capacity)
    return moe_ref.moe_forward(x, inp, r["topk_idx"], gates, d["slot_of"])


def case_inputs(case):
    T, d, ff, E, k, cap, world, skew = case
    inp = wl.draw_custom(11, T=T * world, d=d, ff=ff, E=E, dtype="f32", router_std=0.5)
    if skew:
        # every token prefers rank 0's experts: the other ranks serve nothing
        el = E // world
        inp["logit_bias"] = np.where(np.arange(E) < el, 50.0, 0.0).astype(np.float32)
    return inp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, d, ff, E, k, cap, _, _ = case
        inp = case_inputs(case)
        x = inp["x"][rank * T:(rank + 1) * T].astype(np.float64)
        e0, e1 = ep.expert_range(E, world, rank)
        out = ep.ep_forward(torch.from_numpy(x), OracleSteps(inp, k, e0, e1), E, k, cap)
        ref = one_device_reference(x, inp, k, E, cap)
        scale = max(float(np.abs(ref).max()), 1e-30)
        q.put((rank, float(np.abs(out.numpy() - ref).max()) / scale, float(np.abs(out.numpy()).max())))
    finally:
        dist.destroy_process_group()


CASES = [
    # T per rank, d, ff, E, k, capacity, ranks, skewed
    (40, 16, 24, 8, 2, -1, 2, False),
    (60, 16, 24, 4, 1, 9, 2, False),       # drops
    (30, 8, 16, 8, 2, 5, 4, False),        # four ranks, two experts each, drops
    (32, 8, 16, 4, 2, -1, 2, True),        # rank 1 receives no rows
    (20, 8, 16, 4, 1, 0, 2, False),        # capacity 0: nothing kept anywhere
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c[0]}-E{c[3]}-k{c[4]}-cap{c[5]}-G{c[6]}"
                         + ("-skew" if c[7] else ""))
def test_ep_forward_equals_one_device_layer(case):
    world = case[6]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, mx in res:
        if case[5] == 0:
            assert mx == 0.0                # every slot dropped: zero output
        else:
            assert err <= 1e-12, (rank, err)


# ---------------------------------------------------------------------------
# every expert's hidden units split over the ranks (MoEShard's decomposition)
# ---------------------------------------------------------------------------

def test_hidden_range():
    assert ep.hidden_range(64, 4, 3) == (48, 64)
    with pytest.raises(ValueError):
        ep.hidden_range(48, 4, 0)           # slices of 12: not a multiple of 8


def cpu_params(inp):
    from mixture_experts_layer_45_b200 import _lib
    from mixture_experts_layer_45_b200.layer import MoEParams
    return MoEParams.from_arrays(inp, _lib.MOE_F32, "cpu")


def test_shard_helpers_slice_the_parameters():
    inp = wl.draw_custom(5, T=8, d=16, ff=32, E=4, dtype="f32")
    p = cpu_params(inp)
    w1, b1, w2, b2 = ep.shard_experts(p, 1, 2)
    np.testing.assert_array_equal(w1.numpy(), inp["w1"][2:4])
    np.testing.assert_array_equal(w2.numpy(), inp["w2"][2:4])
    np.testing.assert_array_equal(b2.numpy(), inp["b2"][2:4])
    for rank in range(4):
        w1, b1, w2, b2 = ep.shard_hidden(p, rank, 4)
        f0, f1 = 8 * rank, 8 * rank + 8
        np.testing.assert_array_equal(w1.numpy(), inp["w1"][:, f0:f1])
        np.testing.assert_array_equal(b1.numpy(), inp["b1"][:, f0:f1])
        np.testing.assert_array_equal(w2.numpy(), inp["w2"][:, :, f0:f1])
        np.testing.assert_array_equal(b2.numpy(), inp["b2"] if rank == 0 else 0.0)
        assert w1.is_contiguous() and w2.is_contiguous()


class OracleSliceSteps(OracleSteps):
    """The oracle steps on this rank's hidden-unit slice of every expert, as
    shard_hidden cuts it (b2 on rank 0 only)."""

    def __init__(self, inp, k, rank, world):
        self.inp, self.k = inp, k
        w1, b1, w2, b2 = ep.shard_hidden(cpu_params(inp), rank, world)
        self.local = {"w1": w1.numpy(), "b1": b1.numpy(), "w2": w2.numpy(), "b2": b2.numpy()}


def _sharded_rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, d, ff, E, k, cap, _, _ = case
        inp = case_inputs(case)
        x = inp["x"][:T].astype(np.float64)              # the same batch on every rank
        out = ep.sharded_forward(torch.from_numpy(x), OracleSliceSteps(inp, k, rank, world), E, k, cap)
        ref = one_device_reference(x, inp, k, E, cap)
        scale = max(float(np.abs(ref).max()), 1e-30)
        q.put((rank, float(np.abs(out.numpy() - ref).max()) / scale, float(np.abs(out.numpy()).max())))
    finally:
        dist.destroy_process_group()


SHARD_CASES = [
    # T, d, ff, E, k, capacity, ranks, skewed
    (40, 16, 32, 4, 2, -1, 2, False),
    (50, 16, 64, 4, 1, 7, 4, False),       # drops, four slices of 16 hidden units
    (32, 8, 16, 4, 2, -1, 2, True),        # skewed routing changes nothing in the split
    (20, 8, 16, 4, 1, 0, 2, False),        # capacity 0
]


@pytest.mark.parametrize("case", SHARD_CASES, ids=lambda c: f"T{c[0]}-ff{c[2]}-k{c[4]}-cap{c[5]}-G{c[6]}"
                         + ("-skew" if c[7] else ""))
def test_sharded_forward_equals_one_device_layer(case):
    world = case[6]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, mx in res:
        if case[5] == 0:
            assert mx == 0.0
        else:
            assert err <= 1e-12, (rank, err)
