"""The multi-GPU forms on the GPU kernels: expert parallelism (`ExpertParallelMoE`:
each rank holds E/G experts; blog "MoE Parallelism for Inference", sections
"Expert Parallelism" and "Communication Overhead") and the MoEShard
row/column decomposition (`ShardedExpertsMoE`: every rank holds a slice of
every expert's hidden units; the MoEShard abstract), with every step in
libmoe's kernels through the C ABI.

Two gloo ranks run as two processes that share the one GPU: their kernels
never wait on one another, and every exchange goes through host memory
(`Exchange` stages device tensors for gloo), so no peer memory, no NCCL and
no multicast is involved.  Each rank's output must equal the float64
one-device layer (all experts) on that rank's tokens, on the GPU's own
routing: max-norm relative error <= 1e-4 (fp32) or 2e-2 (bf16); tokens
whose every assignment was dropped give exactly 0.  The cases cover drops,
k = 1 and k = 2, and a rank that receives no rows.
"""
import os
import socket
import traceback

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

WORLD = 2

# name: T per rank, d, ff, E, k, capacity factor (None: no limit), dtype, skewed
EP_CASES = {
    "ep-k2-f32": (300, 64, 192, 8, 2, None, "f32", False),
    "ep-k1-drops-bf16": (700, 128, 256, 8, 1, 1.0, "bf16", False),
    "ep-k2-drops-f32": (500, 64, 128, 4, 2, 0.8, "f32", False),
    "ep-k2-skew-bf16": (400, 64, 128, 4, 2, None, "bf16", True),      # rank 1 receives no rows
    "ep-k1-large-bf16": (2000, 128, 256, 4, 1, None, "bf16", False),   # ~1000 rows per local expert
}
# name: T (the same batch on every rank), d, ff, E, k, capacity factor, dtype, skewed
SHARD_CASES = {
    "shard-k2-f32": (300, 64, 256, 8, 2, None, "f32", False),
    "shard-k1-drops-bf16": (600, 128, 512, 8, 1, 1.0, "bf16", False),
    "shard-k2-skew-bf16": (400, 64, 128, 4, 2, None, "bf16", True),
}


def _inputs(case, T_total, seed):
    from mixture_experts_layer_45_b200 import workloads as wl
    T, d, ff, E, k, cf, dtype, skew = case
    inp = wl.draw_custom(seed, T=T_total, d=d, ff=ff, E=E, dtype=dtype, router_std=0.5)
    if skew:
        # every token prefers the first E/G experts (rank 0's block)
        inp["logit_bias"] = np.where(np.arange(E) < E // WORLD, 30.0, 0.0).astype(np.float32)
    return inp


def _oracle_on_gpu_routing(x_np, inp, idx_np, k, E, cap):
    from oracle import moe_ref
    r = moe_ref.route(x_np, inp["w_router"], k, inp.get("logit_bias"))
    gates = np.take_along_axis(r["gates"], idx_np.astype(np.int64), 1)
    dsp = moe_ref.dispatch(idx_np, E, cap)
    return moe_ref.moe_forward(x_np, inp, idx_np, gates, dsp["slot_of"]), dsp


def _check(out, ref, dsp, T, k, dtype):
    import parity_util as pu
    err = pu.max_rel_err(out, ref) if np.abs(ref).max() > 0 else float(np.abs(out).max())
    all_dropped = (dsp["slot_of"].reshape(T, k) < 0).all(1)
    return {"err": err, "tol": pu.TOL[dtype], "zero_where_dropped": bool(np.all(out[all_dropped] == 0.0)),
            "n_all_dropped": int(all_dropped.sum()), "finite": bool(np.isfinite(out).all())}


def _run_ep(rank, name, case, dev):
    import torch
    from mixture_experts_layer_45_b200 import _lib
    from mixture_experts_layer_45_b200 import expert_parallel as ep
    from mixture_experts_layer_45_b200.layer import MoEParams, dtype_code, to_device
    from oracle import moe_ref
    T, d, ff, E, k, cf, dtype, skew = case
    inp = _inputs(case, T * WORLD, seed=100 + len(name))
    x_np = inp["x"][rank * T:(rank + 1) * T]
    dt = dtype_code(dtype)
    cap = moe_ref.capacity(T, k, E, cf)             # each rank's own batch budget
    params = MoEParams.from_arrays(inp, dt, dev)
    w1, b1, w2, b2 = ep.shard_experts(params, rank, WORLD)
    layer = ep.ExpertParallelMoE(params.w_router, params.logit_bias, w1, b1, w2, b2, dt, k, cap)
    x = to_device(x_np, dt, dev)
    out = layer(x).float().cpu().numpy()
    idx, _ = layer.steps.route(x)
    torch.cuda.synchronize()
    assert _lib.moe_get_error() == _lib.MOE_OK
    idx_np = idx.cpu().numpy()
    ref, dsp = _oracle_on_gpu_routing(x_np, inp, idx_np, k, E, cap)
    res = _check(out, ref, dsp, T, k, dtype)
    el = E // WORLD
    # rows this rank sends to each rank (its kept assignments, by expert block)
    kept = dsp["slot_of"].reshape(T, k) >= 0
    res["sent"] = [int((kept & (idx_np // el == q)).sum()) for q in range(WORLD)]
    res["dropped"] = int((~kept).sum())
    return res


def _run_shard(rank, name, case, dev):
    import torch
    from mixture_experts_layer_45_b200 import _lib
    from mixture_experts_layer_45_b200 import expert_parallel as ep
    from mixture_experts_layer_45_b200.layer import MoEParams, dtype_code, to_device
    from oracle import moe_ref
    T, d, ff, E, k, cf, dtype, skew = case
    inp = _inputs(case, T, seed=200 + len(name))
    x_np = inp["x"]
    dt = dtype_code(dtype)
    cap = moe_ref.capacity(T, k, E, cf)
    params = MoEParams.from_arrays(inp, dt, dev)
    w1, b1, w2, b2 = ep.shard_hidden(params, rank, WORLD)
    layer = ep.ShardedExpertsMoE(params.w_router, params.logit_bias, w1, b1, w2, b2, dt, k, cap)
    x = to_device(x_np, dt, dev)
    out = layer(x).float().cpu().numpy()
    idx, _ = layer.steps.route(x)
    torch.cuda.synchronize()
    assert _lib.moe_get_error() == _lib.MOE_OK
    idx_np = idx.cpu().numpy()
    ref, dsp = _oracle_on_gpu_routing(x_np, inp, idx_np, k, E, cap)
    res = _check(out, ref, dsp, T, k, dtype)
    res["dropped"] = int((dsp["slot_of"] < 0).sum())
    return res


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=120))
    results = {}
    try:
        from mixture_experts_layer_45_b200 import _lib
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        _lib.load()
        # every rank runs the same cases in the same order (same collectives)
        for name, case in EP_CASES.items():
            results[name] = _run_ep(rank, name, case, dev)
        for name, case in SHARD_CASES.items():
            results[name] = _run_shard(rank, name, case, dev)
        q.put((rank, results, None))
    except Exception:
        q.put((rank, results, traceback.format_exc()))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def rank_results():
    import torch
    import torch.multiprocessing as mp
    assert torch.cuda.is_available(), "these tests need a CUDA GPU"
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, res, err = q.get(timeout=600)
        assert err is None, f"rank {rank}:\n{err}"
        got[rank] = res
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("name", sorted(EP_CASES))
def test_expert_parallel_on_gpu_kernels(rank_results, name):
    T, d, ff, E, k, cf, dtype, skew = EP_CASES[name]
    for rank in range(WORLD):
        r = rank_results[rank][name]
        assert r["finite"] and r["zero_where_dropped"]
        assert r["err"] <= r["tol"], (rank, r)
    if cf is not None:
        assert sum(rank_results[r][name]["dropped"] for r in range(WORLD)) > 0, "the case should drop"
    if skew:
        # nobody sends rows to rank 1: it serves no rows and still returns its output
        assert all(rank_results[r][name]["sent"][1] == 0 for r in range(WORLD))


@pytest.mark.parametrize("name", sorted(SHARD_CASES))
def test_sharded_experts_on_gpu_kernels(rank_results, name):
    T, d, ff, E, k, cf, dtype, skew = SHARD_CASES[name]
    for rank in range(WORLD):
        r = rank_results[rank][name]
        assert r["finite"] and r["zero_where_dropped"]
        assert r["err"] <= r["tol"], (rank, r)
    if cf is not None:
        assert rank_results[0][name]["dropped"] > 0
