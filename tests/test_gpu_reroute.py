"""GPU parity of overflow rerouting (the blog "MoE Parallelism for Inference",
section "Common Bottlenecks", item 1; the cookbook notebook, section "What")
against the float64 oracle's dispatch_reroute, through the C ABI.

The dispatch is integer work: bit-exact given the same ranked expert lists.
The layer output is checked on the GPU's own ranking (indices valid within
the fp32 logit error bound) with max-norm relative error <= 1e-4 (fp32) or
2e-2 (bf16).
"""
import numpy as np
import pytest
import torch

import parity_util as pu
from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import workloads as wl
from mixture_experts_layer_45_b200.layer import MoELayer, MoEParams, dtype_code, read_stats, to_device
from oracle import moe_ref

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "these tests need a CUDA GPU"
    _lib.load()
    yield
    torch.cuda.synchronize()


def random_ranked(seed, T, E, K):
    """Distinct experts per row, skewed towards a few hot experts."""
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.ones(E) * 0.3)
    idx = np.stack([rng.choice(E, size=K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, K)).astype(np.float32)
    return idx, gate


def run_dispatch_reroute(ranked, gate, k, F, E, cap, x_np=None, dt=_lib.MOE_F32):
    T = ranked.shape[0]
    A = T * k
    t_rank = torch.from_numpy(np.ascontiguousarray(ranked, np.int32)).to(DEV)
    t_gate = torch.from_numpy(np.ascontiguousarray(gate, np.float32)).to(DEV)
    counts = torch.full((E,), -1, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), -1, dtype=torch.int32, device=DEV)
    perm = torch.full((max(A, 1),), -1, dtype=torch.int32, device=DEV)
    slot_of = torch.full((max(A, 1),), -9, dtype=torch.int32, device=DEV)
    drop = torch.full((max(A, 1),), 7, dtype=torch.uint8, device=DEV)
    row_gate = torch.full((max(A, 1),), -1.0, dtype=torch.float32, device=DEV)
    x = xp = None
    d = 8
    if x_np is not None:
        d = x_np.shape[1]
        x = to_device(x_np, dt, DEV)
        xp = torch.zeros((max(A, 1), d), dtype=x.dtype, device=DEV)
    nws = _lib.moe_dispatch_reroute_workspace_size(T, k, F, E)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=DEV)
    _lib.moe_dispatch_reroute(t_rank, t_gate, T, k, F, E, cap, counts, offsets, perm, slot_of, drop, row_gate, x, xp,
                              d, dt, ws, nws)
    assert _lib.moe_get_error() == _lib.MOE_OK
    out = dict(counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(), perm=perm.cpu().numpy(),
               slot_of=slot_of.cpu().numpy(), drop_mask=drop.cpu().numpy(), row_gate=row_gate.cpu().numpy())
    if xp is not None:
        out["xp"] = xp.float().cpu().numpy()
    return out


def assert_reroute_equal(g, o, A, ranked_gate=None, k=1):
    R = int(o["offsets"][-1])
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["offsets"], o["offsets"])
    np.testing.assert_array_equal(g["perm"][:R], o["perm"])
    np.testing.assert_array_equal(g["slot_of"][:A], o["slot_of"])
    np.testing.assert_array_equal(g["drop_mask"][:A], o["drop_mask"])
    if ranked_gate is not None:
        t, j = np.divmod(o["perm"], k)
        np.testing.assert_array_equal(g["row_gate"][:R], o["final_gate"][t, j].astype(np.float32))


@pytest.mark.parametrize("T,k,F,E,cap,seed", [
    (5000, 1, 1, 8, 500, 0),      # top-1, one round
    (5000, 2, 2, 16, 500, 1),     # top-2, two rounds
    (3000, 1, 3, 8, 300, 2),      # deeper fallbacks
    (4097, 3, 5, 16, 600, 3),     # k + F = 8 (the router's limit), ragged last chunk
    (2048, 1, 7, 256, 5, 4),      # many experts, tiny capacity
    (700, 2, 1, 4, 0, 5),         # capacity 0: nothing can be served
    (1000, 2, 2, 8, -1, 6),       # no capacity: nothing dropped, nothing rerouted
    (1, 1, 1, 2, 0, 7),           # one token
    (20000, 1, 2, 64, 250, 8),    # many chunks
])
def test_dispatch_reroute_bit_exact(T, k, F, E, cap, seed):
    ranked, gate = random_ranked(seed, T, E, k + F)
    g = run_dispatch_reroute(ranked, gate, k, F, E, cap)
    o = moe_ref.dispatch_reroute(ranked, gate.astype(np.float64), k, E, cap, F)
    assert_reroute_equal(g, o, T * k, gate, k)
    if cap > 0 and T > 100:
        assert o["rerouted"] > 0           # the case exercises rerouting


def test_dispatch_reroute_gathers_rows():
    T, k, F, E, cap, d = 3000, 2, 2, 12, 420, 72
    ranked, gate = random_ranked(11, T, E, k + F)
    x = wl.round_to_bf16(np.random.default_rng(3).normal(size=(T, d)).astype(np.float32))
    g = run_dispatch_reroute(ranked, gate, k, F, E, cap, x, _lib.MOE_BF16)
    o = moe_ref.dispatch_reroute(ranked, gate.astype(np.float64), k, E, cap, F)
    assert_reroute_equal(g, o, T * k, gate, k)
    R = int(o["offsets"][-1])
    np.testing.assert_array_equal(g["xp"][:R], x[o["perm"] // k])


def test_dispatch_reroute_zero_rounds_is_dispatch():
    T, k, E, cap = 4000, 2, 8, 700
    ranked, gate = random_ranked(12, T, E, k)
    g = run_dispatch_reroute(ranked, gate, k, 0, E, cap)
    o = moe_ref.dispatch(ranked, E, cap)
    R = int(o["offsets"][-1])
    np.testing.assert_array_equal(g["offsets"], o["offsets"])
    np.testing.assert_array_equal(g["perm"][:R], o["perm"])
    np.testing.assert_array_equal(g["slot_of"][:T * k], o["slot_of"])


# ---------------------------------------------------------------------------
# the whole layer with rerouting
# ---------------------------------------------------------------------------
def gpu_ranking(layer, T, k, F, idx_t):
    fb = layer.workspace_view(T, "fallback_idx", torch.int32, T * F).cpu().numpy().reshape(T, F)
    return np.concatenate([idx_t.cpu().numpy(), fb], axis=1)


REROUTE_WORKLOADS = [
    (wl.workload("switch-top1", dtype="bf16", cf=1.0), 1),
    (wl.workload("switch-top1", dtype="bf16", cf=1.0), 2),
    (wl.workload("switch-top1", dtype="f32", cf=1.0), 1),
    (wl.workload("encoder-prefill-top1"), 2),
]


@pytest.mark.parametrize("w,F", REROUTE_WORKLOADS, ids=lambda v: str(v) if isinstance(v, int) else
                         f"{v.name}-{v.dtype}")
def test_forward_reroute_matches_oracle(w, F):
    inp = wl.draw_inputs(w)
    dt = dtype_code(w.dtype)
    cap = _lib.moe_capacity(w.T, w.k, w.E, w.cf)
    params = MoEParams.from_arrays(inp, dt, DEV)
    layer = MoELayer(params, w.k, cap, reroute=F)
    x = to_device(inp["x"], dt, DEV)
    idx_t = torch.empty((w.T, w.k), dtype=torch.int32, device=DEV)
    out = layer.forward(x, stats=True, topk_idx=idx_t).float().cpu().numpy()
    assert _lib.moe_get_error() == _lib.MOE_OK
    ranked = gpu_ranking(layer, w.T, w.k, F, idx_t)
    # the GPU's ranking is the oracle's wherever the float64 logits separate it
    r = moe_ref.route(inp["x"], inp["w_router"], w.k + F, inp["logit_bias"])
    delta = pu.logit_error_bound(inp["x"], inp["w_router"], inp["logit_bias"])
    n_diff, _ = pu.check_routing(ranked, r["logits"], w.k + F, delta)
    assert n_diff <= max(2, w.T // 2000)
    # dispatch on the GPU's ranking: bit-exact
    gates = np.take_along_axis(r["gates"], ranked.astype(np.int64), 1)
    o = moe_ref.dispatch_reroute(ranked, gates, w.k, w.E, cap, F)
    A = w.T * w.k
    R = int(o["offsets"][-1])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "offsets", torch.int32, w.E + 1).cpu().numpy(),
                                  o["offsets"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "perm", torch.int32, R).cpu().numpy(), o["perm"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "slot_of", torch.int32, A).cpu().numpy(),
                                  o["slot_of"])
    assert o["rerouted"] > 0
    st = read_stats(layer.stats_buf)
    assert st["rows_kept"] == R and st["dropped"] == A - R and st["rerouted"] == o["rerouted"]
    assert st["drop_rate"] == pytest.approx((A - R) / A, rel=1e-6, abs=1e-7)
    # output rows: rerouted tokens first, then a sample
    rerouted = np.nonzero((o["final_idx"] != ranked[:, :w.k]).any(1))[0][:48]
    rows = pu.sample_rows(w.T, 64, seed=w.seed, must=list(rerouted))
    ref = moe_ref.moe_forward_rows(inp["x"], inp, o["final_idx"], o["final_gate"], o["slot_of"], rows)
    assert pu.max_rel_err(out[rows], ref) <= pu.TOL[w.dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,d,ff,E,k,cap,F,S", [
    (1000, 72, 200, 6, 2, 330, 2, 0),    # top-2, two rounds, ragged tails
    (1500, 64, 128, 8, 1, 195, 1, 1),    # top-1 rerouting with a shared expert (combine path)
    (900, 64, 64, 16, 1, 54, 3, 0),      # top-1, direct output rows, all three rounds serve slots
    (300, 64, 64, 4, 2, 0, 2, 0),        # capacity 0: nothing served, output 0
])
def test_forward_reroute_edge_cases(dtype, T, d, ff, E, k, cap, F, S):
    inp = wl.draw_custom(13, T=T, d=d, ff=ff, E=E, dtype=dtype, router_std=0.5, shared=S)
    dt = dtype_code(dtype)
    layer = MoELayer(MoEParams.from_arrays(inp, dt, DEV), k, cap, reroute=F)
    x = to_device(inp["x"], dt, DEV)
    idx_t = torch.empty((T, k), dtype=torch.int32, device=DEV)
    out = layer.forward(x, stats=True, topk_idx=idx_t).float().cpu().numpy()
    assert _lib.moe_get_error() == _lib.MOE_OK
    ranked = gpu_ranking(layer, T, k, F, idx_t)
    r = moe_ref.route(inp["x"], inp["w_router"], k + F)
    gates = np.take_along_axis(r["gates"], ranked.astype(np.int64), 1)
    o = moe_ref.dispatch_reroute(ranked, gates, k, E, cap, F)
    np.testing.assert_array_equal(layer.workspace_view(T, "slot_of", torch.int32, T * k).cpu().numpy(),
                                  o["slot_of"])
    ref = moe_ref.moe_forward(inp["x"], inp, o["final_idx"], o["final_gate"], o["slot_of"])
    if S:
        ref = ref + moe_ref.shared_experts(inp["x"], inp)
    if cap == 0 and S == 0:
        assert np.all(out == 0.0)
    else:
        assert pu.max_rel_err(out, ref) <= pu.TOL[dtype]
    if cap > 0:
        assert o["rerouted"] > 0
