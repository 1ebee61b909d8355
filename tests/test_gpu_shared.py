"""GPU parity of the shared always-on experts (cookbook notebook "Mixture-of-
experts and expert parallelism", section "Exercises", item 3) against the
float64 oracle, through the C ABI.

The routed part is checked on the GPU's own routing as in test_gpu_parity;
the shared experts add, on every token, the ungated sum of their MLPs.
Tolerances: max-norm relative error <= 1e-4 (fp32) or 2e-2 (bf16).
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


def run_layer(inp, k, cap, dt, T):
    params = MoEParams.from_arrays(inp, dt, DEV)
    layer = MoELayer(params, k, cap)
    x = to_device(inp["x"], dt, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    out = layer.forward(x, stats=True, topk_idx=idx)
    assert _lib.moe_get_error() == _lib.MOE_OK
    return layer, out.float().cpu().numpy(), idx.cpu().numpy()


def oracle_rows(inp, idx_np, k, E, cap, rows):
    """The oracle's output rows (routed on the GPU's expert choice, gates the
    oracle's softmax at those experts, plus the shared experts)."""
    r = moe_ref.route(inp["x"], inp["w_router"], k, inp.get("logit_bias"))
    gates = np.take_along_axis(r["gates"], idx_np.astype(np.int64), 1)
    dsp = moe_ref.dispatch(idx_np, E, cap)
    return moe_ref.moe_forward_rows_shared(inp["x"], inp, idx_np, gates, dsp["slot_of"], rows), dsp, r


SHARED_WORKLOADS = [
    wl.workload("dense-top2-f32", shared=1),
    wl.workload("switch-top1", dtype="f32", cf=1.0, shared=1),
    wl.workload("switch-top1", dtype="bf16", cf=1.0, shared=2),
    wl.workload("skewed-top2", shared=2),
]


@pytest.mark.parametrize("w", SHARED_WORKLOADS, ids=lambda w: f"{w.name}-{w.dtype}-S{w.shared}")
def test_forward_shared_matches_oracle(w):
    inp = wl.draw_inputs(w)
    dt = dtype_code(w.dtype)
    cap = _lib.moe_capacity(w.T, w.k, w.E, w.cf)
    layer, out, idx = run_layer(inp, w.k, cap, dt, w.T)
    assert np.isfinite(out).all()
    dsp0 = moe_ref.dispatch(idx, w.E, cap)
    dropped = np.nonzero((dsp0["slot_of"].reshape(w.T, w.k) < 0).all(1))[0][:16]
    if cap >= 0:
        assert len(dropped) > 0 or w.cf is None or w.cf > 1.0
    # every 128-row M tile of every routed and shared group (so every
    # 256-row CTA-pair tile too), plus random and dropped rows
    tiles = pu.tile_covering_rows(dsp0["offsets"], dsp0["perm"], w.k, w.T, seed=w.seed, shared=w.shared)
    rows = pu.sample_rows(w.T, 96 if w.T > 2048 else w.T, seed=w.seed, must=list(dropped) + list(tiles))
    print(f"{w.name} S={w.shared}: {len(rows)} sampled output rows reach all "
          f"{pu.m_tiles(dsp0['offsets']) + w.shared * -(-w.T // 128)} 128-row M tiles")
    ref, dsp, r = oracle_rows(inp, idx, w.k, w.E, cap, rows)
    err = pu.max_rel_err(out[rows], ref)
    assert err <= pu.TOL[w.dtype], err
    # tokens with every routed assignment dropped receive the shared sum alone
    if len(dropped):
        ref_d = moe_ref.shared_experts(inp["x"][dropped], inp)
        assert pu.max_rel_err(out[dropped], ref_d) <= pu.TOL[w.dtype]
    # the shared experts' own rows in the workspace (rows T*k + s*T + t of yp)
    A = w.T * w.k
    yp = layer.workspace_view(w.T, "yp", torch.float32 if dt == _lib.MOE_F32 else torch.bfloat16,
                              (A + w.shared * w.T) * w.d).float().cpu().numpy().reshape(-1, w.d)
    some = rows[:24]
    ys_ref = moe_ref.shared_expert_outputs(inp["x"][some], inp)
    for s in range(w.shared):
        assert pu.max_rel_err(yp[A + s * w.T + some], ys_ref[s]) <= pu.TOL[w.dtype]
    # routing, dispatch and statistics are the routed layer's
    R = int(dsp["offsets"][-1])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "offsets", torch.int32, w.E + 1).cpu().numpy(),
                                  dsp["offsets"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "perm", torch.int32, R).cpu().numpy(), dsp["perm"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "slot_of", torch.int32, A).cpu().numpy(),
                                  dsp["slot_of"])
    st = read_stats(layer.stats_buf)
    ref_st = moe_ref.layer_stats(idx, r["gates"], w.E, cap)
    assert st["rows_kept"] == ref_st["rows_kept"] and st["dropped"] == ref_st["dropped"]
    assert st["aux_loss"] == pytest.approx(ref_st["aux_loss"], rel=1e-4)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,d,ff,E,k,cap,S", [
    (1000, 72, 200, 5, 2, -1, 1),      # ragged K and N tails, ragged last row tile
    (500, 64, 64, 8, 2, 0, 2),         # capacity 0: the output is the shared sum alone
    (1, 64, 64, 8, 2, -1, 3),          # one token
    (777, 64, 128, 1, 1, -1, 8),       # the most shared experts, one routed expert
    (2000, 128, 256, 16, 1, 60, 2),    # top-1 with drops (no direct fc2 output with shared experts)
    (300, 136, 320, 4, 4, -1, 1),      # k = E
    (3000, 64, 128, 2, 1, -1, 2),      # >= 384 rows per expert: CTA-pair kernels with shared groups
])
def test_forward_shared_edge_cases(dtype, T, d, ff, E, k, cap, S):
    inp = wl.draw_custom(7, T=T, d=d, ff=ff, E=E, dtype=dtype, router_std=0.5, shared=S)
    dt = dtype_code(dtype)
    _, out, idx = run_layer(inp, k, cap, dt, T)
    ref, dsp, _ = oracle_rows(inp, idx, k, E, cap, np.arange(T))
    assert pu.max_rel_err(out, ref) <= pu.TOL[dtype]
    if cap == 0:
        assert (dsp["slot_of"] < 0).all()
        assert pu.max_rel_err(out, moe_ref.shared_experts(inp["x"], inp)) <= pu.TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shared_ffn_and_combine_steps(dtype):
    T, d, ff, S, k = 700, 72, 200, 3, 2
    inp = wl.draw_custom(9, T=T, d=d, ff=ff, E=4, dtype=dtype, shared=S)
    dt = dtype_code(dtype)
    p = MoEParams.from_arrays(inp, dt, DEV)
    x = to_device(inp["x"], dt, DEV)
    h = torch.full((S * T, ff), float("nan"), dtype=x.dtype, device=DEV)
    ys = torch.full((S * T, d), float("nan"), dtype=x.dtype, device=DEV)
    _lib.moe_shared_ffn(x, T, d, ff, S, p.shared_w1, p.shared_b1, p.shared_w2, p.shared_b2, h, ys, dt)
    assert _lib.moe_get_error() == _lib.MOE_OK
    ys_np = ys.float().cpu().numpy().reshape(S, T, d)
    ref = moe_ref.shared_expert_outputs(inp["x"], inp)
    for s in range(S):
        assert pu.max_rel_err(ys_np[s], ref[s]) <= pu.TOL[dtype]
    # combine: random routed slots and gates plus the shared rows
    rng = np.random.default_rng(2)
    R = 900
    yp = rng.normal(size=(R, d)).astype(np.float32)
    slot = rng.permutation(T * k).astype(np.int32)
    slot[slot >= R] = -1
    gate = rng.random((T, k)).astype(np.float32)
    yp_dev = to_device(yp, dt, DEV)
    out = torch.empty((T, d), dtype=x.dtype, device=DEV)
    _lib.moe_combine_shared(yp_dev, torch.from_numpy(slot).to(DEV), torch.from_numpy(gate).to(DEV), ys, S, T, k,
                            d, dt, out)
    assert _lib.moe_get_error() == _lib.MOE_OK
    want = moe_ref.combine(yp_dev.float().cpu().numpy(), slot, T, k, gate) + ys_np.astype(np.float64).sum(0)
    assert pu.max_rel_err(out.float().cpu().numpy(), want) <= (4e-3 if dtype == "bf16" else 1e-6)


def test_shared_zero_is_plain_forward():
    """S = 0 and no rerouting through moe_forward_ex gives moe_forward's bits."""
    w = wl.workload("switch-top1", dtype="bf16", cf=1.0)
    inp = wl.draw_inputs(w, T=1500)
    p = MoEParams.from_arrays(inp, _lib.MOE_BF16, DEV)
    x = to_device(inp["x"], _lib.MOE_BF16, DEV)
    T, cap = 1500, _lib.moe_capacity(1500, w.k, w.E, w.cf)
    n = _lib.moe_workspace_size(T, w.d, w.ff, w.E, w.k, _lib.MOE_BF16)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    a = torch.empty_like(x)
    b = torch.empty_like(x)
    _lib.moe_forward(x, p.w_router, None, p.w1, p.b1, p.w2, p.b2, T, w.d, w.ff, w.E, w.k, cap, _lib.MOE_BF16, a,
                     None, None, None, ws, n)
    _lib.moe_forward_ex(x, p.w_router, None, p.w1, p.b1, p.w2, p.b2, 0, None, None, None, None, 0, T, w.d, w.ff,
                        w.E, w.k, cap, _lib.MOE_BF16, b, None, None, None, ws, n)
    assert _lib.moe_get_error() == _lib.MOE_OK
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shared_launch_count():
    inp = wl.draw_custom(12, T=512, d=64, ff=128, E=8, dtype="bf16", shared=2)
    p = MoEParams.from_arrays(inp, _lib.MOE_BF16, DEV)
    layer = MoELayer(p, 1, -1)
    x = to_device(inp["x"], _lib.MOE_BF16, DEV)
    layer.forward(x)
    torch.cuda.synchronize()
    n0 = _lib.moe_launch_count()
    layer.forward(x)
    torch.cuda.synchronize()
    # router, dispatch (scan + permute + gather), ffn1 (routed + shared), ffn2 (routed + shared), combine
    assert _lib.moe_launch_count() - n0 == 5
