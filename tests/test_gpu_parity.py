"""GPU parity: every step of the CUDA path against the float64 oracle, on the
seeded workloads at their full sizes and on small ragged cases, called
through the C ABI.

Routing: indices bit-exact wherever the float64 logits separate the choice
by more than the fp32 error bound, valid elsewhere (parity_util.check_routing).
Dispatch: bit-exact given identical indices (both the GPU's and the oracle's).
FFN, combine and the whole layer: max-norm relative error <= 1e-4 (fp32) or
2e-2 (bf16) against the oracle run on the GPU's own routing.
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

VARIANTS = wl.all_workloads()
VARIANT_IDS = [f"{w.name}-{w.dtype}-cf{w.capacity_factor_label()}" for w in VARIANTS]
# the oracle computes every output row of these; the others are sampled
FULL_ORACLE = {"dense-top2-f32", "switch-top1"}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "these tests need a CUDA GPU"
    _lib.load()
    yield
    torch.cuda.synchronize()


_INPUT_CACHE = {}


def inputs_for(w):
    key = (w.name, w.dtype)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE.clear()
        _INPUT_CACHE[key] = wl.draw_inputs(w)
    return _INPUT_CACHE[key]


def bias_t(inp):
    b = inp.get("logit_bias")
    return None if b is None else torch.from_numpy(np.asarray(b, np.float32)).to(DEV)


def run_router(inp, k, dt):
    x = to_device(inp["x"], dt, DEV)
    wr = to_device(inp["w_router"], dt, DEV)
    T, d = inp["x"].shape
    E = inp["w_router"].shape[0]
    idx = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    gate = torch.full((T, k), -1.0, dtype=torch.float32, device=DEV)
    psum = torch.full((E,), 123.0, dtype=torch.float32, device=DEV)
    _lib.moe_router_topk(x, wr, bias_t(inp), T, d, E, k, dt, idx, gate, psum)
    assert _lib.moe_get_error() == _lib.MOE_OK
    return idx.cpu().numpy(), gate.cpu().numpy(), psum.cpu().numpy()


def run_dispatch(idx_np, gate_np, E, cap, x_np=None, dt=_lib.MOE_F32):
    T, k = idx_np.shape
    A = T * k
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).to(DEV)
    gate = torch.from_numpy(np.ascontiguousarray(gate_np, np.float32)).to(DEV)
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
    nws = _lib.moe_dispatch_workspace_size(T, k, E)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=DEV)
    _lib.moe_dispatch(idx, gate, T, k, E, cap, counts, offsets, perm, slot_of, drop, row_gate, x, xp, d, dt,
                      ws, nws)
    assert _lib.moe_get_error() == _lib.MOE_OK
    out = dict(counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(), perm=perm.cpu().numpy(),
               slot_of=slot_of.cpu().numpy(), drop_mask=drop.cpu().numpy(), row_gate=row_gate.cpu().numpy())
    if xp is not None:
        out["xp_dev"] = xp
        out["xp"] = xp.float().cpu().numpy()
        out["x_dev"] = x
    out["dev"] = dict(offsets=offsets, slot_of=slot_of, row_gate=row_gate)
    return out


def assert_dispatch_equal(g, o, A):
    R = int(o["offsets"][-1])
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["offsets"], o["offsets"])
    np.testing.assert_array_equal(g["perm"][:R], o["perm"])
    np.testing.assert_array_equal(g["slot_of"][:A], o["slot_of"])
    np.testing.assert_array_equal(g["drop_mask"][:A], o["drop_mask"])


# ---------------------------------------------------------------------------
# step 1: router
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", VARIANTS, ids=VARIANT_IDS)
def test_router_matches_oracle(w):
    inp = wl.draw_router_inputs(w)
    dt = dtype_code(w.dtype)
    idx, gate, psum = run_router(inp, w.k, dt)
    r = moe_ref.route(inp["x"], inp["w_router"], w.k, inp["logit_bias"])
    delta = pu.logit_error_bound(inp["x"], inp["w_router"], inp["logit_bias"])
    n_diff, n_undecided = pu.check_routing(idx, r["logits"], w.k, delta)
    assert n_diff <= max(2, w.T // 2000), (n_diff, n_undecided)
    # gates: the oracle's softmax at the GPU's experts
    ref_gate = np.take_along_axis(r["gates"], idx.astype(np.int64), 1)
    assert pu.max_rel_err(gate, ref_gate) <= 1e-5
    assert pu.max_rel_err(psum, r["gates"].sum(0)) <= 1e-4


def test_router_exact_ties_go_to_lower_index():
    T, d, E, k = 100, 64, 16, 3
    inp = {"x": np.random.default_rng(0).normal(size=(T, d)).astype(np.float32),
           "w_router": np.zeros((E, d), np.float32), "logit_bias": None}
    idx, gate, psum = run_router(inp, k, _lib.MOE_F32)
    np.testing.assert_array_equal(idx, np.tile(np.arange(k), (T, 1)))
    np.testing.assert_allclose(gate, 1.0 / E, rtol=1e-6)
    np.testing.assert_allclose(psum, T / E, rtol=1e-5)


@pytest.mark.parametrize("E,k", [(1, 1), (5, 5), (256, 8), (40, 3)])
def test_router_expert_count_edges(E, k):
    inp = wl.draw_custom(3, T=333, d=136, ff=8, E=E, dtype="bf16", router_std=0.3)
    idx, gate, _ = run_router(inp, k, _lib.MOE_BF16)
    r = moe_ref.route(inp["x"], inp["w_router"], k)
    delta = pu.logit_error_bound(inp["x"], inp["w_router"])
    pu.check_routing(idx, r["logits"], k, delta)
    assert pu.max_rel_err(gate, np.take_along_axis(r["gates"], idx.astype(np.int64), 1)) <= 1e-5


@pytest.mark.parametrize("T,d,E,k,bias", [
    (1000, 1024, 8, 2, False),     # 16 K stages, 8 tiles: the K split over CTA pairs, ragged last tile
    (300, 1096, 40, 3, True),      # split with a K tail (1096 = 17 * 64 + 8) and a logit bias
    (4000, 2048, 64, 2, False),    # split at 64 experts (two logit chunks), 32 tiles
    (64, 4096, 16, 1, True),       # one tile, 64 K stages: the pair's halves of 32 stages each
])
def test_router_k_split_matches_oracle(T, d, E, k, bias):
    """Tiles of large d on few tokens split their K stages over the two CTAs
    of a cluster (the second's partial logits added in the first's shared
    memory); indices, gates, probability sums and the per-tile histograms
    must be those of the one-CTA form's definition."""
    inp = wl.draw_custom(13, T=T, d=d, ff=8, E=E, dtype="bf16", router_std=0.05)
    if bias:
        inp["logit_bias"] = np.linspace(-1.0, 1.0, E).astype(np.float32)
    idx, gate, psum = run_router(inp, k, _lib.MOE_BF16)
    r = moe_ref.route(inp["x"], inp["w_router"], k, inp.get("logit_bias"))
    delta = pu.logit_error_bound(inp["x"], inp["w_router"], inp.get("logit_bias"))
    n_diff, _ = pu.check_routing(idx, r["logits"], k, delta)
    assert n_diff <= 2
    assert pu.max_rel_err(gate, np.take_along_axis(r["gates"], idx.astype(np.int64), 1)) <= 1e-5
    assert pu.max_rel_err(psum, r["gates"].sum(0)) <= 1e-4


# ---------------------------------------------------------------------------
# step 2: dispatch (bit-exact)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", VARIANTS, ids=VARIANT_IDS)
def test_dispatch_bit_exact(w):
    inp = wl.draw_router_inputs(w)
    dt = dtype_code(w.dtype)
    idx_gpu, gate_gpu, _ = run_router(inp, w.k, dt)
    cap = moe_ref.capacity(w.T, w.k, w.E, w.cf)
    r = moe_ref.route(inp["x"], inp["w_router"], w.k, inp["logit_bias"])
    for idx, gate in ((idx_gpu, gate_gpu), (r["topk_idx"].astype(np.int32), r["topk_gate"].astype(np.float32))):
        g = run_dispatch(idx, gate, w.E, cap, inp["x"], dt)
        o = moe_ref.dispatch(idx, w.E, cap)
        assert_dispatch_equal(g, o, w.T * w.k)
        R = int(o["offsets"][-1])
        np.testing.assert_array_equal(g["row_gate"][:R], gate.reshape(-1)[o["perm"]])
        np.testing.assert_array_equal(g["xp"][:R], inp["x"][o["perm"] // w.k])


@pytest.mark.parametrize("T,k,E,cap,seed", [(1, 1, 1, -1, 0), (5000, 2, 7, -1, 1), (5000, 2, 7, 100, 2),
                                            (4097, 3, 16, 0, 3), (2048, 1, 256, 5, 4), (70000, 8, 64, 8000, 5),
                                            (3000, 1, 3, 1, 6)])
def test_dispatch_random_indices(T, k, E, cap, seed):
    rng = np.random.default_rng(seed)
    # skewed distinct-per-row indices
    p = rng.dirichlet(np.ones(E) * 0.3)
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    g = run_dispatch(idx, gate, E, cap)
    o = moe_ref.dispatch(idx, E, cap)
    assert_dispatch_equal(g, o, T * k)


def test_dispatch_empty_batch():
    g = run_dispatch(np.zeros((0, 2), np.int32), np.zeros((0, 2), np.float32), 8, -1)
    np.testing.assert_array_equal(g["counts"], 0)
    np.testing.assert_array_equal(g["offsets"], 0)


def test_dispatch_reports_bad_routing():
    idx = np.array([[0, 1], [2, 9], [3, -1], [1, 0]], np.int32)
    T, k, E = 4, 2, 4
    t_idx = torch.from_numpy(idx).to(DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    slot_of = torch.empty(T * k, dtype=torch.int32, device=DEV)
    nws = _lib.moe_dispatch_workspace_size(T, k, E)
    ws = torch.empty(nws, dtype=torch.uint8, device=DEV)
    _lib.moe_dispatch(t_idx, None, T, k, E, -1, counts, offsets, perm, slot_of, None, None, None, None, 8,
                      _lib.MOE_F32, ws, nws)
    assert _lib.moe_get_error() == _lib.MOE_ERR_BAD_ROUTING
    assert _lib.moe_get_error() == _lib.MOE_OK          # reading clears the word
    s = slot_of.cpu().numpy()
    assert s[3] == -1 and s[5] == -1                      # the bad indices were dropped
    np.testing.assert_array_equal(counts.cpu().numpy(), [2, 2, 1, 1])


# ---------------------------------------------------------------------------
# step 3: grouped FFN
# ---------------------------------------------------------------------------
def run_ffn(xp_dev, offsets_dev, max_rows, params, row_gate_dev):
    d, ff, E = params.d, params.ff, params.E
    h = torch.full((max_rows, ff), float("nan"), dtype=params.w1.dtype, device=DEV)
    yp = torch.full((max_rows, d), float("nan"), dtype=params.w1.dtype, device=DEV)
    _lib.moe_grouped_ffn(xp_dev, offsets_dev, max_rows, E, d, ff, params.w1, params.b1, params.w2, params.b2,
                         row_gate_dev, h, yp, params.dtype)
    assert _lib.moe_get_error() == _lib.MOE_OK
    return h.float().cpu().numpy(), yp.float().cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("sizes,d,ff", [
    ([0, 1, 127, 128, 129, 255, 300, 0, 5], 128, 256),     # tile boundaries in M
    ([37, 200, 0, 64], 72, 200),                            # ragged K (72) and N (200) tails
    ([513], 256, 1024),                                     # one expert, several M tiles
    ([3, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 2], 64, 64),         # mostly empty experts
])
def test_grouped_ffn_tile_edges(dtype, sizes, d, ff):
    E = len(sizes)
    R = sum(sizes)
    max_rows = R + 17
    inp = wl.draw_custom(11, T=max_rows, d=d, ff=ff, E=E, dtype=dtype)
    dt = dtype_code(dtype)
    params = MoEParams.from_arrays(inp, dt, DEV)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rg = np.random.default_rng(1).random(max_rows).astype(np.float32)
    xp = to_device(inp["x"], dt, DEV)
    h, yp = run_ffn(xp, torch.from_numpy(offsets).to(DEV), max_rows, params, torch.from_numpy(rg).to(DEV))
    ref_y = moe_ref.grouped_ffn(inp["x"][:R], offsets, inp, rg[:R])
    assert pu.max_rel_err(yp[:R], ref_y) <= pu.TOL[dtype]
    ref_h = np.concatenate([moe_ref.fc1_gelu(inp["x"][offsets[e]:offsets[e + 1]], inp["w1"][e], inp["b1"][e])
                            for e in range(E)] + [np.zeros((0, ff))])
    assert pu.max_rel_err(h[:R], ref_h) <= pu.TOL[dtype]
    assert np.isnan(yp[R:]).all()          # rows past R are not written


def test_device_gelu_forms_match_erf():
    """The device GELU forms against CUDA's erff form and the float64 definition:
    the A&S 7.1.26 erf is within its published bound (1.5e-7) plus fp32 rounding,
    and the paired-instruction form the bf16 epilogue runs (variant 2) equals the
    scalar one bit for bit, odd element count included."""
    xs = np.concatenate([np.linspace(-12, 12, 200001),
                         [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 3e-39, 0.5]]).astype(np.float32)
    x = torch.from_numpy(xs).to(DEV)
    y0 = torch.empty_like(x)
    y1 = torch.empty_like(x)
    y2 = torch.empty_like(x)
    _lib.moe_debug_gelu(x, y0, x.numel(), 0)
    _lib.moe_debug_gelu(x, y1, x.numel(), 1)
    _lib.moe_debug_gelu(x, y2, x.numel(), 2)
    assert x.numel() % 2 == 1
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    y0, y1 = y0.cpu().double().numpy(), y1.cpu().double().numpy()
    ref = moe_ref.gelu(xs.astype(np.float64))
    scale = np.maximum(np.abs(xs.astype(np.float64)), 1.0)
    assert np.max(np.abs(y0 - ref) / scale) <= 2e-7
    assert np.max(np.abs(y1 - ref) / scale) <= 0.5 * 1.5e-7 + 4e-7
    assert np.max(np.abs(y1 - y0) / scale) <= 6e-7
    assert y1[np.argmin(np.abs(xs))] == 0.0


# ---------------------------------------------------------------------------
# the whole layer (and step 4, combine)
# ---------------------------------------------------------------------------
def oracle_on_gpu_routing(inp, w, idx_gpu, rows=None):
    """The oracle's layer output given the GPU's expert choice (gates are the
    oracle's softmax values at those experts)."""
    r = moe_ref.route(inp["x"], inp["w_router"], w.k, inp["logit_bias"])
    gates = np.take_along_axis(r["gates"], idx_gpu.astype(np.int64), 1)
    cap = moe_ref.capacity(w.T, w.k, w.E, w.cf)
    dsp = moe_ref.dispatch(idx_gpu, w.E, cap)
    if rows is None:
        out = moe_ref.moe_forward(inp["x"], inp, idx_gpu, gates, dsp["slot_of"])
    else:
        out = moe_ref.moe_forward_rows(inp["x"], inp, idx_gpu, gates, dsp["slot_of"], rows)
    return out, dsp, r


@pytest.mark.parametrize("w", VARIANTS, ids=VARIANT_IDS)
def test_forward_matches_oracle(w):
    inp = inputs_for(w)
    dt = dtype_code(w.dtype)
    params = MoEParams.from_arrays(inp, dt, DEV)
    cap = _lib.moe_capacity(w.T, w.k, w.E, w.cf)
    layer = MoELayer(params, w.k, cap)
    x = to_device(inp["x"], dt, DEV)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=DEV)
    out = layer.forward(x, stats=True, topk_idx=idx)
    assert _lib.moe_get_error() == _lib.MOE_OK
    out_np = out.float().cpu().numpy()
    idx_np = idx.cpu().numpy()
    assert out_np.shape == inp["x"].shape and np.isfinite(out_np).all()
    if w.name in FULL_ORACLE:
        ref, dsp, r = oracle_on_gpu_routing(inp, w, idx_np)
        got = out_np
    else:
        dsp0 = moe_ref.dispatch(idx_np, w.E, cap)
        hot = np.nonzero(idx_np[:, 0] == np.bincount(idx_np.ravel()).argmax())[0][:8]
        dropped = np.nonzero((dsp0["slot_of"].reshape(w.T, w.k) < 0).any(1))[0][:8]
        # one row of every 128-row M tile of every expert group (so every
        # 256-row CTA-pair tile too), plus random, hot-expert and dropped rows
        tiles = pu.tile_covering_rows(dsp0["offsets"], dsp0["perm"], w.k, w.T, seed=w.seed)
        rows = pu.sample_rows(w.T, 96, seed=w.seed, must=list(hot) + list(dropped) + list(tiles))
        print(f"{w.name}: {len(rows)} sampled output rows reach all {pu.m_tiles(dsp0['offsets'])} "
              f"128-row M tiles ({pu.m_tiles(dsp0['offsets'], 256)} 256-row tiles)")
        ref, dsp, r = oracle_on_gpu_routing(inp, w, idx_np, rows)
        got = out_np[rows]
    err = pu.max_rel_err(got, ref)
    assert err <= pu.TOL[w.dtype], err
    # the fused forward dispatch: bit-exact with the oracle's on the GPU's routing
    A = w.T * w.k
    R = int(dsp["offsets"][-1])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "counts", torch.int32, w.E).cpu().numpy(), dsp["counts"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "offsets", torch.int32, w.E + 1).cpu().numpy(),
                                  dsp["offsets"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "perm", torch.int32, R).cpu().numpy(), dsp["perm"])
    np.testing.assert_array_equal(layer.workspace_view(w.T, "slot_of", torch.int32, A).cpu().numpy(),
                                  dsp["slot_of"])
    gate_gpu = layer.workspace_view(w.T, "topk_gate", torch.float32, A).cpu().numpy()
    np.testing.assert_array_equal(layer.workspace_view(w.T, "row_gate", torch.float32, R).cpu().numpy(),
                                  gate_gpu[dsp["perm"]])
    # tokens whose every assignment was dropped produce exactly 0
    all_dropped = (dsp["slot_of"].reshape(w.T, w.k) < 0).all(1)
    assert np.all(out_np[all_dropped] == 0.0)
    # statistics
    st = read_stats(layer.stats_buf)
    ref_st = moe_ref.layer_stats(idx_np, r["gates"], w.E, cap)
    assert st["rows_kept"] == ref_st["rows_kept"] and st["dropped"] == ref_st["dropped"]
    assert st["max_count"] == ref_st["max_count"]
    assert st["imbalance"] == pytest.approx(ref_st["imbalance"], rel=1e-6)
    assert st["drop_rate"] == pytest.approx(ref_st["drop_rate"], rel=1e-6, abs=1e-7)
    assert st["aux_loss"] == pytest.approx(ref_st["aux_loss"], rel=1e-4)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,d,ff,E,k,cap", [
    (1000, 72, 200, 5, 2, -1),       # ragged everywhere
    (777, 64, 128, 1, 1, -1),        # one expert: a plain MLP
    (300, 64, 64, 4, 4, -1),         # k = E
    (500, 64, 64, 8, 2, 0),          # capacity 0: every assignment dropped
    (2000, 128, 256, 16, 2, 60),     # capacity drops on a top-2 layer
    (1, 64, 64, 8, 2, -1),           # one token
    (1000, 520, 256, 40, 3, 700),    # ragged last router tile, K tail (520 = 8 * 64 + 8), k = 3
    (600, 64, 64, 256, 8, -1),       # the most experts and slots: 256 experts, top-8
    (2000, 256, 4096, 8, 1, -1),     # few tiles, long fc2 K, ragged rows
    (1500, 256, 2048, 6, 2, 300),    # k = 2 with capacity drops, long fc2 K
    # >= 384 rows per expert: bf16 runs the CTA-pair (256-row tile) kernels
    (4000, 72, 200, 4, 1, -1),       # pairs, ragged K and N tails, direct fc2 output
    (5000, 128, 256, 8, 2, 900),     # pairs with capacity drops, k = 2
    (6000, 64, 128, 4, 1, 1400),     # pairs, top-1 with drops (zeroed rows)
    (3333, 192, 1088, 3, 1, -1),     # pairs, ragged last 256-row tile and N tail
])
def test_forward_edge_cases(dtype, T, d, ff, E, k, cap):
    inp = wl.draw_custom(5, T=T, d=d, ff=ff, E=E, dtype=dtype, router_std=0.5)
    dt = dtype_code(dtype)
    params = MoEParams.from_arrays(inp, dt, DEV)
    layer = MoELayer(params, k, cap)
    x = to_device(inp["x"], dt, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    out = layer.forward(x, topk_idx=idx).float().cpu().numpy()
    assert _lib.moe_get_error() == _lib.MOE_OK
    idx_np = idx.cpu().numpy()
    r = moe_ref.route(inp["x"], inp["w_router"], k)
    gates = np.take_along_axis(r["gates"], idx_np.astype(np.int64), 1)
    dsp = moe_ref.dispatch(idx_np, E, cap)
    ref = moe_ref.moe_forward(inp["x"], inp, idx_np, gates, dsp["slot_of"])
    if cap == 0:
        assert np.all(out == 0.0)
    else:
        assert pu.max_rel_err(out, ref) <= pu.TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_combine_matches_oracle(dtype):
    T, k, d = 999, 3, 136
    rng = np.random.default_rng(4)
    R = 2400
    yp = rng.normal(size=(R, d)).astype(np.float32)
    slot = rng.permutation(T * k).astype(np.int32)
    slot[slot >= R] = -1
    gate = rng.random((T, k)).astype(np.float32)
    dt = dtype_code(dtype)
    yp_dev = to_device(yp, dt, DEV)
    yp_used = yp_dev.float().cpu().numpy()
    out = torch.empty((T, d), dtype=yp_dev.dtype, device=DEV)
    for g in (None, gate):
        _lib.moe_combine(yp_dev, torch.from_numpy(slot).to(DEV),
                         None if g is None else torch.from_numpy(g).to(DEV), T, k, d, dt, out)
        ref = moe_ref.combine(yp_used, slot, T, k, g)
        assert pu.max_rel_err(out.float().cpu().numpy(), ref) <= (4e-3 if dtype == "bf16" else 1e-6)


def test_forward_is_deterministic():
    w = wl.workload("switch-top1", dtype="bf16", cf=1.0)
    inp = inputs_for(w)
    params = MoEParams.from_arrays(inp, _lib.MOE_BF16, DEV)
    layer = MoELayer(params, w.k, _lib.moe_capacity(w.T, w.k, w.E, w.cf))
    x = to_device(inp["x"], _lib.MOE_BF16, DEV)
    a = layer.forward(x).clone()
    b = layer.forward(x).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_launch_counter_and_timing():
    w = wl.workload("dense-top2-f32")
    inp = inputs_for(w)
    params = MoEParams.from_arrays(inp, _lib.MOE_F32, DEV)
    layer = MoELayer(params, w.k, -1)
    x = to_device(inp["x"], _lib.MOE_F32, DEV)
    layer.forward(x)
    _lib.moe_timing_enable(True)
    _lib.moe_timing_read()
    n0 = _lib.moe_launch_count()
    layer.forward(x, stats=True)
    torch.cuda.synchronize()
    launched = _lib.moe_launch_count() - n0
    t = _lib.moe_timing_read()
    _lib.moe_timing_enable(False)
    # router, dispatch (scan + permute + gather), ffn1, ffn2, combine (k = 2)
    assert launched == 5
    assert sum(n for _, n in t.values()) == 5
    assert all(ms > 0 for ms, n in t.values() if n)
