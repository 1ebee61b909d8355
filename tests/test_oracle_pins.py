"""Pins for the float64 oracle: each check ties an oracle function to something
other than itself -- a library routine, a closed form, brute force on tiny
inputs, or one of the invariants the cookbook notebook "Mixture-of-experts and
expert parallelism" checks (sections "Dispatch and gather", "Capacity factor",
"Switch Transformer auxiliary loss").  The last block plants plausible
mistakes in the oracle and shows that a pin catches each one.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import moe_ref
from mixture_experts_layer_45_b200 import workloads as wl


def _tiny(seed, T=48, d=24, ff=40, E=6, dtype="f32"):
    return wl.draw_custom(seed, T=T, d=d, ff=ff, E=E, dtype=dtype, router_std=0.3)


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def check_router_logits_vs_torch(inp):
    ref = F.linear(torch.from_numpy(inp["x"]).double(),
                   torch.from_numpy(inp["w_router"]).double()).numpy()
    got = moe_ref.router_logits(inp["x"], inp["w_router"])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def check_softmax_vs_library(logits):
    got = moe_ref.softmax(logits)
    np.testing.assert_allclose(got, scipy.special.softmax(logits, axis=-1), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(got.sum(-1), 1.0, rtol=0, atol=1e-13)


def check_topk_vs_stable_argsort(logits, k):
    ref = np.argsort(-np.asarray(logits), axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(moe_ref.topk(logits, k), ref)


def check_route_gates_are_raw_probs(inp, k):
    r = moe_ref.route(inp["x"], inp["w_router"], k)
    probs = scipy.special.softmax(F.linear(torch.from_numpy(inp["x"]).double(),
                                           torch.from_numpy(inp["w_router"]).double()).numpy(), axis=-1)
    np.testing.assert_allclose(r["topk_gate"], np.take_along_axis(probs, r["topk_idx"], 1),
                               rtol=1e-12, atol=0)
    assert np.all(np.diff(r["topk_gate"], axis=1) <= 0), "gates must be in descending order"


def test_router_logits_match_torch_linear():
    check_router_logits_vs_torch(_tiny(1))


def test_softmax_matches_scipy():
    rng = np.random.default_rng(0)
    check_softmax_vs_library(rng.normal(size=(64, 9)) * 30.0)


@pytest.mark.parametrize("k", [1, 2, 3, 6])
def test_topk_matches_stable_argsort_random(k):
    rng = np.random.default_rng(k)
    check_topk_vs_stable_argsort(rng.normal(size=(200, 6)), k)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_topk_ties_go_to_lower_index(k):
    rng = np.random.default_rng(7)
    logits = rng.integers(0, 3, size=(300, 8)).astype(np.float64)   # many exact ties
    check_topk_vs_stable_argsort(logits, k)
    # a row of all-equal logits picks 0, 1, ..., k-1
    np.testing.assert_array_equal(moe_ref.topk(np.zeros((1, 8)), k)[0], np.arange(k))


@pytest.mark.parametrize("k", [1, 2])
def test_topk_gates_are_raw_probabilities(k):
    check_route_gates_are_raw_probs(_tiny(2), k)


def test_k_equals_E_gates_sum_to_one():
    inp = _tiny(3, E=5)
    r = moe_ref.route(inp["x"], inp["w_router"], 5)
    np.testing.assert_allclose(r["topk_gate"].sum(1), 1.0, atol=1e-13)


def test_logit_bias_shifts_logits():
    inp = _tiny(4)
    b = np.linspace(-1, 1, 6).astype(np.float32)
    got = moe_ref.router_logits(inp["x"], inp["w_router"], b)
    ref = F.linear(torch.from_numpy(inp["x"]).double(), torch.from_numpy(inp["w_router"]).double(),
                   torch.from_numpy(b).double()).numpy()
    np.testing.assert_allclose(got, ref, atol=1e-12)


# ---------------------------------------------------------------------------
# counts, capacity, dispatch
# ---------------------------------------------------------------------------

def check_dispatch_vs_stable_sort(idx, E, cap):
    d = moe_ref.dispatch(idx, E, cap)
    flat = np.asarray(idx).reshape(-1)
    order = np.argsort(flat, kind="stable")                     # library stable sort
    counts = np.bincount(flat, minlength=E)
    np.testing.assert_array_equal(d["counts"], counts)
    kept = counts if cap < 0 else np.minimum(counts, cap)
    np.testing.assert_array_equal(d["kept"], kept)
    starts = np.concatenate([[0], np.cumsum(counts)])
    ref_perm = np.concatenate([order[starts[e]:starts[e] + kept[e]] for e in range(E)])
    np.testing.assert_array_equal(d["perm"], ref_perm)
    np.testing.assert_array_equal(d["offsets"], np.concatenate([[0], np.cumsum(kept)]))
    np.testing.assert_array_equal(d["slot_of"][d["perm"]], np.arange(len(ref_perm)))
    assert d["drop_mask"].sum() == (counts - kept).sum() == flat.size - len(ref_perm)
    return d


@pytest.mark.parametrize("cap", [-1, 0, 1, 3, 10, 1000])
def test_dispatch_matches_stable_argsort(cap):
    rng = np.random.default_rng(11)
    idx = np.stack([rng.permutation(7)[:3] for _ in range(57)])   # T=57, k=3, E=7, distinct per token
    check_dispatch_vs_stable_sort(idx, 7, cap)


def test_counts_sum_to_T_times_k_and_active_ratio():
    w = wl.workload("dense-top2-f32")
    inp = wl.draw_router_inputs(w)
    r = moe_ref.route(inp["x"], inp["w_router"], w.k)
    counts = moe_ref.token_count_per_expert(r["topk_idx"], w.E)
    assert counts.sum() == w.T * w.k
    # active expert fraction per token, measured from the routing: exactly k/E
    assert Fraction(int(counts.sum()), w.T * w.E) == Fraction(w.k, w.E)


def test_capacity_closed_form():
    assert moe_ref.capacity(4096, 1, 32, 1.0) == 128
    assert moe_ref.capacity(4096, 1, 32, 1.5) == 192
    assert moe_ref.capacity(16384, 1, 64, 1.25) == 320
    assert moe_ref.capacity(10, 1, 3, 1.0) == 3            # int() truncates 3.33
    assert moe_ref.capacity(1024, 2, 8, None) == -1
    assert moe_ref.capacity(1024, 2, 8, 0.0) == -1


def test_drop_rate_closed_form_and_monotone():
    w = wl.workload("switch-top1", dtype="f32")
    inp = wl.draw_router_inputs(w)
    idx = moe_ref.route(inp["x"], inp["w_router"], w.k)["topk_idx"]
    drops = {}
    for cf in (1.0, 1.5):
        cap = moe_ref.capacity(w.T, w.k, w.E, cf)
        d = moe_ref.dispatch(idx, w.E, cap)
        counts = np.bincount(idx.ravel(), minlength=w.E)
        closed = sum(max(int(c) - cap, 0) for c in counts) / (w.T * w.k)
        assert moe_ref.drop_rate(d["counts"], cap) == pytest.approx(closed, abs=0)
        assert d["drop_mask"].sum() / (w.T * w.k) == pytest.approx(closed, abs=0)
        drops[cf] = closed
    assert drops[1.5] <= drops[1.0]
    assert drops[1.0] > 0        # the untrained router overflows some expert at cf 1.0


# A hand-built top-2 routing of T = 10 tokens over E = 4 experts.  Counting
# by hand: expert 0 is in rows 0-7 (8), expert 1 in rows 0, 3, 5, 8, 9 (5),
# expert 2 in rows 1, 4, 7, 8 (4), expert 3 in rows 2, 6, 9 (3); 20 = T*k.
_HAND_IDX = np.array([[0, 1], [0, 2], [0, 3], [0, 1], [0, 2], [0, 1], [0, 3], [0, 2], [1, 2], [3, 1]])
_HAND_COUNTS = [8, 5, 4, 3]


def check_imbalance_closed_form():
    """The notebook's imbalance ratio ("Capacity factor") is the largest
    count over the balanced load T*k/E.  Hand-worked: T*k/E = 10*2/4 = 5,
    so 8/5 = 1.6 (a T/E denominator would give 3.2).  Round-robin routing
    loads every expert with exactly T*k/E assignments: 1.0."""
    np.testing.assert_array_equal(moe_ref.token_count_per_expert(_HAND_IDX, 4), _HAND_COUNTS)
    assert moe_ref.imbalance(np.array(_HAND_COUNTS), 10, 2, 4) == pytest.approx(1.6, abs=1e-15)
    st = moe_ref.layer_stats(_HAND_IDX, np.full((10, 4), 0.25), 4, -1)
    assert st["imbalance"] == pytest.approx(1.6, abs=1e-15) and st["max_count"] == 8
    for T, k, E in ((64, 2, 8), (96, 1, 32), (40, 2, 4)):
        rr = (np.arange(T * k) % E).reshape(T, k)
        assert moe_ref.imbalance(moe_ref.token_count_per_expert(rr, E), T, k, E) == 1.0


def test_imbalance_closed_form():
    check_imbalance_closed_form()


def check_layer_stats_drops_are_capacity_check():
    """Without rerouting, the statistics' drop count and rate are the
    notebook's capacity_check ("Capacity factor"): sum(max(counts - cap, 0))
    and that over counts.sum() = T*k.  Hand-worked on _HAND_IDX: cap 4 drops
    (8-4) + (5-4) = 5 of 20 (0.25), cap 5 drops 3 (0.15), cap 2 drops
    6+3+2+1 = 12 (0.6), no limit drops nothing."""
    gates = np.full((10, 4), 0.25)
    for cap, dropped in ((4, 5), (5, 3), (2, 12), (8, 0), (0, 20), (-1, 0)):
        st = moe_ref.layer_stats(_HAND_IDX, gates, 4, cap)
        closed = sum(max(c - cap, 0) for c in _HAND_COUNTS) if cap >= 0 else 0
        assert closed == dropped
        assert st["dropped"] == dropped and st["rows_kept"] == 20 - dropped
        assert st["drop_rate"] == pytest.approx(dropped / 20, abs=1e-15)
        assert st["drop_rate"] == pytest.approx(moe_ref.drop_rate(_HAND_COUNTS, cap), abs=1e-15)
    # and on a seeded routing, against the dispatch's own drop mask
    w = wl.workload("switch-top1", dtype="f32")
    inp = wl.draw_router_inputs(w)
    r = moe_ref.route(inp["x"], inp["w_router"], w.k)
    for cf in (1.0, 1.5):
        cap = moe_ref.capacity(w.T, w.k, w.E, cf)
        st = moe_ref.layer_stats(r["topk_idx"], r["gates"], w.E, cap)
        counts = moe_ref.token_count_per_expert(r["topk_idx"], w.E)
        assert st["drop_rate"] == pytest.approx(moe_ref.drop_rate(counts, cap), abs=1e-15)
        assert st["dropped"] == int(moe_ref.dispatch(r["topk_idx"], w.E, cap)["drop_mask"].sum())


def test_layer_stats_drops_are_capacity_check():
    check_layer_stats_drops_are_capacity_check()


# ---------------------------------------------------------------------------
# GELU, expert FFN, combine
# ---------------------------------------------------------------------------

def check_gelu(gelu):
    v = np.array([-10.0, -3.0, -1.0, -0.5, -1e-3, 0.0, 1e-3, 0.5, 1.0, 3.0, 10.0, 40.0])
    ref = np.array([0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0))) for t in v])
    np.testing.assert_allclose(gelu(v), ref, rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(gelu(v), F.gelu(torch.from_numpy(v)).numpy(), rtol=1e-14, atol=1e-300)
    assert gelu(np.array([0.0]))[0] == 0.0
    assert abs(gelu(np.array([40.0]))[0] - 40.0) == 0.0
    assert abs(gelu(np.array([-40.0]))[0]) < 1e-300


def test_gelu_exact_erf_form():
    check_gelu(moe_ref.gelu)


def check_single_expert_is_mlp(inp):
    """E = 1, k = 1: the gate is 1 and the layer is fc2(gelu(fc1(x)))."""
    x = torch.from_numpy(inp["x"]).double()
    h = F.gelu(F.linear(x, torch.from_numpy(inp["w1"][0]).double(), torch.from_numpy(inp["b1"][0]).double()))
    ref = F.linear(h, torch.from_numpy(inp["w2"][0]).double(), torch.from_numpy(inp["b2"][0]).double()).numpy()
    out = moe_ref.moe_layer(inp, k=1, cap=-1)["out"]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_single_expert_top1_is_plain_mlp():
    check_single_expert_is_mlp(_tiny(5, E=1))


def brute_force_dense(inp, idx, gates, slot_of):
    """Every expert on every token, then a per-token mask of kept gates."""
    x = np.asarray(inp["x"], np.float64)
    T, k = idx.shape
    E = inp["w1"].shape[0]
    out = np.zeros_like(x)
    for e in range(E):
        h = x @ inp["w1"][e].astype(np.float64).T + inp["b1"][e]
        h = 0.5 * h * (1.0 + scipy.special.erf(h / np.sqrt(2.0)))
        y = h @ inp["w2"][e].astype(np.float64).T + inp["b2"][e]
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e and slot_of[t * k + j] >= 0:
                    out[t] += gates[t, j] * y[t]
    return out


def check_forward_vs_brute_force(inp, k, cap):
    E = inp["w1"].shape[0]
    res = moe_ref.moe_layer(inp, k=k, cap=cap)
    ref = brute_force_dense(inp, res["topk_idx"], res["topk_gate"], res["slot_of"])
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)
    # the dispatched form (grouped FFN on the permuted rows, then combine) agrees
    xp = np.asarray(inp["x"], np.float64)[res["perm"] // k]
    row_gate = res["topk_gate"].reshape(-1)[res["perm"]]
    yp = moe_ref.grouped_ffn(xp, res["offsets"], inp, row_gate)
    out2 = moe_ref.combine(yp, res["slot_of"], inp["x"].shape[0], k)
    np.testing.assert_allclose(out2, ref, rtol=0, atol=1e-12)
    rows = np.array([0, 3, inp["x"].shape[0] - 1])
    np.testing.assert_allclose(
        moe_ref.moe_forward_rows(inp["x"], inp, res["topk_idx"], res["topk_gate"], res["slot_of"], rows),
        ref[rows], rtol=0, atol=1e-12)
    return res


@pytest.mark.parametrize("k,cap", [(1, -1), (2, -1), (2, 5), (1, 4), (3, 2), (6, -1)])
def test_forward_matches_brute_force_dense(k, cap):
    res = check_forward_vs_brute_force(_tiny(10 + k), k, cap)
    if cap >= 0:
        assert res["drop_mask"].sum() > 0     # the case really drops something
        dropped_all = (res["slot_of"].reshape(-1, k) < 0).all(1)
        assert np.all(res["out"][dropped_all] == 0.0)


def test_forward_bf16_rounded_inputs_brute_force():
    check_forward_vs_brute_force(_tiny(21, dtype="bf16"), 2, 9)


# ---------------------------------------------------------------------------
# shared always-on experts (notebook section "Exercises", item 3)
# ---------------------------------------------------------------------------

def _torch_mlp(x, w1, b1, w2, b2):
    """fc2(gelu(fc1(x))) with torch's float64 Linear and exact GELU."""
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    h = F.gelu(F.linear(t(x), t(w1), t(b1)))
    return F.linear(h, t(w2), t(b2)).numpy()


def _routed_only(inp):
    return {key: v for key, v in inp.items() if not key.startswith("shared_")}


def check_shared_experts_added_ungated(inp, k, cap):
    """With shared experts the output gains, on every token (dropped or not),
    the plain sum of the shared MLPs; routing, dispatch and statistics are
    those of the routed layer alone."""
    res = moe_ref.moe_layer(inp, k=k, cap=cap)
    base = moe_ref.moe_layer(_routed_only(inp), k=k, cap=cap)
    S = inp["shared_w1"].shape[0]
    ref = sum(_torch_mlp(inp["x"], inp["shared_w1"][s], inp["shared_b1"][s],
                         inp["shared_w2"][s], inp["shared_b2"][s]) for s in range(S))
    np.testing.assert_allclose(res["out"] - base["out"], ref, rtol=0, atol=1e-12)
    for key in ("topk_idx", "topk_gate", "perm", "slot_of", "offsets", "counts"):
        assert np.array_equal(res[key], base[key]), key
    assert res["stats"] == base["stats"]
    # per-expert outputs, in order
    ys = moe_ref.shared_expert_outputs(inp["x"], inp)
    assert ys.shape == (S,) + inp["x"].shape
    for s in range(S):
        np.testing.assert_allclose(ys[s], _torch_mlp(inp["x"], inp["shared_w1"][s], inp["shared_b1"][s],
                                                     inp["shared_w2"][s], inp["shared_b2"][s]),
                                   rtol=0, atol=1e-12)
    return res, ref


@pytest.mark.parametrize("k,cap,S", [(1, -1, 1), (2, -1, 2), (2, 5, 2), (1, 4, 3)])
def test_shared_experts_add_plain_mlps(k, cap, S):
    inp = wl.draw_custom(30 + S, T=48, d=24, ff=40, E=6, dtype="f32", router_std=0.3, shared=S)
    res, ref = check_shared_experts_added_ungated(inp, k, cap)
    if cap >= 0:
        dropped_all = (res["slot_of"].reshape(-1, k) < 0).all(1)
        assert dropped_all.any()
        # a token with every assignment dropped receives exactly the shared sum
        np.testing.assert_allclose(res["out"][dropped_all], ref[dropped_all], rtol=0, atol=1e-12)


def test_shared_experts_with_zero_capacity_is_shared_sum():
    inp = wl.draw_custom(41, T=20, d=16, ff=24, E=4, dtype="bf16", router_std=0.3, shared=2)
    res = moe_ref.moe_layer(inp, k=2, cap=0)
    assert (res["slot_of"] < 0).all()
    np.testing.assert_allclose(res["out"], moe_ref.shared_experts(inp["x"], inp), rtol=0, atol=0)
    check_shared_experts_added_ungated(inp, 2, 0)


def test_shared_expert_equals_routed_single_expert_layer():
    """A shared expert is the E = 1, k = 1 routed layer (gate softmax over one
    expert = 1, no capacity) with the same weights."""
    inp = wl.draw_custom(43, T=32, d=16, ff=24, E=3, dtype="f32", router_std=0.3, shared=2)
    for s in range(2):
        single = {"x": inp["x"], "w_router": inp["w_router"][:1], "logit_bias": None,
                  "w1": inp["shared_w1"][s:s + 1], "b1": inp["shared_b1"][s:s + 1],
                  "w2": inp["shared_w2"][s:s + 1], "b2": inp["shared_b2"][s:s + 1]}
        np.testing.assert_allclose(moe_ref.shared_expert_outputs(inp["x"], inp)[s],
                                   moe_ref.moe_layer(single, k=1, cap=-1)["out"], rtol=0, atol=1e-12)


def test_shared_rows_match_full_layer():
    inp = wl.draw_custom(44, T=40, d=16, ff=24, E=5, dtype="f32", router_std=0.3, shared=2)
    res = moe_ref.moe_layer(inp, k=2, cap=6)
    rows = np.array([0, 7, 39])
    np.testing.assert_allclose(
        moe_ref.moe_forward_rows_shared(inp["x"], inp, res["topk_idx"], res["topk_gate"], res["slot_of"], rows),
        res["out"][rows], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# overflow rerouting (dispatch_reroute)
# ---------------------------------------------------------------------------

def _ranked(rows):
    idx = np.array(rows, dtype=np.int64)
    gate = (idx + 1) / 100.0 + np.arange(idx.shape[0])[:, None] / 1000.0   # distinct, traceable gates
    return idx, gate


def check_reroute_hand_example_top1():
    """Worked by hand.  E = 4, k = 1, cap = 2, two rounds.
    Own choices: tokens 0-4 pick expert 0, token 5 expert 1, token 6 expert 2.
    Expert 0 keeps tokens 0, 1 and drops 2, 3, 4 (loads 2, 1, 1, 0).
    Round 1 offers (second choices): t2 -> 1 (accepted, load 2), t3 -> 1
    (full), t4 -> 2 (accepted, load 2).  Round 2: t3 -> its third choice 3
    (accepted).  Rows: e0 [t0 t1], e1 [t5 t2], e2 [t6 t4], e3 [t3]."""
    idx, gate = _ranked([[0, 1, 2], [0, 1, 2], [0, 1, 2], [0, 1, 3], [0, 2, 1], [1, 0, 2], [2, 0, 1]])
    res = moe_ref.dispatch_reroute(idx, gate, 1, 4, 2, 2)
    np.testing.assert_array_equal(res["perm"], [0, 1, 5, 2, 6, 4, 3])
    np.testing.assert_array_equal(res["offsets"], [0, 2, 4, 6, 7])
    np.testing.assert_array_equal(res["slot_of"], [0, 1, 3, 6, 5, 2, 4])
    np.testing.assert_array_equal(res["final_idx"][:, 0], [0, 0, 1, 3, 2, 1, 2])
    np.testing.assert_array_equal(res["final_gate"][:, 0],
                                  [gate[0, 0], gate[1, 0], gate[2, 1], gate[3, 2], gate[4, 1], gate[5, 0], gate[6, 0]])
    np.testing.assert_array_equal(res["counts"], [5, 1, 1, 0])
    np.testing.assert_array_equal(res["kept_primary"], [2, 1, 1, 0])
    assert res["rerouted"] == 3 and res["drop_mask"].sum() == 0
    # one round only: token 3 stays dropped
    one = moe_ref.dispatch_reroute(idx, gate, 1, 4, 2, 1)
    np.testing.assert_array_equal(one["slot_of"], [0, 1, 3, -1, 5, 2, 4])
    assert one["rerouted"] == 2


def check_reroute_hand_example_top2():
    """Worked by hand.  E = 4, k = 2, cap = 1, two rounds.  Tokens 0 and 1
    choose (0, 1) with fallbacks (2, 3); token 2 chooses (1, 0), fallbacks
    (3, 2).  Kept: a0 = (t0, slot 0) at expert 0, a1 = (t0, 1) at expert 1.
    Round 1: t1 offers its first dropped slot (slot 0) to expert 2
    (accepted); t2 offers slot 0 to expert 3 (accepted).  Round 2: t1 offers
    slot 1 to expert 3, t2 slot 1 to expert 2: both full."""
    idx, gate = _ranked([[0, 1, 2, 3], [0, 1, 2, 3], [1, 0, 3, 2]])
    res = moe_ref.dispatch_reroute(idx, gate, 2, 4, 1, 2)
    np.testing.assert_array_equal(res["perm"], [0, 1, 2, 4])
    np.testing.assert_array_equal(res["offsets"], [0, 1, 2, 3, 4])
    np.testing.assert_array_equal(res["slot_of"], [0, 1, 2, -1, 3, -1])
    np.testing.assert_array_equal(res["final_idx"], [[0, 1], [2, 1], [3, 0]])
    assert res["final_gate"][1, 0] == gate[1, 2] and res["final_gate"][2, 0] == gate[2, 2]
    assert res["rerouted"] == 2


def test_reroute_hand_worked_examples():
    check_reroute_hand_example_top1()
    check_reroute_hand_example_top2()


def _random_ranked(seed, T, E, kk):
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.ones(E) * 0.4)
    idx = np.stack([rng.choice(E, size=kk, replace=False, p=p) for _ in range(T)])
    return idx, rng.random((T, kk))


@pytest.mark.parametrize("T,E,k,cap,rounds,seed", [(200, 8, 1, 20, 1, 0), (300, 6, 2, 70, 3, 1),
                                                   (150, 16, 1, 3, 4, 2), (100, 5, 3, 40, 2, 3),
                                                   (64, 4, 1, 0, 2, 4)])
def test_reroute_invariants(T, E, k, cap, rounds, seed):
    idx, gate = _random_ranked(seed, T, E, k + rounds)
    res = moe_ref.dispatch_reroute(idx, gate, k, E, cap, rounds)
    base = moe_ref.dispatch(idx[:, :k], E, cap)
    # the router's choices are dispatched as before; rerouting only adds rows
    np.testing.assert_array_equal(res["counts"], base["counts"])
    np.testing.assert_array_equal(res["kept_primary"], base["kept"])
    assert np.all(res["kept"] <= cap) and np.all(res["kept"] >= base["kept"])
    np.testing.assert_array_equal(np.diff(res["offsets"]), res["kept"])
    served = res["slot_of"] >= 0
    assert np.all(served[base["slot_of"] >= 0])
    assert res["rerouted"] == int(served.sum() - (base["slot_of"] >= 0).sum())
    assert sorted(res["perm"]) == sorted(np.nonzero(served)[0])
    fi = res["final_idx"]
    for t in range(T):
        used = [fi[t, j] for j in range(k) if served[t * k + j]]
        assert len(set(used)) == len(used)            # never the same expert twice
    # each row belongs to its expert; within an expert: own rows in token
    # order first, then rerouted rows by (round, token)
    for e in range(E):
        rows = res["perm"][res["offsets"][e]:res["offsets"][e + 1]]
        keys = []
        for a in rows:
            t, j = divmod(int(a), k)
            assert fi[t, j] == e
            pos = list(idx[t]).index(e)
            rnd = 0 if pos < k else pos - k + 1
            assert rnd == 0 or res["final_gate"][t, j] == gate[t, pos]
            keys.append((rnd, t))
        assert keys == sorted(keys)
    # an offer is refused only when the expert is full by the end of its round
    if cap == 0:
        assert res["rerouted"] == 0 and not served.any()


def test_reroute_one_round_top1_closed_form():
    """k = 1, one round: expert c takes, in token order, the first
    cap - kept_c dropped tokens whose second choice is c (a stable sort)."""
    T, E, cap = 500, 10, 35
    idx, gate = _random_ranked(7, T, E, 2)
    res = moe_ref.dispatch_reroute(idx, gate, 1, E, cap, 1)
    base = moe_ref.dispatch(idx[:, :1], E, cap)
    dropped = np.nonzero(base["slot_of"] < 0)[0]
    second = idx[dropped, 1]
    order = np.argsort(second, kind="stable")
    expect = np.zeros(T, bool)
    for c in range(E):
        mine = dropped[order][second[order] == c]
        expect[mine[:cap - base["kept"][c]]] = True
    np.testing.assert_array_equal((res["slot_of"] >= 0) & (base["slot_of"] < 0), expect)


def test_reroute_degenerate_cases():
    idx, gate = _random_ranked(9, 120, 6, 4)
    base = moe_ref.dispatch(idx[:, :2], 6, 25)
    zero = moe_ref.dispatch_reroute(idx, gate, 2, 6, 25, 0)
    for key in ("counts", "offsets", "perm", "slot_of", "drop_mask"):
        np.testing.assert_array_equal(zero[key], base[key])
    unlimited = moe_ref.dispatch_reroute(idx, gate, 2, 6, -1, 2)
    plain = moe_ref.dispatch(idx[:, :2], 6, -1)
    np.testing.assert_array_equal(unlimited["perm"], plain["perm"])
    assert unlimited["rerouted"] == 0


def check_reroute_forward_vs_brute_force(inp, k, cap, rounds):
    res = moe_ref.moe_layer(inp, k=k, cap=cap, reroute=rounds)
    ref = brute_force_dense(inp, res["final_idx"], res["final_gate"], res["slot_of"])
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)
    # the router's full softmax gives the fallback gates
    np.testing.assert_allclose(res["final_gate"], np.take_along_axis(res["gates"], res["final_idx"], 1),
                               rtol=0, atol=0)
    st = res["stats"]
    assert st["rows_kept"] == int((res["slot_of"] >= 0).sum()) and st["rerouted"] == res["rerouted"]
    plain = moe_ref.moe_layer(inp, k=k, cap=cap)
    assert st["dropped"] <= plain["stats"]["dropped"]
    assert st["aux_loss"] == plain["stats"]["aux_loss"] and st["imbalance"] == plain["stats"]["imbalance"]
    return res


@pytest.mark.parametrize("k,cap,rounds", [(1, 7, 1), (2, 14, 2), (1, 6, 3)])
def test_reroute_forward_matches_brute_force(k, cap, rounds):
    res = check_reroute_forward_vs_brute_force(_tiny(50 + k), k, cap, rounds)
    assert res["rerouted"] > 0


# ---------------------------------------------------------------------------
# Switch auxiliary loss
# ---------------------------------------------------------------------------

def check_aux_balanced_closed_form(T, k, E):
    """Round-robin routing with uniform gates: f_e = k/E (each token hits k distinct
    experts when E divides evenly), p_e = 1/E, so L = E * sum_e (k/E)(1/E) = k."""
    idx = (np.arange(T * k) % E).reshape(T, k)
    gates = np.full((T, E), 1.0 / E)
    assert moe_ref.switch_aux_loss(idx, gates, E) == pytest.approx(k, abs=1e-12)


@pytest.mark.parametrize("T,k,E", [(1024, 2, 8), (4096, 1, 32), (64, 2, 64)])
def test_aux_loss_round_robin_equals_k(T, k, E):
    check_aux_balanced_closed_form(T, k, E)


def test_aux_loss_f_is_counts_over_T():
    inp = _tiny(30)
    r = moe_ref.route(inp["x"], inp["w_router"], 2)
    counts = np.bincount(r["topk_idx"].ravel(), minlength=6)
    ref = 6 * np.sum(counts / 48 * r["gates"].mean(0))
    assert moe_ref.switch_aux_loss(r["topk_idx"], r["gates"], 6) == pytest.approx(ref, rel=1e-13)


# ---------------------------------------------------------------------------
# the notebook's six checks, on the notebook's own sizes
# ---------------------------------------------------------------------------

def test_notebook_checks_on_dense_top2():
    w = wl.workload("dense-top2-f32")
    inp = wl.draw_inputs(w)
    res = moe_ref.moe_layer(inp, k=w.k, cap=-1)
    assert res["out"].shape == inp["x"].shape                          # moe_output_shape_matches
    assert np.isfinite(res["out"]).all()                               # moe_output_finite
    counts = res["counts"]
    balanced = w.T * w.k / w.E
    d10 = moe_ref.drop_rate(counts, int(balanced * 1.0))
    d15 = moe_ref.drop_rate(counts, int(balanced * 1.5))
    assert d15 <= d10                                                  # higher_capacity_reduces_drops
    assert moe_ref.imbalance(counts, w.T, w.k, w.E) >= 1.05            # untrained_router_has_measurable_imbalance
    bal_idx = (np.arange(w.T * w.k) % w.E).reshape(w.T, w.k)
    bal = moe_ref.switch_aux_loss(bal_idx, np.full((w.T, w.E), 1.0 / w.E), w.E)
    assert res["stats"]["aux_loss"] > bal                              # aux_loss_imbalanced_higher_than_balanced
    assert Fraction(int(counts.sum()), w.T * w.E) == Fraction(w.k, w.E)  # active_params_equal_k_over_N


def test_zipf_alpha_gives_thirty_percent_hot_expert():
    w = wl.workload("skewed-top2")
    r = wl.draw_router_inputs(w)
    idx = moe_ref.topk(moe_ref.router_logits(r["x"], r["w_router"], r["logit_bias"]), w.k)
    share = (idx == 0).sum() / idx.size
    assert 0.295 <= share <= 0.305


# ---------------------------------------------------------------------------
# planted mistakes: each plausible bug in the oracle fails one pin
# ---------------------------------------------------------------------------

def _tanh_gelu(v):
    v = np.asarray(v, np.float64)
    return 0.5 * v * (1 + np.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3)))


def _topk_upper_ties(logits, k):
    l = np.asarray(logits, np.float64)
    return (l.shape[1] - 1 - np.argsort(-l[:, ::-1], axis=1, kind="stable"))[:, :k]


def _renormalised_route(x, w_router, k, logit_bias=None):
    r = _ORIG_ROUTE(x, w_router, k, logit_bias)
    r["topk_gate"] = r["topk_gate"] / r["topk_gate"].sum(1, keepdims=True)
    return r


def _dispatch_keep_last(topk_idx, E, cap):
    flat = np.asarray(topk_idx).reshape(-1)
    rev = _ORIG_DISPATCH(flat[::-1].copy(), E, cap)
    A = flat.size
    perm = (A - 1 - rev["perm"])
    out = dict(rev)
    out["perm"] = perm
    slot_of = np.full(A, -1, np.int64)
    slot_of[perm] = np.arange(len(perm))
    out["slot_of"] = slot_of
    return out


def _fc2_without_bias(h_e, w2_e, b2_e):
    return np.asarray(h_e, np.float64) @ np.asarray(w2_e, np.float64).T


def _softmax_wrong_axis(logits):
    l = np.asarray(logits, np.float64)
    z = np.exp(l - l.max(axis=0, keepdims=True))
    return z / z.sum(axis=0, keepdims=True)


def _aux_without_E(topk_idx, gates, E):
    return _ORIG_AUX(topk_idx, gates, E) / E


def _transposed_w1(x_e, w1_e, b1_e):
    w = np.asarray(w1_e, np.float64)
    w = w.reshape(w.shape[1], w.shape[0]).T if w.shape[0] != w.shape[1] else w.T
    return moe_ref.gelu(np.asarray(x_e, np.float64) @ w.T + np.asarray(b1_e)[None, :])


def _shared_mean_not_sum(x, params):
    return moe_ref.shared_expert_outputs(x, params).mean(axis=0)


def _shared_without_fc2_bias(x, params):
    p = dict(params)
    p["shared_b2"] = np.zeros_like(np.asarray(params["shared_b2"]))
    return _ORIG_SHARED_OUT(x, p)


def _offers_reverse_token_order(ranked_idx, served, k, r):
    return _ORIG_OFFERS(ranked_idx, served, k, r)[::-1]


def _offers_always_first_fallback(ranked_idx, served, k, r):
    return _ORIG_OFFERS(ranked_idx, served, k, 1)


def _imbalance_over_T(counts, T, k, E):
    return float(np.max(counts) / (T / E))


def _layer_stats_drop_rate_over_T(topk_idx, gates, E, cap, slot_of=None):
    st = _ORIG_LAYER_STATS(topk_idx, gates, E, cap, slot_of)
    st["drop_rate"] = st["dropped"] / np.asarray(topk_idx).shape[0]
    return st


def _layer_stats_dropped_counts_kept(topk_idx, gates, E, cap, slot_of=None):
    st = _ORIG_LAYER_STATS(topk_idx, gates, E, cap, slot_of)
    st["dropped"] = st["rows_kept"]
    return st


_ORIG_ROUTE = moe_ref.route
_ORIG_DISPATCH = moe_ref.dispatch
_ORIG_AUX = moe_ref.switch_aux_loss
_ORIG_SHARED_OUT = moe_ref.shared_expert_outputs
_ORIG_OFFERS = moe_ref.reroute_offers
_ORIG_LAYER_STATS = moe_ref.layer_stats

MUTATIONS = {
    "tanh-gelu": ("gelu", _tanh_gelu, lambda: check_gelu(moe_ref.gelu)),
    "ties-to-upper-index": ("topk", _topk_upper_ties,
                            lambda: check_topk_vs_stable_argsort(np.zeros((3, 8)), 2)),
    "renormalised-gates": ("route", _renormalised_route, lambda: check_route_gates_are_raw_probs(_tiny(2), 2)),
    "drop-first-not-last": ("dispatch", _dispatch_keep_last,
                            lambda: check_dispatch_vs_stable_sort(
                                np.random.default_rng(1).integers(0, 4, size=(40, 1)), 4, 3)),
    "fc2-bias-dropped": ("fc2", _fc2_without_bias, lambda: check_single_expert_is_mlp(_tiny(5, E=1))),
    "softmax-over-tokens": ("softmax", _softmax_wrong_axis,
                            lambda: check_softmax_vs_library(np.random.default_rng(0).normal(size=(5, 4)))),
    "aux-loss-missing-E": ("switch_aux_loss", _aux_without_E, lambda: check_aux_balanced_closed_form(64, 2, 8)),
    "w1-transposed": ("fc1_gelu", _transposed_w1, lambda: check_single_expert_is_mlp(_tiny(5, E=1))),
    "shared-averaged": ("shared_experts", _shared_mean_not_sum,
                        lambda: check_shared_experts_added_ungated(
                            wl.draw_custom(32, T=24, d=16, ff=24, E=4, dtype="f32", router_std=0.3, shared=2), 2, 5)),
    "shared-fc2-bias-dropped": ("shared_expert_outputs", _shared_without_fc2_bias,
                                lambda: check_shared_experts_added_ungated(
                                    wl.draw_custom(33, T=24, d=16, ff=24, E=4, dtype="f32", router_std=0.3,
                                                   shared=1), 1, -1)),
    "reroute-offers-reversed": ("reroute_offers", _offers_reverse_token_order, check_reroute_hand_example_top1),
    "reroute-no-deeper-fallback": ("reroute_offers", _offers_always_first_fallback,
                                   check_reroute_hand_example_top1),
    "imbalance-over-T-not-Tk": ("imbalance", _imbalance_over_T, check_imbalance_closed_form),
    "layer-drop-rate-over-T": ("layer_stats", _layer_stats_drop_rate_over_T,
                               check_layer_stats_drops_are_capacity_check),
    "layer-dropped-is-kept": ("layer_stats", _layer_stats_dropped_counts_kept,
                              check_layer_stats_drops_are_capacity_check),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad, pin = MUTATIONS[name]
    pin()                                    # the pin passes on the real oracle
    monkeypatch.setattr(moe_ref, attr, bad)
    with pytest.raises(AssertionError):
        pin()
