"""The GPU tests' routing checker, exercised on the CPU with the oracle: it
accepts the exact answer, accepts a swap inside the floating-point error
bound, and rejects a wrong choice on a decided row."""
import numpy as np
import pytest

import parity_util as pu
from mixture_experts_layer_45_b200 import workloads as wl
from oracle import moe_ref


def _routing(k=2):
    w = wl.workload("dense-top2-f32")
    r = wl.draw_router_inputs(w)
    L = moe_ref.router_logits(r["x"], r["w_router"])
    return r, L, moe_ref.topk(L, k)


def test_exact_answer_passes():
    r, L, idx = _routing()
    delta = pu.logit_error_bound(r["x"], r["w_router"])
    assert pu.check_routing(idx, L, 2, delta)[0] == 0


def test_swap_within_bound_is_accepted_and_wrong_choice_rejected():
    r, L, idx = _routing()
    L = L.copy()
    delta = pu.logit_error_bound(r["x"], r["w_router"])
    # make row 0's top two logits a near tie (gap far below the bound) and swap them
    a, b = idx[0]
    L[0, b] = L[0, a] - 1e-3 * delta[0]
    swapped = idx.copy()
    swapped[0] = [b, a]
    diff, undecided = pu.check_routing(swapped, L, 2, delta)
    assert diff == 1 and undecided >= 1
    # a clearly worse expert on a decided row is rejected
    bad = idx.copy()
    worst = int(np.argmin(L[5]))
    bad[5, 1] = worst
    with pytest.raises(AssertionError):
        pu.check_routing(bad, L, 2, delta)
    # a repeated expert is rejected
    rep = idx.copy()
    rep[7, 1] = rep[7, 0]
    with pytest.raises(AssertionError):
        pu.check_routing(rep, L, 2, delta)


def test_error_bound_is_small_relative_to_logits():
    r, L, _ = _routing()
    delta = pu.logit_error_bound(r["x"], r["w_router"])
    assert np.all(delta > 0) and delta.max() < 1e-3 * np.abs(L).max()


def test_max_rel_err():
    assert pu.max_rel_err([1.0, 2.0], [1.0, 2.0]) == 0.0
    assert pu.max_rel_err([1.0, 2.1], [1.0, 2.0]) == pytest.approx(0.05)


@pytest.mark.parametrize("k,E,T", [(2, 64, 3000), (1, 8, 1000), (2, 8, 4096)])
def test_tile_covering_rows_reach_every_m_tile(k, E, T):
    rng = np.random.default_rng(T)
    # skewed routing: expert 0 takes most rows, some experts are empty
    p = np.r_[0.5, np.full(E - 1, 0.5 / (E - 1))]
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    d = moe_ref.dispatch(idx, E, -1)
    toks = pu.tile_covering_rows(d["offsets"], d["perm"], k, T, seed=1)
    slot = d["slot_of"].reshape(T, k)
    rows_reached = set(int(r) for r in slot[toks].ravel() if r >= 0)
    for tile in (128, 256):
        reached = set()
        for e in range(E):
            lo, hi = int(d["offsets"][e]), int(d["offsets"][e + 1])
            for t0 in range(lo, hi, tile):
                if any(t0 <= r < min(t0 + tile, hi) for r in rows_reached):
                    reached.add((e, t0))
        assert len(reached) == pu.m_tiles(d["offsets"], tile)
    # shared groups: one token of every 128-token block
    toks_s = pu.tile_covering_rows(d["offsets"], d["perm"], k, T, seed=1, shared=2)
    assert set(toks_s // 128) == set(range(-(-T // 128)))
