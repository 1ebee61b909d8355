"""The oracle against the values the pages themselves state
(tests/golden/notebook_stated_values.json, each entry citing its section of
the cookbook notebook "Mixture-of-experts and expert parallelism")."""
import json
import os

import numpy as np

from mixture_experts_layer_45_b200 import workloads as wl
from oracle import moe_ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "notebook_stated_values.json")


def golden():
    with open(GOLDEN) as fh:
        return json.load(fh)


def test_notebook_sizes_are_the_dense_workload():
    g = golden()["sizes"]
    w = wl.workload("dense-top2-f32")
    assert (w.E, w.d, w.T, w.k) == (g["experts"], g["model_dim"], g["tokens"], g["k"])


def test_balanced_aux_loss_is_the_stated_minimum():
    g = golden()
    T, E, k = g["sizes"]["tokens"], g["sizes"]["experts"], g["balanced_aux_loss"]["k"]
    idx = (np.arange(T * k) % E).reshape(T, k)          # round-robin expert ids
    gates = np.full((T, E), 1.0 / E)
    assert moe_ref.switch_aux_loss(idx, gates, E) == g["balanced_aux_loss"]["value"]


def test_active_expert_fraction():
    """Every token's output mixes exactly k of the N experts (no capacity)."""
    g = golden()
    T, E = g["sizes"]["tokens"], g["active_expert_fraction"]["experts"]
    k = g["active_expert_fraction"]["k"]
    inp = wl.draw_inputs(wl.workload("dense-top2-f32"))
    r = moe_ref.route(inp["x"], inp["w_router"], k)
    gates = np.take_along_axis(r["gates"], r["topk_idx"], 1)
    d = moe_ref.dispatch(r["topk_idx"], E, -1)
    M = moe_ref.kept_gate_matrix(r["topk_idx"], gates, d["slot_of"], E)
    frac = (M > 0).sum(axis=1) / E
    assert frac.shape == (T,)
    assert np.all(frac == g["active_expert_fraction"]["value"])
