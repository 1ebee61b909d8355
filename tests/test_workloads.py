"""Seeded input generators: determinism, shapes and the bf16 encoding."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_45_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.normal(size=10000).astype(np.float32) * 1e3,
                        # exact ties between two bf16 neighbours, both parities
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 3.0e-39],
                                 np.float32)])
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(wl.bf16_bits(a), ref)
    back = wl.bf16_to_f32(wl.bf16_bits(a))
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_draws_are_deterministic_and_shaped():
    w = wl.workload("dense-top2-f32")
    a, b = wl.draw_inputs(w), wl.draw_inputs(w)
    for key in ("x", "w_router", "w1", "b1", "w2", "b2"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["x"].shape == (1024, 256) and a["w_router"].shape == (8, 256)
    assert a["w1"].shape == (8, 1024, 256) and a["b1"].shape == (8, 1024)
    assert a["w2"].shape == (8, 256, 1024) and a["b2"].shape == (8, 256)
    assert a["logit_bias"] is None
    # nn.Linear default init bound 1/sqrt(fan_in)
    assert np.abs(a["w1"]).max() <= 1 / 16 and np.abs(a["w2"]).max() <= 1 / 32


def test_bf16_workloads_hold_bf16_values():
    w = wl.workload("switch-top1", dtype="bf16", T=64)
    a = wl.draw_router_inputs(w)
    for key in ("x", "w_router"):
        np.testing.assert_array_equal(wl.round_to_bf16(a[key]), a[key])


def test_sequence_shift_recipe_correlates_tokens():
    w = wl.workload("encoder-prefill-top1")
    x = wl.draw_router_inputs(w)["x"]
    assert x.shape == (16384, 768)
    seq_means = x.reshape(32, 512, 768).mean(1)          # ~ mu_s, std 0.5
    assert 0.4 < seq_means.std() < 0.6


def test_zipf_bias_is_decreasing():
    b = wl.zipf_logit_bias(64)
    assert b.shape == (64,) and np.all(np.diff(b) < 0)


def test_workload_table():
    names = [w.describe() for w in wl.all_workloads()]
    assert len(names) == 8
    with pytest.raises(KeyError):
        wl.workload("nope")


def test_shared_expert_draws_follow_the_routed_ones():
    """Adding shared experts leaves every routed draw unchanged and gives the
    shared experts the routed experts' shapes and bf16 rounding."""
    base = wl.draw_inputs(wl.workload("switch-top1"), T=64)
    w = wl.workload("switch-top1", shared=2)
    got = wl.draw_inputs(w, T=64)
    for key, v in base.items():
        if v is not None:
            assert np.array_equal(got[key], v), key
    assert got["shared_w1"].shape == (2, w.ff, w.d) and got["shared_b1"].shape == (2, w.ff)
    assert got["shared_w2"].shape == (2, w.d, w.ff) and got["shared_b2"].shape == (2, w.d)
    for key in ("shared_w1", "shared_b1", "shared_w2", "shared_b2"):
        assert np.array_equal(wl.round_to_bf16(got[key]), got[key])
    assert not np.array_equal(got["shared_w1"][0], got["w1"][0])
