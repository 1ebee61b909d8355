"""Seeded synthetic inputs for the MoE layer forward pass.

This module draws the inputs of one MoE layer (tokens, router weights, an
optional per-expert logit bias and the stacked expert FFN parameters) for the
five workloads the layer is exercised on.  It holds none of the layer's own
arithmetic: no routing, no softmax, no dispatch, no FFN.  Both the CUDA path
(through ``bench.py`` and the GPU tests) and the float64 CPU oracle (through
the tests) consume exactly the arrays returned here.

Shapes follow the cookbook notebook "Mixture-of-experts and expert
parallelism" (llm-systems-cookbook, 05_serving/09), sections "Top-k router"
and "Dispatch and gather": tokens ``x`` are [T, d]; the router is a
bias-free ``Linear(d -> E)`` whose weight is [E, d]; expert e is
``fc2(gelu(fc1(x)))`` with ``fc1 = Linear(d -> ff)`` (weight [ff, d], bias
[ff]) and ``fc2 = Linear(ff -> d)`` (weight [d, ff], bias [d]).  The experts
are stacked: W1 [E, ff, d], b1 [E, ff], W2 [E, d, ff], b2 [E, d].

bf16 workloads draw in float32 and round every tensor to bfloat16 with
round-to-nearest-even; the returned float32 arrays hold exactly the rounded
values and ``bf16_bits`` gives the 16-bit patterns uploaded to the GPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

# Zipf exponent and calibrated bias scale of the skewed-routing workload.
# The bias of expert e is ZIPF_ALPHA * ln p_(e+1), p_r proportional to r^-1.2
# over the E experts (expert 0 is the hottest).  ZIPF_ALPHA is the value that
# makes expert 0 receive 30% of the T*k assignments on this workload's seeded
# tokens and router weights; it is written by oracle/calibrate_zipf_alpha.py
# and re-checked by the CPU tests.
ZIPF_S = 1.2
ZIPF_ALPHA = 0.4611515402793884


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer workload (sizes, precision and draw recipe)."""

    name: str
    T: int                # tokens
    d: int                # model dim
    ff: int               # expert hidden dim
    E: int                # experts
    k: int                # experts per token
    dtype: str            # "f32" or "bf16": the arithmetic type of the path
    cf: Optional[float]   # capacity factor; None = no capacity limit
    seed: int
    router_std: float     # router weight ~ N(0, router_std^2)
    expert_init: str      # "uniform": nn.Linear default U(+-1/sqrt(fan_in)); "normal002": N(0, 0.02^2), zero bias
    x_recipe: str = "normal"   # "normal" or "seq_shift" (per-sequence mean shift)
    seq_len: int = 0           # tokens per sequence for "seq_shift"
    seq_shift_std: float = 0.0
    zipf_bias: bool = False
    shared: int = 0            # shared always-on experts (same shapes and init as the routed ones)

    def capacity_factor_label(self) -> str:
        return "none" if self.cf is None else f"{self.cf:g}"

    def describe(self) -> str:
        return (f"{self.name}: T={self.T} d={self.d} ff={self.ff} E={self.E} "
                f"k={self.k} {self.dtype} cf={self.capacity_factor_label()}"
                + (f" shared={self.shared}" if self.shared else ""))


_BASE = {
    # Cookbook notebook sizes: 1024 tokens, D=256, 8 experts, top-2, fp32.
    "dense-top2-f32": dict(T=1024, d=256, ff=1024, E=8, k=2, dtype="f32", cf=None,
                           seed=45_001, router_std=0.1, expert_init="uniform"),
    # Switch-style top-1: T=4096, d=768, ff=3072, 32 experts.
    "switch-top1": dict(T=4096, d=768, ff=3072, E=32, k=1, seed=45_002,
                        router_std=0.02, expert_init="uniform"),
    # Skewed routing stress: Zipf(1.2) per-expert logit bias.
    "skewed-top2": dict(T=16384, d=1024, ff=4096, E=64, k=2, dtype="bf16", cf=None,
                        seed=45_003, router_std=0.02, expert_init="uniform", zipf_bias=True),
    # Encoder-style prefill: 32 sequences x 512 tokens, per-sequence mean shift.
    "encoder-prefill-top1": dict(T=16384, d=768, ff=3072, E=64, k=1, dtype="bf16", cf=1.25,
                                 seed=45_004, router_std=0.02, expert_init="uniform",
                                 x_recipe="seq_shift", seq_len=512, seq_shift_std=0.5),
    # Large top-2 layer: T=8192, d=4096, ff=14336, 8 experts.
    "large-top2": dict(T=8192, d=4096, ff=14336, E=8, k=2, dtype="bf16", cf=None,
                       seed=45_005, router_std=0.02, expert_init="normal002"),
}


def workload(name: str, dtype: Optional[str] = None, cf: Optional[float] = "default",
             **overrides) -> Workload:
    """Return a named workload.  ``dtype``/``cf`` select the switch-top1 variants."""
    if name not in _BASE:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(_BASE)}")
    spec = dict(_BASE[name])
    if name == "switch-top1":
        spec.setdefault("dtype", "bf16")
        spec.setdefault("cf", 1.0)
    if dtype is not None:
        spec["dtype"] = dtype
    if cf != "default":
        spec["cf"] = cf
    spec.update(overrides)
    return Workload(name=name, **spec)


def all_workloads():
    """Every workload variant the parity tests cover."""
    out = [workload("dense-top2-f32")]
    for dt in ("f32", "bf16"):
        for cf in (1.0, 1.5):
            out.append(workload("switch-top1", dtype=dt, cf=cf))
    out += [workload("skewed-top2"), workload("encoder-prefill-top1"), workload("large-top2")]
    return out


# ---------------------------------------------------------------------------
# bf16 encoding (input preparation, shared by both sides)
# ---------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to the float32 values they encode."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array holding exactly the bf16-rounded values of ``a``."""
    return bf16_to_f32(bf16_bits(a))


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------

def zipf_logit_bias(E: int, alpha: float = ZIPF_ALPHA, s: float = ZIPF_S) -> np.ndarray:
    """Per-expert logit bias alpha * ln p_(e+1), p_r = r^-s / sum_j j^-s."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return (alpha * np.log(p)).astype(np.float32)


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def _uniform(rng: np.random.Generator, shape, fan_in: int) -> np.ndarray:
    b = 1.0 / math.sqrt(fan_in)
    return rng.uniform(-b, b, size=shape).astype(np.float32)


def draw_router_inputs(w: Workload, T: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Tokens, router weight and logit bias (the first draws of the stream).

    Returns float32 arrays; for bf16 workloads they hold bf16-rounded values.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    return _draw_router(rng, w, T)


def _draw_router(rng, w: Workload, T: Optional[int]):
    T = w.T if T is None else T
    if w.x_recipe == "normal":
        x = rng.standard_normal(size=(T, w.d), dtype=np.float32)
    elif w.x_recipe == "seq_shift":
        n_seq = -(-T // w.seq_len)
        z = rng.standard_normal(size=(n_seq * w.seq_len, w.d), dtype=np.float32)
        mu = _normal(rng, (n_seq, 1, w.d), w.seq_shift_std)
        x = (z.reshape(n_seq, w.seq_len, w.d) + mu).reshape(-1, w.d)[:T].astype(np.float32)
    else:
        raise ValueError(w.x_recipe)
    w_router = _normal(rng, (w.E, w.d), w.router_std)
    bias = zipf_logit_bias(w.E) if w.zipf_bias else None
    out = {"x": x, "w_router": w_router, "logit_bias": bias}
    if w.dtype == "bf16":
        out["x"] = round_to_bf16(out["x"])
        out["w_router"] = round_to_bf16(out["w_router"])
    return out


def draw_inputs(w: Workload, T: Optional[int] = None) -> Dict[str, np.ndarray]:
    """All inputs of one workload, in a fixed draw order from one seeded stream.

    Keys: x [T,d], w_router [E,d], logit_bias [E] or None, w1 [E,ff,d],
    b1 [E,ff], w2 [E,d,ff], b2 [E,d] -- float32 (bf16-rounded for bf16).
    With ``w.shared`` = S > 0 also shared_w1 [S,ff,d], shared_b1 [S,ff],
    shared_w2 [S,d,ff], shared_b2 [S,d], drawn after the routed experts (so
    the routed draws do not depend on S) with the same recipe.
    ``T`` overrides the token count (a prefix-independent redraw, used for
    ragged-size tests).
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    out = _draw_router(rng, w, T)
    w1, b1, w2, b2 = _draw_experts(rng, w, w.E)
    out.update(w1=w1, b1=b1, w2=w2, b2=b2)
    if w.shared > 0:
        sw1, sb1, sw2, sb2 = _draw_experts(rng, w, w.shared)
        out.update(shared_w1=sw1, shared_b1=sb1, shared_w2=sw2, shared_b2=sb2)
    return out


def _draw_experts(rng, w: Workload, n: int):
    d, ff = w.d, w.ff
    if w.expert_init == "uniform":
        w1 = _uniform(rng, (n, ff, d), d)
        b1 = _uniform(rng, (n, ff), d)
        w2 = _uniform(rng, (n, d, ff), ff)
        b2 = _uniform(rng, (n, d), ff)
    elif w.expert_init == "normal002":
        w1 = _normal(rng, (n, ff, d), 0.02)
        b1 = np.zeros((n, ff), np.float32)
        w2 = _normal(rng, (n, d, ff), 0.02)
        b2 = np.zeros((n, d), np.float32)
    else:
        raise ValueError(w.expert_init)
    if w.dtype == "bf16":
        w1, b1, w2, b2 = (round_to_bf16(a) for a in (w1, b1, w2, b2))
    return w1, b1, w2, b2


def draw_custom(seed: int, T: int, d: int, ff: int, E: int, dtype: str,
                router_std: float = 0.1, x_scale: float = 1.0, shared: int = 0) -> Dict[str, np.ndarray]:
    """Small arbitrary-shape inputs for edge-case and brute-force tests."""
    w = Workload(name="custom", T=T, d=d, ff=ff, E=E, k=1, dtype=dtype, cf=None,
                 seed=seed, router_std=router_std, expert_init="uniform", shared=shared)
    out = draw_inputs(w)
    if x_scale != 1.0:
        x = out["x"] * np.float32(x_scale)
        out["x"] = round_to_bf16(x) if dtype == "bf16" else x
    return out
