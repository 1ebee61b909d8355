"""Float64 CPU oracle for the forward pass of one Mixture-of-Experts layer.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.  Only the tests, the
smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py``
may import or run this module.  It shares no code with the CUDA library and
imports nothing from it; it depends on numpy and scipy only.

What it computes, and where that is stated.  The authority is the cookbook
notebook "Mixture-of-experts and expert parallelism" (llm-systems-cookbook,
05_serving/09):

* section "Top-k router": logits = x W_r^T (a bias-free Linear), gates =
  softmax(logits) over experts, then the k largest gates and their experts.
  The returned weights are the raw softmax probabilities; they are not
  renormalised over the k picks.
* section "Dispatch and gather": expert e is fc2(gelu(fc1(x))) with biased
  Linear layers and the exact (erf) GELU; moe_forward starts from zeros and,
  for e = 0..N-1 in order, adds expert e's output times the token's summed
  gate for e to every token routed to e.
* section "Capacity factor": per-expert counts of the T*k assignments, the
  slot budget int(T*k/N*factor) (int() truncates, i.e. floor for positive
  values), the imbalance ratio max(count)/(T*k/N) and the drop rate
  sum(max(count - capacity, 0)) / sum(count).
* section "Switch Transformer auxiliary loss": L_aux = N * sum_i f_i p_i with
  f_i the fraction of tokens whose top-k contains i and p_i the mean gate.

Readings where the notebook is silent (each one is also listed in the design
notes of the repository):

* top-k order and ties: experts are ranked by logit, largest first, and an
  exact tie goes to the lower expert index.  Ranking on logits equals ranking
  on probabilities because softmax is strictly increasing.
* which assignments a full expert drops: the notebook only counts the
  overflow.  Each expert keeps its first ``capacity`` assignments in token
  order and drops the rest; a dropped assignment contributes nothing.
* rows of the dispatched (permuted) layout: expert e's kept assignments
  occupy rows offsets[e] .. offsets[e+1]-1 in token order, experts in
  ascending order.
* softmax is evaluated with the row maximum subtracted (the same function).

Shared always-on experts (notebook section "Exercises", item 3: DeepSeek-V2
keeps a small set of experts that every token uses beside the routed ones;
the exercise asks to extend the forward with them).  Readings: every token
passes through every shared expert and its output is added with weight 1
(no gate); shared experts have the routed experts' form and shapes
(fc2(gelu(fc1(x))), d -> ff -> d, biased); they are outside the router, the
capacity limit and the statistics, so a token whose routed assignments are
all dropped still receives the shared experts' sum.

Every function below works in float64 on whatever values it is given; bf16
workloads pass the bf16-rounded values the GPU also receives.

Parity pins: every function here is pinned by a CPU test in
``tests/test_oracle_pins.py`` to something other than itself (closed forms,
library routines, brute force, the notebook's own invariants).  The absolute
values of the notebook's run are not pinned: its printed outputs were
stripped and its torch random stream is not reproduced.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
from scipy.special import erf as _erf


# ---------------------------------------------------------------------------
# Top-k router (notebook section "Top-k router")
# ---------------------------------------------------------------------------

def router_logits(x, w_router, logit_bias=None) -> np.ndarray:
    """logits[t, e] = sum_i x[t, i] * w_router[e, i]  (+ logit_bias[e]).

    The notebook's router is ``Linear(D, N_EXPERTS, bias=False)``; the
    optional per-expert bias is the skewed-routing workload's logit offset.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    logits = x @ w.T
    if logit_bias is not None:
        logits = logits + np.asarray(logit_bias, dtype=np.float64)[None, :]
    return logits


def softmax(logits) -> np.ndarray:
    """Row softmax over experts, evaluated as exp(l - max) / sum exp(l - max)."""
    l = np.asarray(logits, dtype=np.float64)
    z = np.exp(l - l.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def topk(logits, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first, ties -> lower index.

    Selection by k rounds of first-occurrence argmax with the winner masked
    out, so an exact tie always resolves to the lower expert index.
    """
    l = np.array(logits, dtype=np.float64, copy=True)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError(f"need 1 <= k <= E, got k={k}, E={E}")
    idx = np.empty((T, k), dtype=np.int64)
    rows = np.arange(T)
    for j in range(k):
        pick = np.argmax(l, axis=1)          # first occurrence of the max
        idx[:, j] = pick
        l[rows, pick] = -np.inf
    return idx


def route(x, w_router, k: int, logit_bias=None) -> Dict[str, np.ndarray]:
    """The notebook's router: logits -> softmax -> top-k (weights not renormalised)."""
    logits = router_logits(x, w_router, logit_bias)
    gates = softmax(logits)
    idx = topk(logits, k)
    topk_gate = np.take_along_axis(gates, idx, axis=1)
    return {"logits": logits, "gates": gates, "topk_idx": idx, "topk_gate": topk_gate}


# ---------------------------------------------------------------------------
# Counts, capacity and dispatch (notebook section "Capacity factor")
# ---------------------------------------------------------------------------

def token_count_per_expert(topk_idx, E: int) -> np.ndarray:
    """counts[e] = number of (token, slot) assignments equal to e."""
    idx = np.asarray(topk_idx)
    counts = np.zeros(E, dtype=np.int64)
    for e in range(E):
        counts[e] = int((idx == e).sum())
    return counts


def capacity(T: int, k: int, E: int, cf: Optional[float]) -> int:
    """Per-expert slot budget int(T*k/E*cf); -1 means no limit (cf None or <= 0)."""
    if cf is None or cf <= 0:
        return -1
    return int(T * k / E * cf)


def drop_rate(counts, cap: int) -> float:
    """sum(max(counts - cap, 0)) / sum(counts), as the notebook's capacity_check."""
    counts = np.asarray(counts, dtype=np.float64)
    if cap < 0:
        return 0.0
    total = counts.sum()
    return float(np.clip(counts - cap, 0, None).sum() / total) if total > 0 else 0.0


def imbalance(counts, T: int, k: int, E: int) -> float:
    """max(counts) / (T*k/E)."""
    return float(np.max(counts) / (T * k / E))


def dispatch(topk_idx, E: int, cap: int) -> Dict[str, np.ndarray]:
    """Group assignments by expert, keep each expert's first ``cap`` in token order.

    Assignment a = t*k + j is (token t, slot j).  Returns
      counts [E]       assignments per expert before any drop
      kept [E]         min(counts, cap) (counts when cap < 0)
      offsets [E+1]    exclusive prefix sum of kept; offsets[E] = rows kept R
      perm [R]         perm[offsets[e] + r] = a of expert e's r-th kept assignment
      slot_of [T*k]    row of assignment a in the grouped layout, -1 if dropped
      drop_mask [T*k]  1 where assignment a was dropped
    """
    idx = np.asarray(topk_idx).reshape(-1)
    A = idx.size
    counts = token_count_per_expert(idx, E)
    kept = counts.copy() if cap < 0 else np.minimum(counts, cap)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    perm = np.empty(int(offsets[E]), dtype=np.int64)
    slot_of = np.full(A, -1, dtype=np.int64)
    for e in range(E):
        mine = [a for a in range(A) if idx[a] == e]          # token order
        for r, a in enumerate(mine[: int(kept[e])]):
            row = int(offsets[e]) + r
            perm[row] = a
            slot_of[a] = row
    drop_mask = (slot_of < 0).astype(np.uint8)
    return {"counts": counts, "kept": kept, "offsets": offsets, "perm": perm,
            "slot_of": slot_of, "drop_mask": drop_mask}


# ---------------------------------------------------------------------------
# Overflow rerouting instead of dropping (the blog "MoE Parallelism for
# Inference", section "Common Bottlenecks", item 1, on sending rejected
# tokens to less busy experts; the cookbook notebook, section "What": the
# overflow is dropped or sent to a fallback path)
# ---------------------------------------------------------------------------

def reroute_offers(ranked_idx, served, k: int, r: int):
    """Round r's offers, in the order experts see them (token order): for each
    token with an unserved slot, (t, its first unserved slot j, its (k+r)-th
    expert)."""
    offers = []
    for t in range(served.shape[0]):
        waiting = [j for j in range(k) if not served[t, j]]
        if waiting:
            offers.append((t, waiting[0], int(ranked_idx[t, k + r - 1])))
    return offers


def dispatch_reroute(ranked_idx, ranked_gate, k: int, E: int, cap: int, rounds: int) -> Dict[str, np.ndarray]:
    """Dispatch with up to ``rounds`` rerouting rounds for dropped assignments.

    ranked_idx / ranked_gate [T, k + rounds]: each token's experts in the
    router's order (largest logit first) and their softmax gates; the first
    k are the token's assignments, the rest its fallback experts.

    Readings (the pages name the idea, not the rule): first the plain
    dispatch (each expert keeps its first ``cap`` assignments in token
    order).  Then in round r = 1 .. rounds, every token that still has a
    dropped assignment offers its first such slot j to its (k+r)-th expert
    c = ranked_idx[t, k+r-1]; each expert accepts offers in token order while
    it holds fewer than ``cap`` rows.  An accepted slot is served by c with
    gate ranked_gate[t, k+r-1].  Expert e's rows are its own kept
    assignments in token order, then those it accepted in round 1 (token
    order), round 2, and so on.  A token never gets an expert twice: the
    fallbacks differ from its first k experts and from each other.

    Returns the keys of ``dispatch`` (counts are the router's choices before
    any drop; kept and offsets are final) plus
      final_idx / final_gate [T, k]  the expert and gate serving each slot
      kept_primary [E]               rows each expert kept from its own choices
      rerouted                       assignments served by a fallback expert
    """
    ranked_idx = np.asarray(ranked_idx)
    ranked_gate = np.asarray(ranked_gate, np.float64)
    T = ranked_idx.shape[0]
    if ranked_idx.shape[1] < k + rounds:
        raise ValueError("ranked_idx needs k + rounds columns")
    idx = ranked_idx[:, :k]
    base = dispatch(idx, E, cap)
    final_idx = idx.copy()
    final_gate = ranked_gate[:, :k].copy()
    served = (base["slot_of"].reshape(T, k) >= 0)
    # members[e]: assignments served by e, in row order
    members = [[a for a in base["perm"][base["offsets"][e]:base["offsets"][e + 1]]] for e in range(E)]
    load = np.array([len(m) for m in members], dtype=np.int64)
    rerouted = 0
    if cap >= 0:
        for r in range(1, rounds + 1):
            for t, j, c in reroute_offers(ranked_idx, served, k, r):
                if load[c] < cap:
                    load[c] += 1
                    members[c].append(t * k + j)
                    served[t, j] = True
                    final_idx[t, j] = c
                    final_gate[t, j] = ranked_gate[t, k + r - 1]
                    rerouted += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(load)
    perm = np.array([a for e in range(E) for a in members[e]], dtype=np.int64)
    slot_of = np.full(T * k, -1, dtype=np.int64)
    slot_of[perm] = np.arange(len(perm))
    return {"counts": base["counts"], "kept": load, "kept_primary": base["kept"], "offsets": offsets,
            "perm": perm, "slot_of": slot_of, "drop_mask": (slot_of < 0).astype(np.uint8),
            "final_idx": final_idx, "final_gate": final_gate, "rerouted": rerouted}


# ---------------------------------------------------------------------------
# Expert FFN and gated combine (notebook section "Dispatch and gather")
# ---------------------------------------------------------------------------

def gelu(v) -> np.ndarray:
    """Exact GELU: v * Phi(v) = 0.5 * v * (1 + erf(v / sqrt(2)))."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + _erf(v / math.sqrt(2.0)))


def fc1_gelu(x_e, w1_e, b1_e) -> np.ndarray:
    """H = gelu(x_e W1_e^T + b1_e): the first Linear and the activation."""
    return gelu(np.asarray(x_e, np.float64) @ np.asarray(w1_e, np.float64).T
                + np.asarray(b1_e, np.float64)[None, :])


def fc2(h_e, w2_e, b2_e) -> np.ndarray:
    """Y = H W2_e^T + b2_e: the second Linear."""
    return (np.asarray(h_e, np.float64) @ np.asarray(w2_e, np.float64).T
            + np.asarray(b2_e, np.float64)[None, :])


def expert_ffn(x_e, w1_e, b1_e, w2_e, b2_e) -> np.ndarray:
    """fc2(gelu(fc1(x_e))) for the rows of one expert."""
    return fc2(fc1_gelu(x_e, w1_e, b1_e), w2_e, b2_e)


def kept_gate_matrix(topk_idx, topk_gate, slot_of, E: int) -> np.ndarray:
    """M[t, e] = sum_j gate[t, j] over slots j with idx[t, j] == e that were kept."""
    idx = np.asarray(topk_idx)
    g = np.asarray(topk_gate, np.float64)
    T, k = idx.shape
    keep = (np.asarray(slot_of).reshape(T, k) >= 0)
    M = np.zeros((T, E), np.float64)
    for j in range(k):
        rows = np.nonzero(keep[:, j])[0]
        M[rows, idx[rows, j]] += g[rows, j]
    return M


def moe_forward(x, params, topk_idx, topk_gate, slot_of=None) -> np.ndarray:
    """The notebook's moe_forward with an optional drop set.

    out = 0; for e = 0..E-1: tokens with a kept assignment to e get
    expert_e(x[t]) * (sum of their kept gates for e) added.  ``slot_of`` < 0
    marks dropped assignments (None: nothing dropped).
    """
    x = np.asarray(x, np.float64)
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    E = params["w1"].shape[0]
    if slot_of is None:
        slot_of = np.zeros(T * k, dtype=np.int64)
    M = kept_gate_matrix(idx, topk_gate, slot_of, E)
    keep = np.asarray(slot_of).reshape(T, k) >= 0
    out = np.zeros_like(x)
    for e in range(E):
        mask = ((idx == e) & keep).any(axis=1)     # tokens with a kept assignment to e
        if not mask.any():
            continue
        y = expert_ffn(x[mask], params["w1"][e], params["b1"][e],
                       params["w2"][e], params["b2"][e])
        out[mask] += y * M[mask, e][:, None]
    return out


def moe_forward_rows(x, params, topk_idx, topk_gate, slot_of, rows) -> np.ndarray:
    """Output rows ``rows`` of moe_forward.

    The expert FFN acts on each token independently, so moe_forward applied
    to the sampled tokens (with their routing and drop flags) gives exactly
    those rows of the full output; used for full-size parity checks.
    """
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    rows = np.asarray(rows)
    sub_slot = np.asarray(slot_of).reshape(T, k)[rows].reshape(-1)
    return moe_forward(np.asarray(x)[rows], params, idx[rows], np.asarray(topk_gate)[rows], sub_slot)


def grouped_ffn(xp, offsets, params, row_gate=None) -> np.ndarray:
    """Y[row] = row_gate[row] * expert_e(xp[row]) for rows offsets[e]..offsets[e+1]-1."""
    xp = np.asarray(xp, np.float64)
    E = len(offsets) - 1
    R = int(offsets[E])
    Y = np.zeros((R, params["w2"].shape[1]), np.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            Y[lo:hi] = expert_ffn(xp[lo:hi], params["w1"][e], params["b1"][e],
                                  params["w2"][e], params["b2"][e])
    if row_gate is not None:
        Y *= np.asarray(row_gate, np.float64)[:R, None]
    return Y


def combine(yp, slot_of, T: int, k: int, topk_gate=None) -> np.ndarray:
    """out[t] = sum over kept slots j of (gate[t,j] *) yp[slot_of[t*k+j]]; 0 if none kept."""
    yp = np.asarray(yp, np.float64)
    s = np.asarray(slot_of).reshape(T, k)
    out = np.zeros((T, yp.shape[1]), np.float64)
    for j in range(k):
        rows = np.nonzero(s[:, j] >= 0)[0]
        contrib = yp[s[rows, j]]
        if topk_gate is not None:
            contrib = contrib * np.asarray(topk_gate, np.float64)[rows, j][:, None]
        out[rows] += contrib
    return out


# ---------------------------------------------------------------------------
# Shared always-on experts (notebook section "Exercises", item 3)
# ---------------------------------------------------------------------------

def has_shared(params) -> bool:
    return params.get("shared_w1") is not None and np.asarray(params["shared_w1"]).shape[0] > 0


def shared_expert_outputs(x, params) -> np.ndarray:
    """Ys[s] = shared expert s applied to every token: [S, T, d]."""
    x = np.asarray(x, np.float64)
    S = np.asarray(params["shared_w1"]).shape[0]
    return np.stack([expert_ffn(x, params["shared_w1"][s], params["shared_b1"][s],
                                params["shared_w2"][s], params["shared_b2"][s]) for s in range(S)])


def shared_experts(x, params) -> np.ndarray:
    """Sum over the shared experts of their outputs, weight 1, every token: [T, d]."""
    return shared_expert_outputs(x, params).sum(axis=0)


def moe_forward_rows_shared(x, params, topk_idx, topk_gate, slot_of, rows) -> np.ndarray:
    """Output rows ``rows`` of the layer with shared experts (routed part
    from moe_forward_rows; the shared experts act on each token alone)."""
    out = moe_forward_rows(x, params, topk_idx, topk_gate, slot_of, rows)
    if has_shared(params):
        out = out + shared_experts(np.asarray(x)[np.asarray(rows)], params)
    return out


# ---------------------------------------------------------------------------
# Switch auxiliary loss and the layer's statistics
# (notebook sections "Switch Transformer auxiliary loss" and "Capacity factor")
# ---------------------------------------------------------------------------

def switch_aux_loss(topk_idx, gates, E: int) -> float:
    """L_aux = E * sum_e f_e p_e, f_e = fraction of tokens with e in their top-k,
    p_e = mean over tokens of the full softmax gate of e."""
    idx = np.asarray(topk_idx)
    f = np.zeros(E, np.float64)
    for e in range(E):
        f[e] = (idx == e).any(axis=1).mean()
    p = np.asarray(gates, np.float64).mean(axis=0)
    return float(E * (f * p).sum())


def layer_stats(topk_idx, gates, E: int, cap: int, slot_of=None) -> Dict[str, float]:
    """The layer's reported statistics from its routing (the router's own
    choices).  With ``slot_of`` from a rerouting dispatch, rows_kept,
    dropped and drop_rate count the assignments served after rerouting and
    ``rerouted`` those served by a fallback expert."""
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    counts = token_count_per_expert(idx, E)
    kept = counts if cap < 0 else np.minimum(counts, cap)
    served = int(kept.sum()) if slot_of is None else int((np.asarray(slot_of) >= 0).sum())
    return {
        "aux_loss": switch_aux_loss(idx, gates, E),
        "imbalance": imbalance(counts, T, k, E),
        "drop_rate": (T * k - served) / (T * k) if T * k else 0.0,
        "rows_kept": served,
        "max_count": int(counts.max()),
        "dropped": T * k - served,
        "rerouted": served - int(kept.sum()),
    }


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def moe_layer(inputs, k: int, cap: int, reroute: int = 0) -> Dict[str, np.ndarray]:
    """Router -> dispatch -> expert FFN -> combine, all in float64.

    With shared experts in ``inputs`` (keys shared_w1 [S,ff,d], shared_b1
    [S,ff], shared_w2 [S,d,ff], shared_b2 [S,d]) their ungated sum over all
    tokens is added to the routed output; routing and statistics are those
    of the routed experts alone.  ``reroute`` > 0 gives dropped assignments
    that many rounds of fallback experts (dispatch_reroute).
    """
    E = inputs["w_router"].shape[0]
    if reroute <= 0:
        r = route(inputs["x"], inputs["w_router"], k, inputs.get("logit_bias"))
        dsp = dispatch(r["topk_idx"], E, cap)
        out = moe_forward(inputs["x"], inputs, r["topk_idx"], r["topk_gate"], dsp["slot_of"])
    else:
        r = route(inputs["x"], inputs["w_router"], k + reroute, inputs.get("logit_bias"))
        ranked_idx, ranked_gate = r["topk_idx"], r["topk_gate"]
        r["ranked_idx"], r["ranked_gate"] = ranked_idx, ranked_gate
        r["topk_idx"], r["topk_gate"] = ranked_idx[:, :k], ranked_gate[:, :k]
        dsp = dispatch_reroute(ranked_idx, ranked_gate, k, E, cap, reroute)
        out = moe_forward(inputs["x"], inputs, dsp["final_idx"], dsp["final_gate"], dsp["slot_of"])
    if has_shared(inputs):
        out = out + shared_experts(inputs["x"], inputs)
    r.update(dsp)
    r["out"] = out
    r["stats"] = layer_stats(r["topk_idx"], r["gates"], E, cap, slot_of=dsp["slot_of"])
    return r
