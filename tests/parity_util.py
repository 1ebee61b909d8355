"""Comparison helpers for the GPU parity tests (test infrastructure).

Tolerances: the float outputs are compared with the max-norm relative error
max|y - r| / max|r| against the float64 oracle r: at most 1e-4 for fp32
paths and 2e-2 for bf16 paths.  Integer outputs (routing indices away from
floating-point near-ties, counts, offsets, permutation, slots, drop set) are
compared bit for bit.
"""
from __future__ import annotations

import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}

# unit roundoff used for the fp32 logit error bound (2^-23 covers round-to-
# nearest and truncating accumulation alike)
U32 = 2.0 ** -23


def max_rel_err(y, r) -> float:
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    den = np.abs(r).max()
    if den == 0:
        return float(np.abs(y).max())
    return float(np.abs(y - r).max() / den)


def logit_error_bound(x, w_router, logit_bias=None) -> np.ndarray:
    """Per-token bound on |fp32 logit - exact logit| for a d-term fp32 dot
    product (Higham's gamma_d * sum |x_i||w_i|), plus the bias addition and
    final rounding.  Returned per token as the max over experts."""
    x = np.abs(np.asarray(x, np.float64))
    w = np.abs(np.asarray(w_router, np.float64))
    d = x.shape[1]
    gamma = d * U32 / (1.0 - d * U32)
    mag = x @ w.T                                    # [T, E] sum |x||w|
    bias_mag = 0.0 if logit_bias is None else np.abs(np.asarray(logit_bias, np.float64))[None, :]
    return (gamma * mag + 2 * U32 * (mag + bias_mag)).max(axis=1)


def check_routing(gpu_idx, logits, k, delta):
    """Validate GPU top-k indices against float64 logits.

    * every row holds k distinct experts in range;
    * the chosen set and its order are correct up to ties within 2*delta_t
      (the GPU's logits are each within delta_t of the exact ones);
    * rows whose decisive gaps all exceed 2*delta_t match the oracle exactly.
    Returns (number of rows that differ from the oracle, number of undecided rows).
    """
    gpu_idx = np.asarray(gpu_idx, np.int64)
    L = np.asarray(logits, np.float64)
    T, E = L.shape
    assert gpu_idx.shape == (T, k)
    assert gpu_idx.min() >= 0 and gpu_idx.max() < E
    s = np.sort(gpu_idx, axis=1)
    assert np.all(s[:, 1:] != s[:, :-1]), "repeated expert in a row"
    tol = 2 * np.asarray(delta)[:, None]
    chosen = np.take_along_axis(L, gpu_idx, 1)
    assert np.all(chosen[:, :-1] >= chosen[:, 1:] - tol), "slot order violated beyond the error bound"
    if k < E:
        mask = np.ones_like(L, bool)
        np.put_along_axis(mask, gpu_idx, False, 1)
        best_out = np.where(mask, L, -np.inf).max(1)
        assert np.all(chosen.min(1) >= best_out - tol[:, 0]), "a better expert was left out"
    # oracle order: largest first, ties to the lower index
    order = np.argsort(-L, axis=1, kind="stable")
    ref = order[:, :k]
    srt = np.take_along_axis(L, order[:, :min(k + 1, E)], 1)
    gaps = srt[:, :-1] - srt[:, 1:]
    decided = np.all(gaps > tol, axis=1) if gaps.shape[1] else np.ones(T, bool)
    diff = np.any(gpu_idx != ref, axis=1)
    assert not np.any(diff & decided), f"{int((diff & decided).sum())} decided rows differ from the oracle"
    return int(diff.sum()), int((~decided).sum())


def sample_rows(T: int, n: int, seed: int = 0, must=()) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in rng.choice(T, size=min(n, T), replace=False))
    rows.update(int(m) for m in must if 0 <= m < T)
    rows.update([0, T - 1])
    return np.array(sorted(rows))


def tile_covering_rows(offsets, perm, k: int, T: int, tile: int = 128, seed: int = 0, shared: int = 0) -> np.ndarray:
    """Output tokens whose rows together reach every `tile`-row M tile of the
    grouped FFN.

    For each expert group (grouped rows offsets[e] .. offsets[e+1]-1, tiles
    starting at offsets[e]) one random row of every tile and the group's last
    row are taken, each mapped to its token perm[row] // k.  Tiles of 2*tile
    rows (the CTA-pair kernel) are unions of two such tiles, so they are
    reached too; a token's output row depends on every N tile of both GEMMs.
    With shared experts (each a group of all T tokens in order) one token of
    every `tile`-token block is added as well.
    """
    rng = np.random.default_rng(seed)
    offsets = np.asarray(offsets, np.int64)
    perm = np.asarray(perm, np.int64)
    toks = set()
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for t0 in range(lo, hi, tile):
            t1 = min(t0 + tile, hi)
            toks.add(int(perm[int(rng.integers(t0, t1))] // k))
        if hi > lo:
            toks.add(int(perm[hi - 1] // k))
    if shared:
        for t0 in range(0, T, tile):
            toks.add(int(rng.integers(t0, min(t0 + tile, T))))
    return np.array(sorted(toks), dtype=np.int64)


def m_tiles(offsets, tile: int = 128) -> int:
    """M tiles of `tile` rows over the expert groups of the grouped layout."""
    offsets = np.asarray(offsets, np.int64)
    return int(sum(-(-int(offsets[e + 1] - offsets[e]) // tile) for e in range(len(offsets) - 1)))
