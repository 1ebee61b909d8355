"""moe_dispatch_noalloc: dispatch for callers that cannot allocate device
memory (a runtime whose allocator already owns the whole device, or a
latency-critical path that must not call cudaMalloc), using the library's
fixed scratch array instead of a caller workspace.

Checked through the C ABI against moe_dispatch (which takes a workspace)
on two calls in a row with different sizes; dispatch is integer work, so
the outputs must agree bit for bit.  This file is collected last so that a
run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_45_b200 import _lib

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(T, k, E, d, dtype):
    A = max(T * k, 1)
    tdt = torch.bfloat16 if dtype == _lib.MOE_BF16 else torch.float32
    return dict(
        counts=torch.full((E,), -1, dtype=torch.int32, device=DEV),
        offsets=torch.full((E + 1,), -1, dtype=torch.int32, device=DEV),
        perm=torch.full((A,), -1, dtype=torch.int32, device=DEV),
        slot_of=torch.full((A,), -9, dtype=torch.int32, device=DEV),
        drop=torch.full((A,), 7, dtype=torch.uint8, device=DEV),
        row_gate=torch.full((A,), -1.0, dtype=torch.float32, device=DEV),
        xp=torch.zeros((A, d), dtype=tdt, device=DEV),
    )


def _case(seed, T, k, E, d, cap, dtype):
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.ones(E) * 0.5)
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == _lib.MOE_BF16 else torch.float32
    x = torch.from_numpy(rng.normal(size=(T, d)).astype(np.float32)).to(DEV, tdt)
    return torch.from_numpy(idx).to(DEV), torch.from_numpy(gate).to(DEV), x


def _run_both(seed, T, k, E, d, cap, dtype):
    idx, gate, x = _case(seed, T, k, E, d, cap, dtype)
    a = _outputs(T, k, E, d, dtype)
    _lib.moe_dispatch_noalloc(idx, gate, T, k, E, cap, a["counts"], a["offsets"], a["perm"], a["slot_of"],
                              a["drop"], a["row_gate"], x, a["xp"], d, dtype)
    b = _outputs(T, k, E, d, dtype)
    nws = _lib.moe_dispatch_workspace_size(T, k, E)
    ws = torch.empty(nws, dtype=torch.uint8, device=DEV)
    _lib.moe_dispatch(idx, gate, T, k, E, cap, b["counts"], b["offsets"], b["perm"], b["slot_of"], b["drop"],
                      b["row_gate"], x, b["xp"], d, dtype, ws, nws)
    assert _lib.moe_get_error() == _lib.MOE_OK
    for key in a:
        assert torch.equal(a[key].view(torch.uint8), b[key].view(torch.uint8)), key
    return a


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    assert torch.cuda.is_available()
    # first call: top-2 over 64 experts with capacity drops, bf16 rows
    a = _run_both(1, T=20000, k=2, E=64, d=256, cap=500, dtype=_lib.MOE_BF16)
    assert int(a["drop"][:40000].sum()) > 0
    # second call in a row reuses the same fixed scratch with other sizes
    a = _run_both(2, T=3001, k=1, E=7, d=64, cap=-1, dtype=_lib.MOE_F32)
    assert int(a["offsets"][-1]) == 3001


def test_noalloc_dispatch_rejects_sizes_beyond_its_limit():
    T = _lib.MOE_NOALLOC_MAX_ASSIGNMENTS // 2 + 1
    dummy = torch.empty(16, dtype=torch.int32, device=DEV)
    with pytest.raises(_lib.MoeError) as ei:
        _lib.moe_dispatch_noalloc(dummy, None, T, 2, 8, -1, dummy, dummy, dummy, dummy, None, None, None, None,
                                  8, _lib.MOE_F32)
    assert ei.value.status == _lib.MOE_ERR_WORKSPACE


def test_noalloc_dispatch_at_its_exact_limit():
    """T*k exactly MOE_NOALLOC_MAX_ASSIGNMENTS with the most experts: the
    per-chunk histograms and bases then fill the fixed scratch to its last
    byte.  The call is accepted and agrees bit for bit with moe_dispatch."""
    A = _lib.MOE_NOALLOC_MAX_ASSIGNMENTS
    E, k, d = _lib.MOE_MAX_EXPERTS, 2, 64
    T = A // k
    rng = np.random.default_rng(9)
    p = rng.dirichlet(np.ones(E) * 0.5)
    first = rng.choice(E, size=T, p=p)
    second = (first + 1 + rng.integers(0, E - 1, size=T)) % E          # a different expert
    idx = torch.from_numpy(np.stack([first, second], 1).astype(np.int32)).to(DEV)
    gate = torch.from_numpy(rng.random((T, k)).astype(np.float32)).to(DEV)
    x = torch.from_numpy(rng.normal(size=(T, d)).astype(np.float32)).to(DEV, torch.bfloat16)
    cap = int(T * k / E)                                                 # capacity factor 1.0: drops
    a = _outputs(T, k, E, d, _lib.MOE_BF16)
    _lib.moe_dispatch_noalloc(idx, gate, T, k, E, cap, a["counts"], a["offsets"], a["perm"], a["slot_of"],
                              a["drop"], a["row_gate"], x, a["xp"], d, _lib.MOE_BF16)
    b = _outputs(T, k, E, d, _lib.MOE_BF16)
    nws = _lib.moe_dispatch_workspace_size(T, k, E)
    ws = torch.empty(nws, dtype=torch.uint8, device=DEV)
    _lib.moe_dispatch(idx, gate, T, k, E, cap, b["counts"], b["offsets"], b["perm"], b["slot_of"], b["drop"],
                      b["row_gate"], x, b["xp"], d, _lib.MOE_BF16, ws, nws)
    assert _lib.moe_get_error() == _lib.MOE_OK
    for key in a:
        assert torch.equal(a[key].view(torch.uint8), b[key].view(torch.uint8)), key
    assert int(a["counts"].sum()) == A and int(a["drop"].sum()) > 0
