"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import build as build_mod
from oracle import moe_ref

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return _lib.load()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_surface():
    assert header_functions() == _lib.EXPORTED


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert _lib.moe_version() == 10000
    for code in range(7):
        assert _lib.status_string(code) not in ("", "unknown status")
    assert _lib.status_string(99) == "unknown status"


@pytest.mark.parametrize("T,k,E,cf", [(4096, 1, 32, 1.0), (4096, 1, 32, 1.5), (16384, 1, 64, 1.25),
                                      (1024, 2, 8, 1.0), (10, 1, 3, 1.0), (7, 3, 5, 0.7), (100, 2, 7, 2.5),
                                      (1024, 2, 8, None), (1024, 2, 8, 0.0), (1024, 2, 8, -1.0)])
def test_capacity_matches_oracle(lib, T, k, E, cf):
    assert _lib.moe_capacity(T, k, E, cf) == moe_ref.capacity(T, k, E, cf)


def test_workspace_size(lib):
    a = _lib.moe_workspace_size(4096, 768, 3072, 32, 1, _lib.MOE_BF16)
    b = _lib.moe_workspace_size(4096, 768, 3072, 32, 1, _lib.MOE_F32)
    assert a > 4096 * (768 * 2 + 3072) * 2          # bf16 grouped activations xp, h, yp
    assert b > 4096 * (768 * 2 + 3072) * 4          # fp32 grouped activations
    assert _lib.moe_workspace_size(4096, 12, 3072, 32, 1, _lib.MOE_BF16) == 0     # d % 8
    assert _lib.moe_workspace_size(4096, 768, 3072, 32, 33, _lib.MOE_BF16) == 0   # k > E
    assert _lib.moe_workspace_size(4096, 768, 3072, 300, 1, _lib.MOE_BF16) == 0   # E too large
    assert _lib.moe_dispatch_workspace_size(4096, 1, 32) > 0
    assert _lib.moe_dispatch_workspace_size(-1, 1, 32) == 0


FAKE = 1 << 20          # an aligned non-null address that is never dereferenced
MISALIGNED = FAKE + 4


def router(lib, **kw):
    a = dict(x=FAKE, w=FAKE, bias=None, T=64, d=64, E=8, k=2, dtype=_lib.MOE_BF16, idx=FAKE, gate=FAKE, psum=None)
    a.update(kw)
    return lib.moe_router_topk(a["x"], a["w"], a["bias"], a["T"], a["d"], a["E"], a["k"], a["dtype"],
                               a["idx"], a["gate"], a["psum"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=9), _lib.MOE_ERR_INVALID_ARG),            # k > E
    (dict(E=300, k=2), _lib.MOE_ERR_UNSUPPORTED),      # E > 256
    (dict(E=16, k=9), _lib.MOE_ERR_UNSUPPORTED),       # k > 8
    (dict(dtype=7), _lib.MOE_ERR_UNSUPPORTED),
    (dict(d=12), _lib.MOE_ERR_UNSUPPORTED),
    (dict(T=-1), _lib.MOE_ERR_INVALID_ARG),
    (dict(x=None), _lib.MOE_ERR_INVALID_ARG),
    (dict(idx=None), _lib.MOE_ERR_INVALID_ARG),
    (dict(x=MISALIGNED), _lib.MOE_ERR_INVALID_ARG),
    (dict(T=1 << 30, k=2), _lib.MOE_ERR_UNSUPPORTED),  # T*k overflows int32
])
def test_router_rejects_bad_arguments(lib, kw, code):
    assert router(lib, **kw) == code


def forward(lib, ws_bytes, ws=FAKE, **kw):
    a = dict(T=256, d=64, ff=128, E=8, k=2, cap=-1, dtype=_lib.MOE_BF16, out=FAKE)
    a.update(kw)
    return lib.moe_forward(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, a["T"], a["d"], a["ff"], a["E"], a["k"],
                           a["cap"], a["dtype"], a["out"], None, None, None, ws, ws_bytes, None)


def test_forward_checks_workspace(lib):
    need = _lib.moe_workspace_size(256, 64, 128, 8, 2, _lib.MOE_BF16)
    assert forward(lib, need - 1) == _lib.MOE_ERR_WORKSPACE
    assert forward(lib, need, ws=None) == _lib.MOE_ERR_WORKSPACE
    assert forward(lib, need, ws=FAKE + 16) == _lib.MOE_ERR_WORKSPACE      # not 256-byte aligned
    assert forward(lib, need, out=None) == _lib.MOE_ERR_INVALID_ARG
    assert forward(lib, need, ff=100) == _lib.MOE_ERR_UNSUPPORTED
    assert forward(lib, 0, T=0) == _lib.MOE_OK                              # empty batch: nothing to do


def test_dispatch_checks(lib):
    ws_need = _lib.moe_dispatch_workspace_size(100, 2, 8)
    call = lambda **kw: lib.moe_dispatch(
        kw.get("idx", FAKE), kw.get("gate", None), 100, 2, 8, -1, FAKE, FAKE, FAKE, FAKE, None,
        kw.get("row_gate", None), kw.get("x", None), kw.get("xp", None), 64, _lib.MOE_BF16,
        kw.get("ws", FAKE), kw.get("ws_bytes", ws_need), None)
    assert call(ws_bytes=ws_need - 1) == _lib.MOE_ERR_WORKSPACE
    assert call(row_gate=FAKE) == _lib.MOE_ERR_INVALID_ARG          # row_gate needs topk_gate
    assert call(x=FAKE) == _lib.MOE_ERR_INVALID_ARG                 # x without xp
    assert call(idx=None) == _lib.MOE_ERR_INVALID_ARG


def test_grouped_ffn_and_combine_checks(lib):
    assert lib.moe_grouped_ffn(FAKE, FAKE, 64, 8, 64, 128, FAKE, FAKE, FAKE, MISALIGNED, None, FAKE, FAKE,
                               _lib.MOE_BF16, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(FAKE, FAKE, None, 64, 9, 64, _lib.MOE_BF16, FAKE, None) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_combine(None, FAKE, None, 64, 2, 64, _lib.MOE_BF16, FAKE, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_stats(FAKE, FAKE, FAKE, 0, 1, 8, FAKE, None) == _lib.MOE_ERR_INVALID_ARG


def test_no_launch_and_timing_read_without_gpu(lib):
    assert _lib.moe_launch_count() == 0
    assert lib.moe_timing_enable(0) == _lib.MOE_OK
    t = _lib.moe_timing_read()
    assert set(t) == set(_lib.KERNEL_NAMES) and all(v == (0.0, 0) for v in t.values())


def test_ffn_clock_calls_fail_cleanly_without_gpu(lib):
    """Without a device the clock record's calls report MOE_ERR_CUDA (they
    touch device memory) and launch nothing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.moe_ffn_clock_enable(1) == _lib.MOE_ERR_CUDA
    mhz = (ctypes.c_double * 2)()
    assert lib.moe_ffn_clock_read(ctypes.cast(mhz, ctypes.c_void_p), None) == _lib.MOE_ERR_CUDA
    assert _lib.moe_launch_count() == 0


def test_shared_workspace_size_and_offsets(lib):
    T, d, ff, E, k = 4096, 768, 3072, 32, 1
    base = _lib.moe_workspace_size(T, d, ff, E, k, _lib.MOE_BF16)
    assert _lib.moe_forward_ex_workspace_size(T, d, ff, E, k, 0, 0, _lib.MOE_BF16) == base
    two = _lib.moe_forward_ex_workspace_size(T, d, ff, E, k, 2, 0, _lib.MOE_BF16)
    assert two >= base + 2 * T * (ff + d) * 2          # S*T more rows of h and yp
    # routed rows first, then the shared rows: yp holds (T*k + S*T) rows
    yp = _lib.moe_forward_ex_workspace_offset(T, d, ff, E, k, 2, 0, _lib.MOE_BF16, "yp")
    h = _lib.moe_forward_ex_workspace_offset(T, d, ff, E, k, 2, 0, _lib.MOE_BF16, "h")
    assert yp - h >= (T * k + 2 * T) * ff * 2
    assert _lib.moe_forward_ex_workspace_size(T, d, ff, E, k, _lib.MOE_MAX_SHARED + 1, 0, _lib.MOE_BF16) == 0
    assert _lib.moe_forward_ex_workspace_size(T, d, ff, E, k, -1, 0, _lib.MOE_BF16) == 0
    assert _lib.moe_forward_ex_workspace_size(1 << 28, d, ff, E, k, 7, 0, _lib.MOE_BF16) == 0   # T*(k+S) overflows


def forward_shared(lib, ws_bytes, ws=FAKE, S=2, shared=FAKE, F=0, **kw):
    a = dict(T=256, d=64, ff=128, E=8, k=2, cap=-1, dtype=_lib.MOE_BF16, out=FAKE)
    a.update(kw)
    return lib.moe_forward_ex(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, S, shared, FAKE, FAKE, FAKE, F,
                              a["T"], a["d"], a["ff"], a["E"], a["k"], a["cap"], a["dtype"], a["out"], None,
                              None, None, ws, ws_bytes, None)


def test_forward_shared_checks(lib):
    need = _lib.moe_forward_ex_workspace_size(256, 64, 128, 8, 2, 2, 0, _lib.MOE_BF16)
    assert need > _lib.moe_workspace_size(256, 64, 128, 8, 2, _lib.MOE_BF16)
    assert forward_shared(lib, need - 1) == _lib.MOE_ERR_WORKSPACE
    assert forward_shared(lib, need, shared=None) == _lib.MOE_ERR_INVALID_ARG
    assert forward_shared(lib, need, shared=MISALIGNED) == _lib.MOE_ERR_INVALID_ARG
    assert forward_shared(lib, need, S=-1) == _lib.MOE_ERR_INVALID_ARG
    assert forward_shared(lib, need, S=_lib.MOE_MAX_SHARED + 1) == _lib.MOE_ERR_UNSUPPORTED
    assert forward_shared(lib, 0, T=0) == _lib.MOE_OK
    # S = 0 needs no shared pointers and exactly moe_forward's workspace
    base = _lib.moe_workspace_size(256, 64, 128, 8, 2, _lib.MOE_BF16)
    assert forward_shared(lib, base - 1, S=0, shared=None) == _lib.MOE_ERR_WORKSPACE


def test_shared_ffn_and_combine_checks(lib):
    call = lambda **kw: lib.moe_shared_ffn(kw.get("x", FAKE), kw.get("T", 64), 64, 128, kw.get("S", 2),
                                           kw.get("w1", FAKE), FAKE, FAKE, FAKE, kw.get("h", FAKE), FAKE,
                                           _lib.MOE_BF16, None)
    assert call(x=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(w1=MISALIGNED) == _lib.MOE_ERR_INVALID_ARG
    assert call(h=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(S=9) == _lib.MOE_ERR_UNSUPPORTED
    assert call(S=0, x=None) == _lib.MOE_OK          # nothing to do
    assert call(T=0, x=None) == _lib.MOE_OK
    comb = lambda **kw: lib.moe_combine_shared(FAKE, FAKE, None, kw.get("ys", FAKE), kw.get("S", 2), 64, 2, 64,
                                               _lib.MOE_BF16, FAKE, None)
    assert comb(ys=None) == _lib.MOE_ERR_INVALID_ARG
    assert comb(ys=MISALIGNED) == _lib.MOE_ERR_INVALID_ARG
    assert comb(S=9) == _lib.MOE_ERR_UNSUPPORTED
    assert comb(S=-1) == _lib.MOE_ERR_INVALID_ARG


def test_reroute_checks(lib):
    # workspace grows with the rounds; k + F must fit the router's selection and E
    base = _lib.moe_forward_ex_workspace_size(4096, 768, 3072, 32, 1, 0, 0, _lib.MOE_BF16)
    one = _lib.moe_forward_ex_workspace_size(4096, 768, 3072, 32, 1, 0, 1, _lib.MOE_BF16)
    three = _lib.moe_forward_ex_workspace_size(4096, 768, 3072, 32, 1, 0, 3, _lib.MOE_BF16)
    assert base < one < three
    assert _lib.moe_forward_ex_workspace_size(4096, 768, 3072, 32, 2, 0, 7, _lib.MOE_BF16) == 0   # k + F > 8
    assert _lib.moe_forward_ex_workspace_size(64, 64, 64, 3, 2, 0, 2, _lib.MOE_BF16) == 0         # k + F > E
    assert _lib.moe_forward_ex_workspace_size(64, 64, 64, 3, 2, 0, -1, _lib.MOE_BF16) == 0
    fb = _lib.moe_forward_ex_workspace_offset(4096, 768, 3072, 32, 1, 0, 2, _lib.MOE_BF16, "fallback_idx")
    fg = _lib.moe_forward_ex_workspace_offset(4096, 768, 3072, 32, 1, 0, 2, _lib.MOE_BF16, "fallback_gate")
    assert fg - fb >= 4096 * 2 * 4
    need = _lib.moe_forward_ex_workspace_size(256, 64, 128, 8, 2, 0, 2, _lib.MOE_BF16)
    assert forward_shared(lib, need - 1, S=0, shared=None, F=2, cap=10) == _lib.MOE_ERR_WORKSPACE
    assert forward_shared(lib, need, S=0, shared=None, F=7, cap=10) == _lib.MOE_ERR_UNSUPPORTED
    assert forward_shared(lib, need, S=0, shared=None, F=-2, cap=10) == _lib.MOE_ERR_INVALID_ARG
    # step form
    nws = _lib.moe_dispatch_reroute_workspace_size(1000, 2, 2, 8)
    assert nws > 0 and _lib.moe_dispatch_reroute_workspace_size(1000, 2, 7, 8) == 0
    call = lambda **kw: lib.moe_dispatch_reroute(
        kw.get("idx", FAKE), kw.get("gate", None), 1000, 2, kw.get("F", 2), 8, 100, FAKE, FAKE, FAKE, FAKE, None,
        kw.get("row_gate", None), kw.get("x", None), kw.get("xp", None), 64, _lib.MOE_BF16,
        kw.get("ws", FAKE), kw.get("ws_bytes", nws), None)
    assert call(ws_bytes=nws - 1) == _lib.MOE_ERR_WORKSPACE
    assert call(ws=FAKE + 16) == _lib.MOE_ERR_WORKSPACE
    assert call(row_gate=FAKE) == _lib.MOE_ERR_INVALID_ARG
    assert call(idx=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(x=FAKE) == _lib.MOE_ERR_INVALID_ARG
    assert call(F=7) == _lib.MOE_ERR_UNSUPPORTED


def test_wait_timeout_probe_checks_its_limit(lib):
    assert lib.moe_debug_wait_timeout(0, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_wait_timeout(-5, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_wait_timeout(3_000_000_000, None) == _lib.MOE_ERR_INVALID_ARG   # above the 2 s cap


def test_pipeline_checks(lib):
    """moe_pipeline_create / run / destroy reject bad arguments before any CUDA call."""
    T, d, ff, E, k = 256, 64, 128, 8, 2
    need = lib.moe_forward_ex_workspace_size(T, d, ff, E, k, 0, 0, _lib.MOE_BF16)
    arr = lambda *v: (ctypes.c_void_p * len(v))(*v)
    handle = ctypes.c_void_p(FAKE)

    def create(depth=2, x=None, o=None, ws=None, ws_bytes=need, flags=_lib.MOE_PIPELINE_GRAPHS, out=True, T=T,
               E=E):
        x = arr(*([FAKE] * depth)) if x is None else x
        o = arr(*([FAKE] * depth)) if o is None else o
        ws = arr(*([FAKE] * depth)) if ws is None else ws
        return lib.moe_pipeline_create(FAKE, None, FAKE, FAKE, FAKE, FAKE, 0, None, None, None, None, 0, T, d, ff,
                                       E, k, -1, _lib.MOE_BF16, depth, x, o, ws, ws_bytes, flags,
                                       ctypes.byref(handle) if out else None)

    assert create(out=False) == _lib.MOE_ERR_INVALID_ARG
    assert handle.value == FAKE                                          # untouched without an out pointer
    assert create(depth=0) == _lib.MOE_ERR_INVALID_ARG
    assert create(depth=_lib.MOE_PIPELINE_MAX_DEPTH + 1) == _lib.MOE_ERR_INVALID_ARG
    assert handle.value is None                                          # cleared on every other failure
    assert create(flags=2) == _lib.MOE_ERR_INVALID_ARG
    assert create(T=0) == _lib.MOE_ERR_INVALID_ARG
    assert create(E=_lib.MOE_MAX_EXPERTS + 1) == _lib.MOE_ERR_INVALID_ARG           # sizes the layer rejects
    assert create(x=arr(FAKE, None)) == _lib.MOE_ERR_INVALID_ARG
    assert create(o=arr(FAKE, MISALIGNED)) == _lib.MOE_ERR_INVALID_ARG
    assert create(ws_bytes=need - 1) == _lib.MOE_ERR_WORKSPACE
    assert create(ws=arr(FAKE, FAKE + 16)) == _lib.MOE_ERR_WORKSPACE    # not 256-byte aligned
    assert lib.moe_pipeline_run(None, None, None, 0, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_run(FAKE, None, None, -1, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_run(FAKE, None, None, 2, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_run(FAKE, arr(FAKE, None), arr(FAKE, FAKE), 2, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_destroy(None) == _lib.MOE_OK


def test_nvtx_ranges_default_off_and_switch(lib, monkeypatch):
    """The profiler ranges are off unless asked for; the switch returns the
    previous setting; calls that reject their arguments still work with the
    ranges on (no GPU needed)."""
    if os.environ.get("MOE_NVTX") == "1":
        pytest.skip("MOE_NVTX=1 in this environment")
    assert _lib.moe_trace_enabled() is False
    assert _lib.moe_trace_enable(True) is False
    try:
        assert _lib.moe_trace_enabled() is True
        rc = lib.moe_combine(None, None, None, 4, 1, 8, _lib.MOE_F32, None, None)
        assert rc == _lib.MOE_ERR_INVALID_ARG
    finally:
        assert _lib.moe_trace_enable(False) is True
    assert _lib.moe_trace_enabled() is False
