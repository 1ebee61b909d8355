"""ctypes binding of libmoe (include/moe.h): the same entry points, argument
marshalling only.  Every computation happens in the CUDA library; there is
no Python or CPU fallback, and a missing library raises on first use.

Tensors are passed as torch tensors (or None for a NULL pointer) and
reduced to their device pointers; ``stream`` is a ``torch.cuda.Stream``, a
raw ``cudaStream_t`` integer, or None for torch's current stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_BAD_ROUTING = 5
MOE_ERR_TIMEOUT = 6

MOE_F32 = 0
MOE_BF16 = 1
MOE_MAX_EXPERTS = 256
MOE_MAX_TOPK = 8
MOE_MAX_SHARED = 8
MOE_PIPELINE_GRAPHS = 1
MOE_PIPELINE_MAX_DEPTH = 8

KERNEL_NAMES = ["router", "count", "scan", "permute", "gather", "ffn1", "ffn2", "combine", "stats", "reroute"]
MOE_NUM_KERNELS = len(KERNEL_NAMES)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class MoeStats(ctypes.Structure):
    _fields_ = [("aux_loss", ctypes.c_float), ("imbalance", ctypes.c_float), ("drop_rate", ctypes.c_float),
                ("rows_kept", ctypes.c_int32), ("max_count", ctypes.c_int32), ("dropped", ctypes.c_int32),
                ("rerouted", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_version": (_I, []),
    "moe_capacity": (_I, [_I, _I, _I, ctypes.c_double]),
    "moe_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "moe_dispatch_workspace_size": (ctypes.c_size_t, [_I, _I, _I]),
    "moe_workspace_offset": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "moe_router_topk": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "moe_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P,
                          ctypes.c_size_t, _P]),
    "moe_dispatch_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P]),
    "moe_grouped_ffn": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "moe_layer_stats": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_forward": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                         ctypes.c_size_t, _P]),
    "moe_forward_ex_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "moe_forward_ex_workspace_offset": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "moe_forward_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                            _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_dispatch_reroute_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "moe_dispatch_reroute": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P,
                                  ctypes.c_size_t, _P]),
    "moe_shared_ffn": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P]),
    "moe_combine_shared": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "moe_pipeline_create": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                 _I, _P, _P, _P, ctypes.c_size_t, _I, _P]),
    "moe_pipeline_run": (_I, [_P, _P, _P, _I, _P]),
    "moe_pipeline_destroy": (_I, [_P]),
    "moe_get_error": (_I, [_P]),
    "moe_debug_gelu": (_I, [_P, _P, _I, _I, _P]),
    "moe_debug_wait_timeout": (_I, [ctypes.c_int64, _P]),
    "moe_launch_count": (ctypes.c_uint64, []),
    "moe_timing_enable": (_I, [_I]),
    "moe_timing_read": (_I, [_P, _P]),
    "moe_trace_enable": (_I, [_I]),
    "moe_ffn_clock_enable": (_I, [_I]),
    "moe_ffn_clock_read": (_I, [_P, _P]),
    "moe_trace_enabled": (_I, []),
}
EXPORTED = sorted(_SIGS)

_lib = None
_lock = threading.Lock()


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"libmoe.so not found at {path}; build it with "
                                   "`python -m mixture_experts_layer_45_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoeError(rc, where)


# ---- entry points (names as in include/moe.h) -----------------------------

def moe_version() -> int:
    return load().moe_version()


def moe_capacity(T: int, k: int, E: int, cf) -> int:
    return load().moe_capacity(T, k, E, 0.0 if cf is None else float(cf))


def moe_workspace_size(T, d, ff, E, k, dtype) -> int:
    return load().moe_workspace_size(T, d, ff, E, k, dtype)


WS_VIEWS = {"topk_idx": 0, "topk_gate": 1, "counts": 2, "offsets": 3, "perm": 4, "slot_of": 5, "row_gate": 6,
            "xp": 7, "h": 8, "yp": 9, "fallback_idx": 10, "fallback_gate": 11}


def moe_workspace_offset(T, d, ff, E, k, dtype, which) -> int:
    code = WS_VIEWS[which] if isinstance(which, str) else which
    return load().moe_workspace_offset(T, d, ff, E, k, dtype, code)


def moe_dispatch_workspace_size(T, k, E) -> int:
    return load().moe_dispatch_workspace_size(T, k, E)


def moe_router_topk(x, w_router, logit_bias, T, d, E, k, dtype, topk_idx, topk_gate, prob_sum, stream=None):
    _check(load().moe_router_topk(_ptr(x), _ptr(w_router), _ptr(logit_bias), T, d, E, k, dtype,
                                  _ptr(topk_idx), _ptr(topk_gate), _ptr(prob_sum), _stream(stream)),
           "moe_router_topk")


def moe_dispatch(topk_idx, topk_gate, T, k, E, capacity, counts, offsets, perm, slot_of, drop_mask, row_gate,
                 x, xp, d, dtype, ws, ws_bytes, stream=None):
    _check(load().moe_dispatch(_ptr(topk_idx), _ptr(topk_gate), T, k, E, capacity, _ptr(counts), _ptr(offsets),
                               _ptr(perm), _ptr(slot_of), _ptr(drop_mask), _ptr(row_gate), _ptr(x), _ptr(xp),
                               d, dtype, _ptr(ws), ws_bytes, _stream(stream)),
           "moe_dispatch")


MOE_NOALLOC_MAX_ASSIGNMENTS = 1 << 20


def moe_dispatch_noalloc(topk_idx, topk_gate, T, k, E, capacity, counts, offsets, perm, slot_of, drop_mask,
                         row_gate, x, xp, d, dtype, stream=None):
    """moe_dispatch with the library's fixed scratch instead of a workspace."""
    _check(load().moe_dispatch_noalloc(_ptr(topk_idx), _ptr(topk_gate), T, k, E, capacity, _ptr(counts),
                                       _ptr(offsets), _ptr(perm), _ptr(slot_of), _ptr(drop_mask), _ptr(row_gate),
                                       _ptr(x), _ptr(xp), d, dtype, _stream(stream)),
           "moe_dispatch_noalloc")


def moe_grouped_ffn(xp, offsets, max_rows, E, d, ff, w1, b1, w2, b2, row_gate, h, yp, dtype, stream=None):
    _check(load().moe_grouped_ffn(_ptr(xp), _ptr(offsets), max_rows, E, d, ff, _ptr(w1), _ptr(b1), _ptr(w2),
                                  _ptr(b2), _ptr(row_gate), _ptr(h), _ptr(yp), dtype, _stream(stream)),
           "moe_grouped_ffn")


def moe_combine(yp, slot_of, topk_gate, T, k, d, dtype, out, stream=None):
    _check(load().moe_combine(_ptr(yp), _ptr(slot_of), _ptr(topk_gate), T, k, d, dtype, _ptr(out),
                              _stream(stream)),
           "moe_combine")


def moe_layer_stats(counts, offsets, prob_sum, T, k, E, stats, stream=None):
    _check(load().moe_layer_stats(_ptr(counts), _ptr(offsets), _ptr(prob_sum), T, k, E, _ptr(stats),
                                  _stream(stream)),
           "moe_layer_stats")


def moe_forward(x, w_router, logit_bias, w1, b1, w2, b2, T, d, ff, E, k, capacity, dtype, out, stats,
                topk_idx_out, topk_gate_out, ws, ws_bytes, stream=None):
    _check(load().moe_forward(_ptr(x), _ptr(w_router), _ptr(logit_bias), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2),
                              T, d, ff, E, k, capacity, dtype, _ptr(out), _ptr(stats), _ptr(topk_idx_out),
                              _ptr(topk_gate_out), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_forward")


def moe_forward_ex_workspace_size(T, d, ff, E, k, S, F, dtype) -> int:
    return load().moe_forward_ex_workspace_size(T, d, ff, E, k, S, F, dtype)


def moe_forward_ex_workspace_offset(T, d, ff, E, k, S, F, dtype, which) -> int:
    code = WS_VIEWS[which] if isinstance(which, str) else which
    return load().moe_forward_ex_workspace_offset(T, d, ff, E, k, S, F, dtype, code)


def moe_forward_ex(x, w_router, logit_bias, w1, b1, w2, b2, S, w1s, b1s, w2s, b2s, reroute_rounds, T, d, ff, E, k,
                   capacity, dtype, out, stats, topk_idx_out, topk_gate_out, ws, ws_bytes, stream=None):
    _check(load().moe_forward_ex(_ptr(x), _ptr(w_router), _ptr(logit_bias), _ptr(w1), _ptr(b1), _ptr(w2),
                                 _ptr(b2), S, _ptr(w1s), _ptr(b1s), _ptr(w2s), _ptr(b2s), reroute_rounds, T, d, ff,
                                 E, k, capacity, dtype, _ptr(out), _ptr(stats), _ptr(topk_idx_out),
                                 _ptr(topk_gate_out), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_forward_ex")


def moe_dispatch_reroute_workspace_size(T, k, F, E) -> int:
    return load().moe_dispatch_reroute_workspace_size(T, k, F, E)


def moe_dispatch_reroute(ranked_idx, ranked_gate, T, k, F, E, capacity, counts, offsets, perm, slot_of, drop_mask,
                         row_gate, x, xp, d, dtype, ws, ws_bytes, stream=None):
    _check(load().moe_dispatch_reroute(_ptr(ranked_idx), _ptr(ranked_gate), T, k, F, E, capacity, _ptr(counts),
                                       _ptr(offsets), _ptr(perm), _ptr(slot_of), _ptr(drop_mask), _ptr(row_gate),
                                       _ptr(x), _ptr(xp), d, dtype, _ptr(ws), ws_bytes, _stream(stream)),
           "moe_dispatch_reroute")


def moe_shared_ffn(x, T, d, ff, S, w1s, b1s, w2s, b2s, h, ys, dtype, stream=None):
    _check(load().moe_shared_ffn(_ptr(x), T, d, ff, S, _ptr(w1s), _ptr(b1s), _ptr(w2s), _ptr(b2s), _ptr(h),
                                 _ptr(ys), dtype, _stream(stream)),
           "moe_shared_ffn")


def moe_combine_shared(yp, slot_of, topk_gate, ys, S, T, k, d, dtype, out, stream=None):
    _check(load().moe_combine_shared(_ptr(yp), _ptr(slot_of), _ptr(topk_gate), _ptr(ys), S, T, k, d, dtype,
                                     _ptr(out), _stream(stream)),
           "moe_combine_shared")


def moe_get_error(stream=None) -> int:
    return load().moe_get_error(_stream(stream))


def moe_debug_gelu(x, y, n, variant, stream=None):
    _check(load().moe_debug_gelu(_ptr(x), _ptr(y), n, variant, _stream(stream)), "moe_debug_gelu")


def moe_launch_count() -> int:
    return int(load().moe_launch_count())


def moe_trace_enable(enable: bool) -> bool:
    """Turn the library's NVTX ranges on or off; returns the previous setting."""
    return bool(load().moe_trace_enable(1 if enable else 0))


def moe_trace_enabled() -> bool:
    return bool(load().moe_trace_enabled())


def moe_timing_enable(enable: bool):
    _check(load().moe_timing_enable(1 if enable else 0), "moe_timing_enable")


def _ptr_array(items):
    return (ctypes.c_void_p * max(1, len(items)))(*[_ptr(t) for t in items])


def moe_pipeline_create(w_router, logit_bias, w1, b1, w2, b2, S, w1s, b1s, w2s, b2s, reroute_rounds, T, d, ff, E,
                        k, capacity, dtype, x_dev, out_dev, ws, ws_bytes, flags=MOE_PIPELINE_GRAPHS) -> int:
    """Returns the pipeline handle (an integer); x_dev, out_dev and ws are
    equal-length lists of device tensors (one per lane)."""
    depth = len(x_dev)
    if len(out_dev) != depth or len(ws) != depth:
        raise ValueError("x_dev, out_dev and ws need one entry per lane")
    handle = ctypes.c_void_p()
    _check(load().moe_pipeline_create(_ptr(w_router), _ptr(logit_bias), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), S,
                                      _ptr(w1s), _ptr(b1s), _ptr(w2s), _ptr(b2s), reroute_rounds, T, d, ff, E, k,
                                      capacity, dtype, depth, _ptr_array(x_dev), _ptr_array(out_dev),
                                      _ptr_array(ws), ws_bytes, flags, ctypes.byref(handle)),
           "moe_pipeline_create")
    return handle.value


def moe_pipeline_run(handle: int, x_host, out_host) -> float:
    """Runs len(x_host) steps (host tensors in, host tensors out); returns the
    device time in milliseconds from before the first copy to after the last."""
    if len(x_host) != len(out_host):
        raise ValueError("one output buffer per input batch")
    ms = ctypes.c_float(0.0)
    _check(load().moe_pipeline_run(handle, _ptr_array(x_host), _ptr_array(out_host), len(x_host),
                                   ctypes.byref(ms)),
           "moe_pipeline_run")
    return ms.value


def moe_pipeline_destroy(handle: int):
    _check(load().moe_pipeline_destroy(handle), "moe_pipeline_destroy")


def moe_timing_read():
    """{kernel name: (total ms, launches)} since the last read."""
    ms = (ctypes.c_double * MOE_NUM_KERNELS)()
    n = (ctypes.c_int64 * MOE_NUM_KERNELS)()
    _check(load().moe_timing_read(ctypes.cast(ms, _P), ctypes.cast(n, _P)), "moe_timing_read")
    return {name: (ms[i], int(n[i])) for i, name in enumerate(KERNEL_NAMES)}


def moe_ffn_clock_enable(enable: bool):
    _check(load().moe_ffn_clock_enable(1 if enable else 0), "moe_ffn_clock_enable")


def moe_ffn_clock_read():
    """{"ffn1": (SM MHz, span us), "ffn2": (...)} of the most recent launches."""
    mhz = (ctypes.c_double * 2)()
    us = (ctypes.c_double * 2)()
    _check(load().moe_ffn_clock_read(ctypes.cast(mhz, _P), ctypes.cast(us, _P)), "moe_ffn_clock_read")
    return {"ffn1": (mhz[0], us[0]), "ffn2": (mhz[1], us[1])}


def moe_debug_wait_timeout(limit_ns: int, stream=None):
    """One bounded wait that runs out; the device error word then holds MOE_ERR_TIMEOUT."""
    _check(load().moe_debug_wait_timeout(int(limit_ns), _stream(stream)), "moe_debug_wait_timeout")
