"""User-facing wrapper around ``moe_forward``: device parameters, a cached
workspace, and an end-to-end call from pinned host memory.

PyTorch provides device memory and streams only; the layer's arithmetic runs
in libmoe's CUDA kernels.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import _lib

TORCH_DTYPE = {_lib.MOE_F32: torch.float32, _lib.MOE_BF16: torch.bfloat16}


def dtype_code(name_or_torch) -> int:
    if name_or_torch in ("f32", torch.float32):
        return _lib.MOE_F32
    if name_or_torch in ("bf16", torch.bfloat16):
        return _lib.MOE_BF16
    raise ValueError(f"unsupported dtype {name_or_torch!r}")


def to_device(a: np.ndarray, dtype: int, device) -> torch.Tensor:
    """Upload a float32 array (already bf16-representable for bf16) in `dtype`."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device=device, dtype=TORCH_DTYPE[dtype])


@dataclass
class MoEParams:
    w_router: torch.Tensor
    logit_bias: Optional[torch.Tensor]
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor
    dtype: int
    # shared always-on experts [S, ...] (None: no shared experts)
    shared_w1: Optional[torch.Tensor] = None
    shared_b1: Optional[torch.Tensor] = None
    shared_w2: Optional[torch.Tensor] = None
    shared_b2: Optional[torch.Tensor] = None

    @property
    def S(self):
        return 0 if self.shared_w1 is None else self.shared_w1.shape[0]

    @property
    def E(self):
        return self.w1.shape[0]

    @property
    def ff(self):
        return self.w1.shape[1]

    @property
    def d(self):
        return self.w1.shape[2]

    @classmethod
    def from_arrays(cls, inputs: Dict[str, np.ndarray], dtype: int, device="cuda") -> "MoEParams":
        bias = inputs.get("logit_bias")
        shared = {}
        if inputs.get("shared_w1") is not None:
            shared = {key: to_device(inputs[key], dtype, device)
                      for key in ("shared_w1", "shared_b1", "shared_w2", "shared_b2")}
        return cls(
            w_router=to_device(inputs["w_router"], dtype, device),
            logit_bias=None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).to(device),
            w1=to_device(inputs["w1"], dtype, device), b1=to_device(inputs["b1"], dtype, device),
            w2=to_device(inputs["w2"], dtype, device), b2=to_device(inputs["b2"], dtype, device),
            dtype=dtype, **shared)


def read_stats(stats_buf: torch.Tensor) -> Dict[str, float]:
    raw = stats_buf.cpu().numpy().tobytes()
    s = _lib.MoeStats.from_buffer_copy(raw)
    return {f: getattr(s, f) for f, _ in _lib.MoeStats._fields_}


class MoELayer:
    """One MoE layer bound to device parameters (routed experts and, if the
    parameters have them, shared always-on experts); reuses its workspace.
    ``reroute`` > 0 gives assignments dropped at capacity that many rounds
    of fallback experts (moe_forward_ex)."""

    def __init__(self, params: MoEParams, k: int, capacity: int = -1, reroute: int = 0):
        self.p = params
        self.k = k
        self.capacity = capacity
        self.reroute = reroute
        self._ws = None
        self._ws_T = -1
        self.stats_buf = torch.zeros(ctypes.sizeof(_lib.MoeStats), dtype=torch.uint8,
                                     device=params.w1.device)

    def workspace(self, T: int) -> torch.Tensor:
        if self._ws is None or self._ws_T < T:
            n = _lib.moe_forward_ex_workspace_size(T, self.p.d, self.p.ff, self.p.E, self.k, self.p.S,
                                                   self.reroute, self.p.dtype)
            if n == 0:
                raise ValueError("invalid layer sizes")
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.p.w1.device)
            self._ws_T = T
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stats: bool = False,
                topk_idx: Optional[torch.Tensor] = None, topk_gate: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        if not x.is_cuda:
            raise ValueError("x must be a CUDA tensor")
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        ws = self.workspace(T)
        p = self.p
        if p.S == 0 and self.reroute == 0:
            _lib.moe_forward(x, p.w_router, p.logit_bias, p.w1, p.b1, p.w2, p.b2, T, p.d, p.ff, p.E, self.k,
                             self.capacity, p.dtype, out, self.stats_buf if stats else None, topk_idx, topk_gate,
                             ws, ws.numel(), stream)
        else:
            _lib.moe_forward_ex(x, p.w_router, p.logit_bias, p.w1, p.b1, p.w2, p.b2, p.S, p.shared_w1,
                                p.shared_b1, p.shared_w2, p.shared_b2, self.reroute, T, p.d, p.ff, p.E, self.k,
                                self.capacity, p.dtype, out, self.stats_buf if stats else None, topk_idx,
                                topk_gate, ws, ws.numel(), stream)
        return out

    __call__ = forward

    def workspace_view(self, T: int, which: str, dtype, count: int) -> torch.Tensor:
        """A view of one of moe_forward's intermediate arrays in the workspace
        (valid after a forward call on T tokens; for inspection and tests)."""
        off = _lib.moe_forward_ex_workspace_offset(T, self.p.d, self.p.ff, self.p.E, self.k, self.p.S,
                                                   self.reroute, self.p.dtype, which)
        ws = self.workspace(T)
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype)

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, x_dev: torch.Tensor,
                     out_dev: torch.Tensor, stream=None) -> torch.Tensor:
        """End to end from (pinned) host memory: H2D copy, forward, D2H copy,
        all enqueued on one stream; returns out_host once the copy is done."""
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            x_dev.copy_(x_host, non_blocking=True)
            self.forward(x_dev, out=out_dev, stream=s)
            out_host.copy_(out_dev, non_blocking=True)
        s.synchronize()
        return out_host


class HostPipeline:
    """End-to-end forward passes from pinned host memory, pipelined
    (libmoe's native pipeline, moe_pipeline_*).

    Each step copies its tokens host -> device, runs the layer and copies
    the output device -> host.  The copies run on their own streams and the
    layer on a third, with `depth` lanes (device input / output buffers and
    a workspace each), so the input copy of step i+1 and the output copy of
    step i-1 overlap the layer of step i (PCIe is full duplex).  Every
    step's copies are still issued and completed.  With `graphs` (default)
    each lane's layer call is captured once into a CUDA graph and replayed;
    the per-step host loop runs in the library.
    """

    def __init__(self, layer: MoELayer, T: int, depth: int = 3, graphs: bool = True):
        p = layer.p
        dev = p.w1.device
        dt = TORCH_DTYPE[p.dtype]
        self.layer = layer
        self.depth = depth
        self.T = T
        self.x_dev = [torch.empty((T, p.d), dtype=dt, device=dev) for _ in range(depth)]
        self.out_dev = [torch.empty((T, p.d), dtype=dt, device=dev) for _ in range(depth)]
        n = _lib.moe_forward_ex_workspace_size(T, p.d, p.ff, p.E, layer.k, p.S, layer.reroute, p.dtype)
        if n == 0:
            raise ValueError("invalid layer sizes")
        self.ws = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(depth)]
        self.handle = None
        with torch.cuda.device(dev):
            self.handle = _lib.moe_pipeline_create(
                p.w_router, p.logit_bias, p.w1, p.b1, p.w2, p.b2, p.S, p.shared_w1, p.shared_b1, p.shared_w2,
                p.shared_b2, layer.reroute, T, p.d, p.ff, p.E, layer.k, layer.capacity, p.dtype, self.x_dev,
                self.out_dev, self.ws, n, _lib.MOE_PIPELINE_GRAPHS if graphs else 0)

    def run(self, x_hosts, out_hosts) -> float:
        """x_hosts[i] (pinned) -> layer -> out_hosts[i] (pinned), for every i;
        returns the device milliseconds from the first copy in to the last
        copy out."""
        for xh, oh in zip(x_hosts, out_hosts):
            if xh.shape != (self.T, self.layer.p.d) or oh.shape != xh.shape or xh.dtype != self.x_dev[0].dtype \
                    or oh.dtype != xh.dtype or not (xh.is_contiguous() and oh.is_contiguous()) \
                    or xh.is_cuda or oh.is_cuda:
                raise ValueError("host batches must be contiguous CPU tensors of the pipeline's shape and dtype")
        return _lib.moe_pipeline_run(self.handle, list(x_hosts), list(out_hosts))

    def close(self):
        if self.handle is not None:
            _lib.moe_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
