"""End-to-end pipeline and CUDA-graph replay of the layer on the GPU.

The pipelined host path (the library's moe_pipeline_*: pinned host
buffers, three streams, one CUDA graph per lane, a native host loop) must
return exactly what the device forward returns, with and without graphs,
for any number of steps and lanes; and a captured forward, replayed on new
inputs, must equal the eager call bit for bit.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import workloads as wl
from mixture_experts_layer_45_b200.layer import HostPipeline, MoELayer, MoEParams, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "these tests need a CUDA GPU"
    _lib.load()
    yield
    torch.cuda.synchronize()


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def scaled_inputs(x, n):
    """n different bf16 token batches derived from x."""
    return [(x.float() * (0.5 + 0.25 * i)).to(x.dtype) for i in range(n)]


@pytest.mark.parametrize("shared,reroute,depth,graphs", [(0, 0, 3, True), (1, 1, 3, True), (0, 0, 2, False),
                                                         (0, 1, 1, True)])
def test_host_pipeline_matches_device_forward(shared, reroute, depth, graphs):
    w = wl.workload("switch-top1", dtype="bf16", cf=1.0, shared=shared)
    inp = wl.draw_inputs(w)
    params = MoEParams.from_arrays(inp, _lib.MOE_BF16, DEV)
    layer = MoELayer(params, w.k, _lib.moe_capacity(w.T, w.k, w.E, w.cf), reroute=reroute)
    x = to_device(inp["x"], _lib.MOE_BF16, DEV)
    xs = scaled_inputs(x, 5)
    x_hosts = [xi.cpu().pin_memory() for xi in xs]
    out_hosts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for _ in xs]
    pipe = HostPipeline(layer, w.T, depth=depth, graphs=graphs)
    ms = pipe.run(x_hosts, out_hosts)
    assert ms > 0.0
    assert _lib.moe_get_error() == _lib.MOE_OK
    for xi, oh in zip(xs, out_hosts):
        ref = layer.forward(xi).cpu()
        assert torch.equal(bits(oh), bits(ref))
    # a second run on the same pipeline, buffers repeated across steps, pageable output
    outs2 = [torch.empty(x.shape, dtype=x.dtype) for _ in range(2)]
    pipe.run([x_hosts[4], x_hosts[0], x_hosts[4]], [outs2[0], outs2[1], outs2[0]])
    assert torch.equal(bits(outs2[0]), bits(out_hosts[4])) and torch.equal(bits(outs2[1]), bits(out_hosts[0]))
    assert pipe.run([], []) >= 0.0
    pipe.close()


def test_host_pipeline_f32_and_ragged_tokens():
    T, d, ff, E, k = 1000, 72, 200, 5, 2
    inp = wl.draw_custom(4, T=T, d=d, ff=ff, E=E, dtype="f32", router_std=0.5, shared=1)
    params = MoEParams.from_arrays(inp, _lib.MOE_F32, DEV)
    layer = MoELayer(params, k, 300, reroute=1)
    x = to_device(inp["x"], _lib.MOE_F32, DEV)
    xs = scaled_inputs(x, 4)
    x_hosts = [xi.cpu().pin_memory() for xi in xs]
    out_hosts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for _ in xs]
    pipe = HostPipeline(layer, T, depth=3)
    pipe.run(x_hosts, out_hosts)
    assert _lib.moe_get_error() == _lib.MOE_OK
    for xi, oh in zip(xs, out_hosts):
        assert torch.equal(oh, layer.forward(xi).cpu())
    pipe.close()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_graph_replay_equals_eager(dtype):
    T, d, ff, E, k, cap = 1500, 128, 512, 8, 2, 300
    inp = wl.draw_custom(21, T=T, d=d, ff=ff, E=E, dtype=dtype, router_std=0.5, shared=1)
    dt = _lib.MOE_BF16 if dtype == "bf16" else _lib.MOE_F32
    params = MoEParams.from_arrays(inp, dt, DEV)
    eager = MoELayer(params, k, cap, reroute=1)
    captured = MoELayer(params, k, cap, reroute=1)
    x0 = to_device(inp["x"], dt, DEV)
    x_in = x0.clone()
    out = torch.empty_like(x0)
    captured.forward(x_in, out=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        captured.forward(x_in, out=out)
    for xi in scaled_inputs(x0, 3):
        x_in.copy_(xi)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(bits(out), bits(eager.forward(xi)))
    assert _lib.moe_get_error() == _lib.MOE_OK
