"""The grouped FFN's in-kernel SM clock record (moe_ffn_clock_enable /
moe_ffn_clock_read): off by default, cleared when switched on, filled by
the fc1 and fc2 launches of a forward pass, and without effect on the
layer's output."""
import pytest
import torch

from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import workloads as wl
from mixture_experts_layer_45_b200.layer import MoELayer, MoEParams, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


# (T, E, k): about 225 rows per expert runs the single-CTA kernels; 2000
# rows per expert runs bf16 fc2 on CTA pairs
@pytest.mark.parametrize("dtype,T,E,k", [("bf16", 900, 8, 2), ("f32", 900, 8, 2), ("bf16", 8000, 4, 1)])
def test_ffn_clock_record(dtype, T, E, k):
    dt = _lib.MOE_BF16 if dtype == "bf16" else _lib.MOE_F32
    inp = wl.draw_custom(5, T=T, d=128, ff=256, E=E, dtype=dtype, router_std=0.5)
    layer = MoELayer(MoEParams.from_arrays(inp, dt, DEV), k, -1)
    x = to_device(inp["x"], dt, DEV)
    ref = layer.forward(x).clone()

    _lib.moe_ffn_clock_enable(True)
    try:
        rec = _lib.moe_ffn_clock_read()
        assert rec["ffn1"] == (0.0, 0.0) and rec["ffn2"] == (0.0, 0.0)   # cleared
        out = layer.forward(x)
        rec = _lib.moe_ffn_clock_read()
    finally:
        _lib.moe_ffn_clock_enable(False)
    assert _lib.moe_get_error() == _lib.MOE_OK
    for k in ("ffn1", "ffn2"):
        mhz, span_us = rec[k]
        assert 100.0 < mhz < 3000.0, (k, mhz)
        assert 0.0 < span_us < 1e6, (k, span_us)
    # recording changes nothing the layer computes
    assert torch.equal(out, ref)

    # switched off: a fresh record stays empty through a forward pass
    _lib.moe_ffn_clock_enable(True)
    _lib.moe_ffn_clock_enable(False)
    layer.forward(x)
    rec = _lib.moe_ffn_clock_read()
    assert rec["ffn1"] == (0.0, 0.0) and rec["ffn2"] == (0.0, 0.0)
