"""layer.py's host helpers on CPU: dtype codes, uploads, parameter bundles,
the statistics record's byte layout, and the refusal of CPU tensors."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import workloads as wl
from mixture_experts_layer_45_b200.layer import MoELayer, MoEParams, dtype_code, read_stats, to_device


def test_dtype_codes():
    assert dtype_code("bf16") == dtype_code(torch.bfloat16) == _lib.MOE_BF16
    assert dtype_code("f32") == dtype_code(torch.float32) == _lib.MOE_F32
    with pytest.raises(ValueError):
        dtype_code("fp8")


def test_upload_keeps_bf16_values_exactly():
    w = wl.workload("switch-top1", dtype="bf16")
    x = wl.draw_inputs(w, T=64)["x"]
    t = to_device(x, _lib.MOE_BF16, "cpu")
    assert t.dtype == torch.bfloat16
    np.testing.assert_array_equal(t.float().numpy(), x)          # the draws are bf16-representable
    np.testing.assert_array_equal(t.view(torch.int16).numpy().view(np.uint16), wl.bf16_bits(x))


def test_params_bundle_shapes():
    inp = wl.draw_custom(3, T=16, d=32, ff=64, E=4, dtype="f32", shared=2)
    p = MoEParams.from_arrays(inp, _lib.MOE_F32, "cpu")
    assert (p.E, p.ff, p.d, p.S) == (4, 64, 32, 2)
    assert p.logit_bias is None
    q = MoEParams.from_arrays(wl.draw_custom(3, T=16, d=32, ff=64, E=4, dtype="f32"), _lib.MOE_F32, "cpu")
    assert q.S == 0 and q.shared_w1 is None


def test_stats_record_layout():
    rec = _lib.MoeStats(aux_loss=1.5, imbalance=2.0, drop_rate=0.25, rows_kept=7, max_count=3, dropped=1,
                        rerouted=2)
    raw = torch.frombuffer(bytearray(ctypes.string_at(ctypes.addressof(rec), ctypes.sizeof(rec))),
                           dtype=torch.uint8)
    st = read_stats(raw)
    assert st == {"aux_loss": 1.5, "imbalance": 2.0, "drop_rate": 0.25, "rows_kept": 7, "max_count": 3,
                  "dropped": 1, "rerouted": 2}
    assert ctypes.sizeof(_lib.MoeStats) == 28


def test_forward_refuses_host_tensors():
    inp = wl.draw_custom(3, T=16, d=32, ff=64, E=4, dtype="f32")
    layer = MoELayer(MoEParams.from_arrays(inp, _lib.MOE_F32, "cpu"), k=2)
    with pytest.raises(ValueError):
        layer.forward(torch.zeros(16, 32))
