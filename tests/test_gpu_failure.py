"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out records MOE_ERR_TIMEOUT in the device error word, the host reads
it, and the context stays usable for the next forward pass."""
import numpy as np
import pytest
import torch

import parity_util as pu
from mixture_experts_layer_45_b200 import _lib
from mixture_experts_layer_45_b200 import workloads as wl
from mixture_experts_layer_45_b200.layer import MoELayer, MoEParams, to_device
from oracle import moe_ref

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_wait_timeout_is_reported_and_context_survives():
    assert torch.cuda.is_available()
    assert _lib.moe_get_error() == _lib.MOE_OK
    _lib.moe_debug_wait_timeout(10_000_000)          # 10 ms on a barrier nothing completes
    assert _lib.moe_get_error() == _lib.MOE_ERR_TIMEOUT
    assert _lib.moe_get_error() == _lib.MOE_OK       # reading clears the word
    # the next forward pass runs and is correct
    inp = wl.draw_custom(31, T=700, d=64, ff=128, E=8, dtype="bf16", router_std=0.5)
    layer = MoELayer(MoEParams.from_arrays(inp, _lib.MOE_BF16, DEV), 2, -1)
    x = to_device(inp["x"], _lib.MOE_BF16, DEV)
    idx = torch.empty((700, 2), dtype=torch.int32, device=DEV)
    out = layer.forward(x, topk_idx=idx).float().cpu().numpy()
    assert _lib.moe_get_error() == _lib.MOE_OK
    idx_np = idx.cpu().numpy()
    r = moe_ref.route(inp["x"], inp["w_router"], 2)
    gates = np.take_along_axis(r["gates"], idx_np.astype(np.int64), 1)
    ref = moe_ref.moe_forward(inp["x"], inp, idx_np, gates, moe_ref.dispatch(idx_np, 8, -1)["slot_of"])
    assert pu.max_rel_err(out, ref) <= pu.TOL["bf16"]
