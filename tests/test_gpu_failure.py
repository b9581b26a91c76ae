"""Failure detection on the GPU without a fault: a wait that can never complete must give up,
latch MOE_ERR_DEVICE_TIMEOUT, and leave the context usable for the next forward pass."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_norm_b200 as moe
import synthetic
from harness import inputs_for

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    shape = synthetic.MoEShape("f", T=96, d=512, I=256, E=8, k=2, n_shared=1, shared_inter=256, wtype="fp8", seed=41)
    inp = inputs_for(shape)
    cfg = moe.Config.from_shape(shape)
    layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
    assert moe.moe_selftest_wait_timeout(layer.workspace, 1 << 20) == moe.MOE_OK
    assert moe.moe_get_status(layer.workspace) == moe.MOE_ERR_DEVICE_TIMEOUT
    # the context still works: a forward pass on the same workspace clears the status and is sane
    out = torch.empty(shape.T, shape.d, dtype=torch.bfloat16, device="cuda")
    ro = torch.empty_like(out)
    layer.forward(inp["x"], inp["residual"], out, ro)
    assert moe.moe_get_status(layer.workspace) == moe.MOE_OK
    assert torch.isfinite(out.float()).all()
    ref = (inp["x"].float() + inp["residual"].float()).to(torch.bfloat16)
    assert torch.equal(ro, ref)


def test_selftest_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert moe.moe_selftest_wait_timeout(ws, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_selftest_wait_timeout(ws[:64], 1000) == moe.MOE_ERR_WORKSPACE
