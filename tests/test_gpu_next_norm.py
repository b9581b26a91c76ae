"""The MoE update with the next block's attn_norm fused into the combine (moe_forward_next_norm).

"MoE update" page, Block excerpt: after `x = self.ffn(x)` the next block starts with
`x, residual = self.attn_norm(x, residual)` -- the residual addition happens inside that
normalisation.  Checked against the oracle's RMSNorm applied to this library's own update and new
residual (bit-exact: the same exact mean of squares, IEEE sqrt and divide), against the plain
forward (the update is the same bits), and end to end against the oracle's layer followed by the
oracle's norm (within the layer's output bound carried through the norm's per-token scaling).
"""
import dataclasses
import json

import numpy as np
import pytest
import torch

import mixture_experts_ffn_norm_b200 as moe
import oracle
import synthetic
from harness import bits_np, inputs_for, sample_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _shape(**kw):
    base = dict(name="nn", T=300, d=1024, I=1024, E=16, k=4, n_shared=1, shared_inter=1024, wtype="fp8", seed=51)
    base.update(kw)
    return synthetic.MoEShape(**base)


@pytest.mark.parametrize("shape", [_shape(), _shape(wtype="bf16", T=200, I=1152), synthetic.CONFIGS["C3"]],
                         ids=["fp8", "bf16", "C3"])
def test_next_norm_fused(shape):
    inp = inputs_for(shape)
    cfg = moe.Config.from_shape(shape)
    layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
    g_next = (1.0 + synthetic.normal(shape.seed, "next_norm_w", (shape.d,), 0.1, device="cuda").float()).contiguous()
    x, r = inp["x"], inp["residual"]
    t = layer.t
    # the plain forward: the update and the new residual
    out0, ro0 = torch.empty_like(x), torch.empty_like(x)
    layer.forward(x, r, out0, ro0)
    # fused, with the update stored
    out1, xn1, nr1 = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    moe.moe_forward_next_norm(cfg, x, r, t["norm_w"], t["gate_w"], t.get("gate_bias"), layer.wstruct, g_next, out1,
                              xn1, nr1, layer.workspace)
    # fused, update not stored, next residual written over the residual input
    r2, xn2 = r.clone(), torch.empty_like(x)
    moe.moe_forward_next_norm(cfg, x, r2, t["norm_w"], t["gate_w"], t.get("gate_bias"), layer.wstruct, g_next, None,
                              xn2, r2, layer.workspace)
    assert moe.moe_get_status(layer.workspace) == moe.MOE_OK
    torch.cuda.synchronize()
    o0, q0, o1, x1, n1, x2, n2 = (bits_np(v) for v in (out0, ro0, out1, xn1, nr1, xn2, r2))
    assert np.array_equal(o1, o0), "the fused call's update differs from moe_forward's"
    assert np.array_equal(x2, x1) and np.array_equal(n2, n1)
    toks = np.arange(shape.T) if shape.T <= 300 else np.unique(np.r_[np.arange(0, shape.T, 7), shape.T - 1])
    gn = g_next.cpu().numpy()
    for tk in toks:   # the oracle's RMSNorm of this library's update and residual: bit for bit
        xn_o, ro_o, _, _ = oracle.norm_token(o0[tk], q0[tk], gn, shape.eps)
        assert np.array_equal(x1[tk], xn_o), f"next xn differs for token {tk}"
        assert np.array_equal(n1[tk], ro_o), f"next residual differs for token {tk}"
    # end to end: the oracle's layer, then the oracle's norm.  The update carries the layer's bound
    # |d delta| <= 2e-2 * RMS(delta); the norm rescales token t by g / rms_t(s), so element i of
    # next_xn may move by 2e-2 * RMS(delta) * g_i / rms_t(s) plus one bf16 step, and the next
    # residual by the update's bound plus one bf16 step.
    o = oracle.Oracle(shape, inp)
    sample = toks if shape.T <= 300 else toks[:24]
    ref = o.forward(sample.astype(np.int32))
    f64 = oracle.bf16_bits_to_f64
    dbound = 2e-2 * float(np.sqrt(np.mean(f64(ref["out"]) ** 2)))
    worst_x = worst_r = 0.0
    for i, tk in enumerate(sample):
        xn_o, ro_o, _, _ = oracle.norm_token(ref["out"][i], ref["residual_out"][i], gn, shape.eps)
        s_o = f64(ro_o)
        rms_t = float(np.sqrt(np.mean(s_o ** 2)))
        ulp = lambda v: 2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126))) - 7)
        tol_x = dbound * gn.astype(np.float64) / rms_t + ulp(f64(xn_o))
        tol_r = dbound + ulp(s_o)
        worst_x = max(worst_x, float((np.abs(f64(x1[tk]) - f64(xn_o)) / tol_x).max()))
        worst_r = max(worst_r, float((np.abs(f64(n1[tk]) - s_o) / tol_r).max()))
    print(shape.name, json.dumps({"next_xn_err_over_bound": worst_x, "next_residual_err_over_bound": worst_r}))
    assert worst_x <= 1.0 and worst_r <= 1.0
