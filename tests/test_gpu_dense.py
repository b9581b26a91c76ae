"""Parity of the dense block (n_experts = 0) with the oracle.

"MoE update" page, Block excerpt: the first n_dense_layers blocks apply MLP(dim, inter_dim) instead
of the MoE, and the very first block's norm sees no residual.  Through the same boundary: E = 0,
k = 0, the MLP held as the shared SwiGLU; the library runs ffn_norm and the two SwiGLU GEMMs over
all tokens (no router, no routing) and the second GEMM writes the output rows directly.
Bounds as for the MoE layers: residual_out and xn bit-exact, out within 2e-2 * RMS.
"""
import dataclasses
import json

import numpy as np
import pytest
import torch

import mixture_experts_ffn_norm_b200 as moe
import oracle
import synthetic
from harness import bits_np, check_out, inputs_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


class DenseRun:
    """One dense-block forward through the C ABI; out, residual_out, xn copied to the host."""

    def __init__(self, shape, inp, residual=True, amode=None):
        self.cfg = moe.Config.from_shape(shape)
        if amode is not None:
            self.cfg = dataclasses.replace(self.cfg, amode=amode)
        assert moe.launches_per_forward(self.cfg) == 3
        layer = moe.MoELayer(self.cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
        x = inp["x"]
        r = inp["residual"] if residual else None
        out = torch.empty_like(x)
        ro = torch.empty_like(x) if residual else None
        layer.forward(x, r, out, ro)
        st = moe.moe_get_status(layer.workspace)
        assert st == moe.MOE_OK, moe.status_string(st)
        xn = torch.empty_like(x)
        moe.moe_debug_norm(self.cfg, layer.workspace, xn)
        with pytest.raises(moe.MoeError):          # a dense block has no routing to export
            moe.moe_debug_routing(self.cfg, layer.workspace, counts=torch.empty(1, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        self.out, self.xn = bits_np(out), bits_np(xn)
        self.residual_out = bits_np(ro) if residual else None


def _dense(**kw):
    base = dict(name="dense", T=300, d=1024, I=128, E=0, k=0, n_shared=1, shared_inter=1152, wtype="fp8", seed=41)
    base.update(kw)
    return synthetic.MoEShape(**base)


@pytest.mark.parametrize("wtype,act,residual", [("fp8", "fp8", True), ("fp8", "bf16", True), ("bf16", "bf16", True),
                                                ("fp8", "fp8", False)])
def test_dense_block_every_token(wtype, act, residual):
    shape = _dense(wtype=wtype)
    inp = inputs_for(shape)
    run = DenseRun(shape, inp, residual=residual, amode=moe.MOE_ACT_BF16 if act == "bf16" else None)
    o = oracle.Oracle(shape, dict(inp, residual=inp["residual"] if residual else None),
                      act_fp8=(wtype == "fp8" and act == "fp8"))
    ref = o.forward()
    toks = np.arange(shape.T, dtype=np.int32)
    if residual:
        assert np.array_equal(run.residual_out, ref["residual_out"])
    assert np.array_equal(run.xn, ref["xn"])
    report = {}
    check_out(run, ref, toks, report, allow_ulp=True)
    print("dense", wtype, act, residual, json.dumps(report))


def test_dense_workload_full_size_sampled():
    """The dense workload (T=16384, d=7168, MLP 18432, FP8) exactly as bench.py runs it, compared on
    a seeded token sample that includes the last token."""
    shape = synthetic.CONFIGS["D1"]
    inp = inputs_for(shape)
    run = DenseRun(shape, inp)
    o = oracle.Oracle(shape, inp)
    rng = np.random.default_rng(shape.seed)
    toks = np.unique(np.concatenate([rng.choice(shape.T, 40, replace=False), [0, shape.T - 1]])).astype(np.int32)
    ref = o.forward(toks)
    assert np.array_equal(run.residual_out[toks], ref["residual_out"])
    assert np.array_equal(run.xn[toks], ref["xn"])
    report = {}
    check_out(run, ref, toks, report)
    print("D1", json.dumps(report))
