"""moe_route_noalloc: the expert grouping step for callers that cannot allocate device memory
when they call in (for instance a serving runtime that reserved all device memory up front and
hands a layer only the tensors it reads and writes).  Its scratch is a static device array, so
this file checks it against moe_forward's own grouping on two calls in a row, each call after
the array holds the previous call's contents.  It sits in a file of its own that is collected
last, and passes alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_norm_b200 as moe
import synthetic
from harness import inputs_for

pytestmark = pytest.mark.gpu


def _existing_routing(shape, bias=None):
    """idx and counts as moe_forward computes them (the existing entry point)."""
    inp = inputs_for(shape)
    if bias is not None:
        inp["gate_bias"] = bias
    cfg = moe.Config.from_shape(shape)
    layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
    out = torch.empty(shape.T, shape.d, dtype=torch.bfloat16, device="cuda")
    ro = torch.empty_like(out)
    layer.forward(inp["x"], inp["residual"], out, ro)
    idx = torch.empty(shape.T, shape.k, dtype=torch.int32, device="cuda")
    counts = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    moe.moe_debug_routing(cfg, layer.workspace, idx=idx, counts=counts)
    assert moe.moe_get_status(layer.workspace) == moe.MOE_OK
    return idx, counts.cpu().numpy()


def _check(idx, counts_ref, E, got):
    counts, offsets, row_of, row_token = (t.cpu().numpy() for t in got)
    T, k = idx.shape
    ids = idx.cpu().numpy().ravel()
    # integer outputs: exact
    assert np.array_equal(counts, counts_ref)
    padded = (counts_ref + 127) // 128 * 128
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(padded)]))
    # every (token, slot) lands inside its expert's rows, in token order, each row used once
    ro = row_of.ravel()
    for e in range(E):
        sel = np.nonzero(ids == e)[0]
        assert np.array_equal(ro[sel], offsets[e] + np.arange(len(sel)))
    assert np.array_equal(np.sort(ro), np.sort(np.unique(ro)))
    used = np.zeros(len(row_token), bool)
    used[ro] = True
    assert np.array_equal(row_token[ro], np.arange(T * k) // k)
    assert np.all(row_token[~used] == -1)


def test_noalloc_grouping_matches_forward_on_two_calls_in_a_row():
    a = synthetic.MoEShape("na", T=700, d=1024, I=1024, E=64, k=6, n_shared=1, shared_inter=1024, wtype="fp8", seed=31)
    b = synthetic.MoEShape("nb", T=1500, d=1024, I=1024, E=64, k=6, n_shared=1, shared_inter=1024, wtype="fp8", seed=32)
    bias = torch.zeros(64, device="cuda")
    bias[:8] = 6.0                           # skewed: most slots go to 8 experts, several get none
    runs = [(a, *_existing_routing(a)), (b, *_existing_routing(b, bias))]
    for shape, idx, counts_ref in runs:
        R = moe.route_rows(shape.T, shape.k, shape.E)
        out = (torch.full((shape.E,), -7, dtype=torch.int32, device="cuda"),
               torch.full((shape.E + 1,), -7, dtype=torch.int32, device="cuda"),
               torch.full((shape.T, shape.k), -7, dtype=torch.int32, device="cuda"),
               torch.full((R,), -7, dtype=torch.int32, device="cuda"))
        moe.moe_route_noalloc(idx, shape.E, *out)
        torch.cuda.synchronize()
        _check(idx, counts_ref, shape.E, out)
    assert (runs[1][2] == 0).any()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    idx = torch.zeros(262145, 1, dtype=torch.int32, device="cuda")
    z = torch.zeros(8, dtype=torch.int32, device="cuda")
    assert moe.moe_route_noalloc(idx, 4, z, z, z, z, check=False) == moe.MOE_ERR_UNSUPPORTED
