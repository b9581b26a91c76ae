"""moe_forward captured into a CUDA graph and replayed.

The forward enqueues only kernels and memsets on the caller's stream -- no host synchronisation, no
allocation, every routing-dependent size read on the device -- so a serving loop can capture it
once and replay it, paying one graph launch instead of eleven kernel launches.  Replays must give
the same bits as eager calls, also after new input values are written into the captured buffers.
"""
import pytest
import torch

import mixture_experts_ffn_norm_b200 as moe
import synthetic
from harness import inputs_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("name", ["C1", "C3", "D1-small"])
def test_forward_replays_from_a_cuda_graph(name):
    if name == "D1-small":
        shape = synthetic.MoEShape("D1-small", T=256, d=1024, I=128, E=0, k=0, n_shared=1, shared_inter=1152,
                                   wtype="fp8", seed=61)
    else:
        shape = synthetic.CONFIGS[name]
    inp = inputs_for(shape)
    cfg = moe.Config.from_shape(shape)
    layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
    x, r = inp["x"].clone(), inp["residual"].clone()
    out_e, ro_e = torch.empty_like(x), torch.empty_like(x)
    layer.forward(x, r, out_e, ro_e)              # eager (also the first call on this device)
    torch.cuda.synchronize()

    out_g, ro_g = torch.empty_like(x), torch.empty_like(x)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        layer.forward(x, r, out_g, ro_g)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_status(layer.workspace) == moe.MOE_OK
    assert torch.equal(out_g, out_e) and torch.equal(ro_g, ro_e)

    # new inputs in the captured buffers: the replay follows them (routing is re-derived on the device)
    x2 = synthetic.normal(shape.seed + 100, "x", tuple(x.shape), 1.0, device="cuda")
    x.copy_(x2)
    graph.replay()
    out_2, ro_2 = torch.empty_like(x), torch.empty_like(x)
    layer.forward(x2, r, out_2, ro_2)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_2) and torch.equal(ro_g, ro_2)
    assert not torch.equal(out_2, out_e)
    del graph
