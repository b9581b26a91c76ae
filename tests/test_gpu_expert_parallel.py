"""The expert-parallel layer ("MoE update" page, MoE.forward excerpt: each rank runs its own range of
experts into a float32 y, `dist.all_reduce(y)` sums the ranks) as two ranks on one GPU.

Each rank is a process with its own CUDA context running moe_forward_expert_slice on its half of
the experts (rank 0 also the shared expert); the partials are summed over gloo on host copies and
rounded once with moe_round_bf16.  Only the reduction crosses processes, and it runs on the host,
so no kernel waits on another process.  The result must equal the single-rank layer up to the
float32 summation order (at most one bf16 step per element) and the oracle within the layer bound.
"""
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import mixture_experts_ffn_norm_b200 as moe
import oracle
import synthetic
from harness import bits_np, check_out, inputs_for

pytestmark = pytest.mark.gpu

SHAPE = dict(name="ep", T=300, d=1024, I=1024, E=16, k=4, n_shared=1, shared_inter=1024, wtype="fp8", seed=71)


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        shape = synthetic.MoEShape(**SHAPE)
        inp = inputs_for(shape)
        cfg = moe.Config.from_shape(shape)
        layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
        out, ro = torch.empty_like(inp["x"]), torch.empty_like(inp["x"])
        moe.expert_parallel_forward(layer, inp["x"], inp["residual"], out, ro, rank, world)
        torch.cuda.synchronize()
        q.put((rank, moe.moe_get_status(layer.workspace), bits_np(out), bits_np(ro)))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def test_two_expert_ranks_sum_to_the_single_rank_layer():
    world, port = 2, _port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda g: g[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for _, st, _, _ in got:
        assert st == moe.MOE_OK
    (_, _, out0, ro0), (_, _, out1, ro1) = got
    assert np.array_equal(out0, out1) and np.array_equal(ro0, ro1)    # every rank holds the full output

    shape = synthetic.MoEShape(**SHAPE)
    inp = inputs_for(shape)
    cfg = moe.Config.from_shape(shape)
    layer = moe.MoELayer(cfg, {n: v for n, v in inp.items() if n not in ("x", "residual")})
    out, ro = torch.empty_like(inp["x"]), torch.empty_like(inp["x"])
    layer.forward(inp["x"], inp["residual"], out, ro)
    torch.cuda.synchronize()
    ref_out, ref_ro = bits_np(out), bits_np(ro)
    assert np.array_equal(ro0, ref_ro)
    a, b = oracle.bf16_bits_to_f64(out0), oracle.bf16_bits_to_f64(ref_out)
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    assert np.all(np.abs(a - b) <= step)                              # float32 order only
    assert np.mean(out0 == ref_out) > 0.99

    # against the oracle with the structural layers' bound (2e-2 * RMS, or one bf16 step of the
    # oracle's value for an element where both sides round an intermediate differently)
    ref = oracle.Oracle(shape, inp).forward()
    check_out(types.SimpleNamespace(out=out0), ref, np.arange(shape.T), {}, allow_ulp=True)
