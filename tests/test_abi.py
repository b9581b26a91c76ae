"""The C ABI without a GPU: the library loads, exports every entry point include/moe.h declares,
sizes workspaces, and rejects bad arguments synchronously (before any CUDA call)."""
import ctypes as C
import dataclasses
import os
import re

import pytest

import mixture_experts_ffn_norm_b200 as moe
from mixture_experts_ffn_norm_b200 import build as moe_build
import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    moe_build.build()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 7
    lib = C.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(moe.EXPORTS) == set(names)


def test_workspace_sizes_and_invalid_configs():
    for s in synthetic.CONFIGS.values():
        cfg = moe.Config.from_shape(s)
        assert moe.workspace_bytes(cfg) > 0
        assert moe.launches_per_forward(cfg) == (3 if s.E == 0 else 11)   # a dense block: norm + 2 GEMMs
    c4 = moe.Config.from_shape(synthetic.CONFIGS["C4"])
    assert moe.workspace_bytes(c4) < 8 * 2 ** 30
    # bf16 activations with FP8 weights: the permuted rows and h are 2 bytes wide, no activation scales
    c4_a16 = dataclasses.replace(c4, amode=moe.MOE_ACT_BF16)
    assert moe.workspace_bytes(c4) < moe.workspace_bytes(c4_a16) < 2 * moe.workspace_bytes(c4)
    bad = [dict(dim=200), dict(inter_dim=100), dict(top_k=0), dict(top_k=300), dict(n_experts=300),
           dict(n_experts=12), dict(num_tokens=0), dict(shared_inter=64), dict(wtype=7),
           dict(n_experts=0), dict(n_experts=0, top_k=0, shared_inter=0)]   # dense: k = 0 and an MLP
    for b in bad:
        kw = dict(num_tokens=64, dim=256, inter_dim=128, n_experts=8, top_k=2, shared_inter=128,
                  wtype=moe.MOE_W_BF16, amode=moe.MOE_ACT_BF16)
        kw.update(b)
        assert moe.workspace_bytes(moe.Config(**kw)) == 0, b


def test_forward_rejects_bad_arguments_without_touching_the_device():
    L = moe.lib()
    cfg = moe.Config.from_shape(synthetic.CONFIGS["C1"]).c()
    fake = 1 << 20                              # aligned, never dereferenced on these paths
    w = moe.moe_weights_t(fake, fake, fake, None, None, None, fake, fake, fake, None, None, None)
    need = L.moe_workspace_bytes(C.byref(cfg))
    args = lambda **o: [C.byref(o.get("cfg", cfg)), o.get("x", fake), o.get("r", fake), fake, fake, None,
                        C.byref(o.get("w", w)), o.get("out", fake + 4096), o.get("ro", fake + 8192),
                        o.get("ws", fake), o.get("wsb", need), None]
    assert L.moe_forward(*args(x=None)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward(*args(x=fake + 2)) == moe.MOE_ERR_INVALID_ARG          # misaligned
    assert L.moe_forward(*args(ro=None)) == moe.MOE_ERR_INVALID_ARG             # residual without output
    assert L.moe_forward(*args(wsb=need - 1)) == moe.MOE_ERR_WORKSPACE
    assert L.moe_forward(*args(ws=None)) == moe.MOE_ERR_WORKSPACE
    assert L.moe_forward(*args(out=fake)) == moe.MOE_ERR_INVALID_ARG            # out aliases x
    bad = moe.Config(64, 256, 128, 8, 9, 128, moe.MOE_W_BF16, moe.MOE_ACT_BF16).c()
    assert L.moe_forward(*args(cfg=bad)) == moe.MOE_ERR_INVALID_ARG
    # FP8 weights need their block scales, in either activation mode
    for amode in (moe.MOE_ACT_FP8_1x128, moe.MOE_ACT_BF16):
        fp8 = moe.Config(64, 256, 128, 8, 2, 128, moe.MOE_W_FP8_E4M3_B128, amode).c()
        assert L.moe_forward(*args(cfg=fp8, wsb=L.moe_workspace_bytes(C.byref(fp8)))) == moe.MOE_ERR_INVALID_ARG
    # bf16 weights with FP8 activations is not a mode
    bf16_a8 = moe.Config(64, 256, 128, 8, 2, 128, moe.MOE_W_BF16, moe.MOE_ACT_FP8_1x128).c()
    assert L.moe_forward(*args(cfg=bf16_a8)) == moe.MOE_ERR_INVALID_ARG
    # the fused next-norm entry point: needs next_xn, a residual and the next gain; not for dense blocks
    nn = lambda cfg=cfg, r=fake, g=fake + 12288, xn=fake + 16384: L.moe_forward_next_norm(
        C.byref(cfg), fake, r, fake, fake, None, C.byref(w), g, None, xn, fake + 8192, fake, need, None)
    assert nn(xn=None) == moe.MOE_ERR_INVALID_ARG
    assert nn(r=None) == moe.MOE_ERR_INVALID_ARG
    assert nn(g=None) == moe.MOE_ERR_INVALID_ARG
    assert nn(xn=fake) == moe.MOE_ERR_INVALID_ARG                                # aliases x
    dense = moe.Config(64, 256, 128, 0, 0, 256, moe.MOE_W_BF16, moe.MOE_ACT_BF16).c()
    assert nn(cfg=dense) == moe.MOE_ERR_UNSUPPORTED
    assert moe.status_string(moe.MOE_ERR_WORKSPACE) == "workspace missing or too small"


def test_expert_slice_and_round_reject_bad_arguments_without_touching_the_device():
    L = moe.lib()
    cfg = moe.Config.from_shape(synthetic.CONFIGS["C1"]).c()
    fake = 1 << 20
    w = moe.moe_weights_t(fake, fake, fake, None, None, None, fake, fake, fake, None, None, None)
    need = L.moe_workspace_bytes(C.byref(cfg))
    sl = lambda cfg=cfg, b=0, e=4, y=fake + 65536: L.moe_forward_expert_slice(
        C.byref(cfg), fake, fake, fake, fake, None, C.byref(w), b, e, 1, y, fake + 8192, fake, need, None)
    assert sl(y=None) == moe.MOE_ERR_INVALID_ARG
    assert sl(b=5, e=4) == moe.MOE_ERR_INVALID_ARG            # empty range reversed
    assert sl(e=9) == moe.MOE_ERR_INVALID_ARG                  # beyond E = 8
    assert sl(y=fake) == moe.MOE_ERR_INVALID_ARG               # aliases x
    dense = moe.Config(64, 256, 128, 0, 0, 256, moe.MOE_W_BF16, moe.MOE_ACT_BF16).c()
    assert sl(cfg=dense) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_round_bf16(fake, fake + 4096, 6, None) == moe.MOE_ERR_INVALID_ARG   # not a multiple of 4
    assert L.moe_round_bf16(None, fake, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_round_bf16(fake, fake, 0, None) == moe.MOE_OK
