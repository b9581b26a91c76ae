"""Seeded synthetic inputs for the MoE FFN layer.

Both the CUDA path (through the tests and ``bench.py``) and the CPU oracle
take their inputs from here.  This module holds none of the layer's
arithmetic: it only draws numbers and stores them in the dtypes the layer
consumes.

Every value is a pure function of ``(seed, stream, index)``: a counter-based
generator (two rounds of the public-domain ``lowbias32`` integer hash by
C. Wellons) turns the element index into 24 uniform bits, so the same call
gives the same bits on the CPU and on a GPU.  Normals use the Box-Muller
transform in float64 and are rounded once to the stored dtype.  All integer
products stay below 2**63, so no step relies on overflow behaviour.

The five workloads (sizes, distributions, seeds) are the ones the layer is
measured on: a tiny layer, a mid-size bf16 layer, and the full
DeepSeek-V3.2 MoE shape (d=7168, moe_inter=2048, 256 routed experts, top-8,
one shared expert) at a decode batch, a prefill batch and under skewed
routing.  Shapes follow the "MoE transformer block" and "Gate projection"
pages: weights are stored [out, in]; FP8 weights carry one float32 scale per
128x128 block.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field, asdict
from typing import Optional

import torch

__all__ = ["MoEShape", "CONFIGS", "uniform24", "normal", "generate", "zipf_bias"]

_M32 = 0xFFFFFFFF
_C1 = 0x7FEB352D
_C2 = 0x846CA68B


@dataclass(frozen=True)
class MoEShape:
    """One workload.  ``n_shared`` shared SwiGLUs of width ``shared_inter`` are
    held as one SwiGLU of width ``n_shared * shared_inter`` (hidden units
    concatenated), which is the same function."""
    name: str
    T: int
    d: int
    I: int
    E: int
    k: int
    n_shared: int
    shared_inter: int
    wtype: str            # "bf16" or "fp8" (e4m3 + fp32 128x128 block scales)
    seed: int
    x_std: float = 1.0
    r_std: float = 1.0
    w_std: float = 0.02   # bf16 expert weights
    gate_std: float = 0.02
    zipf_bias: bool = False
    eps: float = 1e-6

    @property
    def Is(self) -> int:
        return self.n_shared * self.shared_inter

    def flops_per_token(self) -> int:
        """Algorithmic FLOP per token: routed + shared SwiGLUs (3 GEMVs each) + gate."""
        return 2 * self.d * self.I * 3 * self.k + 2 * self.d * self.Is * 3 + 2 * self.d * self.E


CONFIGS = {
    "C1": MoEShape("C1", T=64, d=256, I=128, E=8, k=2, n_shared=1, shared_inter=128, wtype="bf16", seed=0),
    "C2": MoEShape("C2", T=4096, d=2048, I=1024, E=64, k=6, n_shared=2, shared_inter=1024, wtype="bf16", seed=1),
    "C3": MoEShape("C3", T=128, d=7168, I=2048, E=256, k=8, n_shared=1, shared_inter=2048, wtype="fp8", seed=2),
    "C4": MoEShape("C4", T=16384, d=7168, I=2048, E=256, k=8, n_shared=1, shared_inter=2048, wtype="fp8", seed=3),
    "C5": MoEShape("C5", T=8192, d=7168, I=2048, E=256, k=8, n_shared=1, shared_inter=2048, wtype="fp8", seed=4,
                   r_std=2.0, zipf_bias=True),
    # a dense block: no router, one SwiGLU MLP (held as the "shared" weights).  The pages do not
    # give the dense MLP's width; 9 x 2048 = 18432 gives it the per-token FLOPs of the MoE block
    # (8 routed + 1 shared SwiGLU of 2048).
    "D1": MoEShape("D1", T=16384, d=7168, I=128, E=0, k=0, n_shared=1, shared_inter=18432, wtype="fp8", seed=5),
}

DESCRIPTIONS = {
    "C1": "tiny MoE layer: T=64, d=256, inter=128, 8 experts, top-2, 1 shared (inter 128), bf16",
    "C2": "mid bf16 MoE: T=4096, d=2048, inter=1024, 64 experts, top-6, 2 shared (inter 1024 each)",
    "C3": "DeepSeek-V3.2 MoE shape, decode batch: T=128, d=7168, inter=2048, 256 experts, top-8, 1 shared, FP8 128x128",
    "C4": "DeepSeek-V3.2 MoE shape, prefill batch: T=16384 (B=4 x 4096), d=7168, inter=2048, 256 experts, top-8, FP8",
    "C5": "DeepSeek-V3.2 MoE shape, Zipf(1.2) gate bias: T=8192, 256 experts, top-8, FP8, residual ~N(0,4)",
    "D1": "dense-MLP block of the same model (no router): T=16384, d=7168, MLP inter 18432 (stand-in width), FP8",
}


# ----------------------------------------------------------------------------------------------
# counter-based bits
# ----------------------------------------------------------------------------------------------
def _py_hash32(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * _C1) & _M32
    x ^= x >> 15
    x = (x * _C2) & _M32
    x ^= x >> 16
    return x


def _stream_keys(seed: int, stream: str) -> tuple[int, int]:
    s = zlib.crc32(stream.encode())
    k1 = _py_hash32(_py_hash32(seed * 0x9E3779B1 + 0x632BE5AB) ^ s)
    k2 = _py_hash32(k1 ^ 0x5BD1E995)
    return k1, k2


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    # (x * c) mod 2**32 with every partial product below 2**48
    lo = x * (c & 0xFFFF)
    hi = ((x * (c >> 16)) & 0xFFFF) << 16
    return (lo + hi) & _M32


def _hash32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, _C1)
    x = x ^ (x >> 15)
    x = _mul32(x, _C2)
    x = x ^ (x >> 16)
    return x


def uniform24(seed: int, stream: str, start: int, n: int, device="cpu") -> torch.Tensor:
    """24 uniform bits (int64 in [0, 2**24)) for elements start .. start+n-1 of a stream."""
    k1, k2 = _stream_keys(seed, stream)
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    h = _hash32((i & _M32) ^ k1)
    h = _hash32(h ^ (i >> 32) ^ k2)
    return h >> 8


def _unit(seed, stream, start, n, device):
    """uniform in the open interval (0, 1), float64."""
    return (uniform24(seed, stream, start, n, device).to(torch.float64) + 0.5) * (1.0 / 16777216.0)


_CHUNK = 1 << 23


def normal(seed: int, stream: str, shape, std: float, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, std^2) by Box-Muller in float64, rounded once to ``dtype``."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=dtype, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        u1 = _unit(seed, stream + ":u1", s, m, device)
        u2 = _unit(seed, stream + ":u2", s, m, device)
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
        out[s:s + m] = (z * std).to(dtype)
    return out.view(*shape)


def _uniform_range(seed, stream, shape, lo, hi, device) -> torch.Tensor:
    """float32 uniform in (lo, hi), computed in float64 then rounded once."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        u = _unit(seed, stream, s, m, device)
        out[s:s + m] = (lo + (hi - lo) * u).to(torch.float32)
    return out.view(*shape)


def _e4m3_codes(seed, stream, shape, device) -> torch.Tensor:
    """e4m3 codes (uint8 storage) of U(-448, 448) rounded to nearest-even by torch's cast."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.uint8, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        u = _unit(seed, stream, s, m, device)
        v = (-448.0 + 896.0 * u).to(torch.float32)
        out[s:s + m] = v.to(torch.float8_e4m3fn).view(torch.uint8)
    return out.view(*shape)


def zipf_bias(seed: int, E: int, alpha: float, s: float = 1.2) -> torch.Tensor:
    """Per-expert gate bias b_e = alpha * ln(rank_e ** -s), with rank_e the position of expert e in a
    seeded permutation of 1..E (float32, CPU)."""
    key = uniform24(seed, "zipf-rank", 0, E)
    order = torch.argsort(key * E + torch.arange(E), stable=True)   # distinct keys: index breaks ties
    rank = torch.empty(E, dtype=torch.float64)
    rank[order] = torch.arange(1, E + 1, dtype=torch.float64)
    return (alpha * (-s) * torch.log(rank)).to(torch.float32)


def generate(shape: MoEShape, device="cpu", alpha: Optional[float] = None, with_experts: bool = True,
             experts: Optional[list] = None) -> dict:
    """All inputs of one forward call as torch tensors on ``device``.

    FP8 tensors are returned as uint8 (raw e4m3 codes).  ``experts`` restricts the routed
    weights that are drawn (the others are left zero) -- used only by host-side tests that
    touch a few experts of a full-size layer.
    """
    T, d, I, E, Is, sd = shape.T, shape.d, shape.I, shape.E, shape.Is, shape.seed
    g = {}
    g["x"] = normal(sd, "x", (T, d), shape.x_std, device=device)
    g["residual"] = normal(sd, "residual", (T, d), shape.r_std, device=device)
    g["norm_w"] = torch.ones(d, dtype=torch.float32, device=device)
    g["gate_w"] = normal(sd, "gate_w", (E, d), shape.gate_std, device=device) if E > 0 else None
    if shape.zipf_bias:
        if alpha is None:
            raise ValueError("the Zipf-bias workload needs its alpha (tests/golden/c5_alpha.json)")
        g["gate_bias"] = zipf_bias(sd, E, alpha).to(device)
    else:
        g["gate_bias"] = None
    if not with_experts:
        return g
    fp8 = shape.wtype == "fp8"
    wdt = torch.uint8 if fp8 else torch.bfloat16

    def mat(name, rows, cols):
        if fp8:
            return _e4m3_codes(sd, name, (rows, cols), device)
        return normal(sd, name, (rows, cols), shape.w_std, device=device)

    def scl(name, rows, cols):
        return _uniform_range(sd, name + ":scale", (rows // 128, cols // 128), 1e-4, 2e-3, device)

    if E == 0:   # dense block: only the MLP ("shared") weights
        g["sw1"], g["sw3"], g["sw2"] = mat("sw1", Is, d), mat("sw3", Is, d), mat("sw2", d, Is)
        g["w1"] = g["w3"] = g["w2"] = g["s1"] = g["s3"] = g["s2"] = None
        if fp8:
            g["ss1"], g["ss3"], g["ss2"] = scl("sw1", Is, d), scl("sw3", Is, d), scl("sw2", d, Is)
        else:
            g["ss1"] = g["ss3"] = g["ss2"] = None
        return g
    sel = range(E) if experts is None else experts
    w1 = torch.zeros(E, I, d, dtype=wdt, device=device)
    w3 = torch.zeros(E, I, d, dtype=wdt, device=device)
    w2 = torch.zeros(E, d, I, dtype=wdt, device=device)
    if fp8:
        s1 = torch.zeros(E, I // 128, d // 128, dtype=torch.float32, device=device)
        s3 = torch.zeros_like(s1)
        s2 = torch.zeros(E, d // 128, I // 128, dtype=torch.float32, device=device)
    for e in sel:
        w1[e] = mat(f"w1/{e}", I, d)
        w3[e] = mat(f"w3/{e}", I, d)
        w2[e] = mat(f"w2/{e}", d, I)
        if fp8:
            s1[e] = scl(f"w1/{e}", I, d)
            s3[e] = scl(f"w3/{e}", I, d)
            s2[e] = scl(f"w2/{e}", d, I)
    g["w1"], g["w3"], g["w2"] = w1, w3, w2
    g["sw1"], g["sw3"], g["sw2"] = mat("sw1", Is, d), mat("sw3", Is, d), mat("sw2", d, Is)
    if fp8:
        g["s1"], g["s3"], g["s2"] = s1, s3, s2
        g["ss1"], g["ss3"], g["ss2"] = scl("sw1", Is, d), scl("sw3", Is, d), scl("sw2", d, Is)
    else:
        for n in ("s1", "s3", "s2", "ss1", "ss3", "ss2"):
            g[n] = None
    return g


def shape_dict(shape: MoEShape) -> dict:
    return asdict(shape)
