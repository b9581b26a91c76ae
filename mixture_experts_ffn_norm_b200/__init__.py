"""Python binding of libmoe (B200 / sm_100a MoE FFN forward).

Argument marshalling only: every step of the forward pass runs in the library's CUDA kernels.
The functions mirror the C ABI in include/moe.h and take torch tensors (device memory and
streams come from PyTorch).  Importing fails loudly when libmoe.so has not been built; there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT, \
    MOE_ERR_DEVICE_CHECK = range(7)
MOE_W_BF16, MOE_W_FP8_E4M3_B128 = 0, 1
MOE_ACT_FP8_1x128, MOE_ACT_BF16 = 0, 1

EXPORTS = ("moe_workspace_bytes", "moe_forward", "moe_forward_traced", "moe_forward_next_norm",
           "moe_forward_expert_slice", "moe_round_bf16", "moe_get_status",
           "moe_debug_routing",
           "moe_debug_norm", "moe_route_noalloc", "moe_selftest_wait_timeout", "moe_launches_per_forward",
           "moe_status_string")


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class moe_config_t(C.Structure):
    _fields_ = [("num_tokens", C.c_int32), ("dim", C.c_int32), ("inter_dim", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("shared_inter", C.c_int32), ("wtype", C.c_int32), ("amode", C.c_int32),
                ("eps", C.c_float)]


class moe_weights_t(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w1", "w3", "w2", "s1", "s3", "s2", "sw1", "sw3", "sw2", "ss1", "ss3", "ss2")]


_lib = None


def lib() -> C.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mixture_experts_ffn_norm_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, cfgp = C.c_void_p, C.POINTER(moe_config_t)
        L.moe_workspace_bytes.restype = C.c_size_t
        L.moe_workspace_bytes.argtypes = [cfgp]
        L.moe_forward.restype = C.c_int
        L.moe_forward.argtypes = [cfgp, vp, vp, vp, vp, vp, C.POINTER(moe_weights_t), vp, vp, vp, C.c_size_t, vp]
        L.moe_forward_traced.restype = C.c_int
        L.moe_forward_traced.argtypes = [cfgp, vp, vp, vp, vp, vp, C.POINTER(moe_weights_t), vp, vp, vp, C.c_size_t,
                                         vp, C.POINTER(C.c_void_p), C.c_int32]
        L.moe_forward_next_norm.restype = C.c_int
        L.moe_forward_next_norm.argtypes = [cfgp, vp, vp, vp, vp, vp, C.POINTER(moe_weights_t), vp, vp, vp, vp, vp,
                                            C.c_size_t, vp]
        L.moe_forward_expert_slice.restype = C.c_int
        L.moe_forward_expert_slice.argtypes = [cfgp, vp, vp, vp, vp, vp, C.POINTER(moe_weights_t), C.c_int32, C.c_int32,
                                               C.c_int32, vp, vp, vp, C.c_size_t, vp]
        L.moe_round_bf16.restype = C.c_int
        L.moe_round_bf16.argtypes = [vp, vp, C.c_int64, vp]
        L.moe_get_status.restype = C.c_int
        L.moe_get_status.argtypes = [vp, vp]
        L.moe_debug_routing.restype = C.c_int
        L.moe_debug_routing.argtypes = [cfgp, vp, vp, vp, vp, vp, vp]
        L.moe_debug_norm.restype = C.c_int
        L.moe_debug_norm.argtypes = [cfgp, vp, vp, vp, vp, vp]
        L.moe_route_noalloc.restype = C.c_int
        L.moe_route_noalloc.argtypes = [vp, C.c_int32, C.c_int32, C.c_int32, vp, vp, vp, vp, vp]
        L.moe_selftest_wait_timeout.restype = C.c_int
        L.moe_selftest_wait_timeout.argtypes = [vp, C.c_size_t, C.c_int64, vp]
        L.moe_launches_per_forward.restype = C.c_int32
        L.moe_launches_per_forward.argtypes = [cfgp]
        L.moe_status_string.restype = C.c_char_p
        L.moe_status_string.argtypes = [C.c_int]
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


@dataclass
class Config:
    num_tokens: int
    dim: int
    inter_dim: int
    n_experts: int
    top_k: int
    shared_inter: int
    wtype: int = MOE_W_FP8_E4M3_B128
    amode: int = MOE_ACT_FP8_1x128
    eps: float = 1e-6

    def c(self) -> moe_config_t:
        return moe_config_t(self.num_tokens, self.dim, self.inter_dim, self.n_experts, self.top_k, self.shared_inter,
                            self.wtype, self.amode, self.eps)

    @staticmethod
    def from_shape(shape, num_tokens=None) -> "Config":
        fp8 = shape.wtype == "fp8"
        return Config(num_tokens or shape.T, shape.d, shape.I, shape.E, shape.k, shape.Is,
                      MOE_W_FP8_E4M3_B128 if fp8 else MOE_W_BF16, MOE_ACT_FP8_1x128 if fp8 else MOE_ACT_BF16,
                      shape.eps)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def workspace_bytes(cfg: Config) -> int:
    return int(lib().moe_workspace_bytes(C.byref(cfg.c())))


def launches_per_forward(cfg: Config) -> int:
    return int(lib().moe_launches_per_forward(C.byref(cfg.c())))


def weights_struct(w: dict) -> moe_weights_t:
    return moe_weights_t(*[_ptr(w.get(n)) for n, _ in moe_weights_t._fields_])


def moe_forward(cfg: Config, x, residual, norm_w, gate_w, gate_bias, weights, out, residual_out, workspace,
                stream=None, check=True) -> int:
    """Enqueue one fused forward pass (see moe_forward in include/moe.h).  ``weights`` is a dict
    with keys w1, w3, w2, s1, s3, s2, sw1, sw3, sw2, ss1, ss3, ss2 (torch tensors or None) or a
    prepared moe_weights_t."""
    ws = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    rc = lib().moe_forward(C.byref(cfg.c()), _ptr(x), _ptr(residual), _ptr(norm_w), _ptr(gate_w), _ptr(gate_bias),
                           C.byref(ws), _ptr(out), _ptr(residual_out), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_forward")
    return rc


def moe_forward_traced(cfg: Config, x, residual, norm_w, gate_w, gate_bias, weights, out, residual_out, workspace,
                       events, stream=None, check=True) -> int:
    """moe_forward recording ``events`` (torch.cuda.Event, already created) at the stage boundaries."""
    ws = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    arr = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
    rc = lib().moe_forward_traced(C.byref(cfg.c()), _ptr(x), _ptr(residual), _ptr(norm_w), _ptr(gate_w),
                                  _ptr(gate_bias), C.byref(ws), _ptr(out), _ptr(residual_out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream), arr, len(events))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_forward_traced")
    return rc


def moe_forward_next_norm(cfg: Config, x, residual, norm_w, gate_w, gate_bias, weights, next_norm_w, out, next_xn,
                          next_residual, workspace, stream=None, check=True) -> int:
    """The forward pass with the next block's attn_norm fused in (see moe_forward_next_norm in
    include/moe.h); ``out`` may be None."""
    ws = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    rc = lib().moe_forward_next_norm(C.byref(cfg.c()), _ptr(x), _ptr(residual), _ptr(norm_w), _ptr(gate_w),
                                     _ptr(gate_bias), C.byref(ws), _ptr(next_norm_w), _ptr(out), _ptr(next_xn),
                                     _ptr(next_residual), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_forward_next_norm")
    return rc


def moe_forward_expert_slice(cfg: Config, x, residual, norm_w, gate_w, gate_bias, weights, expert_begin, expert_end,
                             with_shared, y_partial, residual_out, workspace, stream=None, check=True) -> int:
    """One rank's float32 partial of the expert-parallel layer (see include/moe.h)."""
    ws = weights if isinstance(weights, moe_weights_t) else weights_struct(weights)
    rc = lib().moe_forward_expert_slice(C.byref(cfg.c()), _ptr(x), _ptr(residual), _ptr(norm_w), _ptr(gate_w),
                                        _ptr(gate_bias), C.byref(ws), int(expert_begin), int(expert_end),
                                        int(bool(with_shared)), _ptr(y_partial), _ptr(residual_out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_forward_expert_slice")
    return rc


def moe_round_bf16(y, out, stream=None, check=True) -> int:
    rc = lib().moe_round_bf16(_ptr(y), _ptr(out), y.numel(), _stream(stream))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_round_bf16")
    return rc


def expert_parallel_forward(layer: "MoELayer", x, residual, out, residual_out, rank: int, world: int, group=None,
                            stream=None):
    """The expert-parallel layer on one rank ("MoE update" page, MoE.forward excerpt): this rank runs
    the contiguous expert range [rank * E / world, (rank + 1) * E / world) (rank 0 also the shared
    expert) into a float32 partial, the partials are summed over the ranks with
    torch.distributed.all_reduce (NCCL for device tensors; a CPU-only backend such as gloo sums a
    host copy), and the sum is rounded once to bf16 into ``out``.  Every rank gets the full output."""
    import torch
    import torch.distributed as dist
    cfg, t = layer.cfg, layer.t
    E = cfg.n_experts
    if E % world:
        raise ValueError("n_experts must divide evenly over the ranks")
    per = E // world
    y = torch.empty(cfg.num_tokens, cfg.dim, dtype=torch.float32, device=x.device)
    moe_forward_expert_slice(cfg, x, residual, t["norm_w"], t["gate_w"], t.get("gate_bias"), layer.wstruct,
                             rank * per, (rank + 1) * per, rank == 0, y, residual_out, layer.workspace, stream)
    if dist.get_backend(group) == "nccl":
        dist.all_reduce(y, group=group)
    else:
        host = y.cpu()
        dist.all_reduce(host, group=group)
        y.copy_(host)
    moe_round_bf16(y, out, stream)
    return out


def moe_get_status(workspace, stream=None) -> int:
    return int(lib().moe_get_status(_ptr(workspace), _stream(stream)))


def moe_debug_routing(cfg: Config, workspace, idx=None, weights=None, counts=None, near_tie=None, stream=None):
    rc = lib().moe_debug_routing(C.byref(cfg.c()), _ptr(workspace), _ptr(idx), _ptr(weights), _ptr(counts),
                                 _ptr(near_tie), _stream(stream))
    if rc != MOE_OK:
        raise MoeError(rc, "moe_debug_routing")


def moe_debug_norm(cfg: Config, workspace, xn=None, xq=None, xs=None, stream=None):
    rc = lib().moe_debug_norm(C.byref(cfg.c()), _ptr(workspace), _ptr(xn), _ptr(xq), _ptr(xs), _stream(stream))
    if rc != MOE_OK:
        raise MoeError(rc, "moe_debug_norm")


def moe_selftest_wait_timeout(workspace, limit_cycles: int = 1 << 21, stream=None) -> int:
    """Run the bounded-wait self-test on ``workspace`` (see include/moe.h); returns the call status."""
    return int(lib().moe_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                                limit_cycles, _stream(stream)))


def route_rows(num_tokens: int, top_k: int, n_experts: int) -> int:
    """Capacity R of the permuted-row space: roundup(T*k + 127*E, 128)."""
    return (num_tokens * top_k + 127 * n_experts + 127) // 128 * 128


def moe_route_noalloc(idx, n_experts: int, counts, offsets, row_of, row_token, stream=None, check=True) -> int:
    """Expert grouping without any workspace (see moe_route_noalloc in include/moe.h).  idx: [T, k]
    int32 device tensor; outputs are caller-provided int32 device tensors."""
    T, k = idx.shape
    rc = lib().moe_route_noalloc(_ptr(idx), T, k, n_experts, _ptr(counts), _ptr(offsets), _ptr(row_of),
                                 _ptr(row_token), _stream(stream))
    if check and rc != MOE_OK:
        raise MoeError(rc, "moe_route_noalloc")
    return rc


class MoELayer:
    """Convenience holder: device weights + workspace for one configuration.  ``forward`` is one
    call of moe_forward on the current stream."""

    def __init__(self, cfg: Config, tensors: dict, device="cuda"):
        import torch
        self.cfg = cfg
        self.t = {k: (None if v is None else v.to(device).contiguous()) for k, v in tensors.items()}
        self.wstruct = weights_struct(self.t)
        self.workspace = torch.empty(workspace_bytes(cfg), dtype=torch.uint8, device=device)
        if self.workspace.numel() == 0:
            raise MoeError(MOE_ERR_INVALID_ARG, "workspace_bytes")

    def forward(self, x, residual, out, residual_out, stream=None, check=True, events=None) -> int:
        t = self.t
        if events is not None:
            return moe_forward_traced(self.cfg, x, residual, t["norm_w"], t["gate_w"], t.get("gate_bias"),
                                      self.wstruct, out, residual_out, self.workspace, events, stream, check)
        return moe_forward(self.cfg, x, residual, t["norm_w"], t["gate_w"], t.get("gate_bias"), self.wstruct, out,
                           residual_out, self.workspace, stream, check)
