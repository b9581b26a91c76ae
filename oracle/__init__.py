"""CPU oracle for the MoE FFN forward pass -- TEST INFRASTRUCTURE ONLY.

Thin ctypes loader around ``oracle.c`` (plain float64 C, OpenMP over tokens).  Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs use it; the
product library never loads it.  It shares no code with the CUDA path: its inputs are numpy
arrays drawn by the ``synthetic`` generator.

Which page passage each C function follows is stated in ``oracle.c``.  Parity of the full
layer on arbitrary inputs is pinned only through the special cases the tests check (closed
forms, reductions to a dense SwiGLU, invariances); the pages print no worked numeric example.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no FMA contraction, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=gnu11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class Cfg(C.Structure):
    _fields_ = [("T", C.c_int), ("d", C.c_int), ("I", C.c_int), ("E", C.c_int), ("k", C.c_int),
                ("Is", C.c_int), ("fp8", C.c_int), ("act_fp8", C.c_int), ("eps", C.c_float)]


class Inputs(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("x", "residual", "norm_w", "gate_w", "gate_bias", "w1", "w3", "w2", "s1", "s3", "s2",
                 "sw1", "sw3", "sw2", "ss1", "ss3", "ss2")]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            vp, i, f, d = C.c_void_p, C.c_int, C.c_float, C.c_double
            L.oracle_bf16_to_f64.restype = d
            L.oracle_bf16_to_f64.argtypes = [C.c_uint16]
            L.oracle_f64_to_bf16.restype = C.c_uint16
            L.oracle_f64_to_bf16.argtypes = [d]
            L.oracle_e4m3_to_f64.restype = d
            L.oracle_e4m3_to_f64.argtypes = [C.c_uint8]
            L.oracle_f64_to_e4m3.restype = C.c_uint8
            L.oracle_f64_to_e4m3.argtypes = [d]
            L.oracle_mean_square.restype = f
            L.oracle_mean_square.argtypes = [i, vp]
            L.oracle_norm_token.restype = None
            L.oracle_norm_token.argtypes = [i, vp, vp, vp, f, vp, vp, vp, vp]
            L.oracle_act_quant.restype = None
            L.oracle_act_quant.argtypes = [i, vp, vp, vp, vp]
            L.oracle_swiglu.restype = None
            L.oracle_swiglu.argtypes = [i, i, i, i, vp, vp, vp, vp, vp, vp, vp, vp]
            L.oracle_gate_token.restype = None
            L.oracle_gate_token.argtypes = [i, i, i, vp, vp, vp, vp, vp, vp, vp]
            L.oracle_forward.restype = None
            L.oracle_forward.argtypes = [C.POINTER(Cfg), C.POINTER(Inputs), i, vp, i, vp, vp, vp, vp, vp, vp,
                                         vp, i]
            L.oracle_gate_scores.restype = None
            L.oracle_gate_scores.argtypes = [i, i, i, vp, vp, vp, vp, i]
            L.oracle_max_threads.restype = i
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _np(t, dtype=None):
    """torch tensor / numpy array / None -> contiguous numpy (uint16 view for bf16)."""
    if t is None:
        return None
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            if t.dtype == torch.float8_e4m3fn:
                return t.view(torch.uint8).numpy()
            t = t.numpy()
    except ImportError:
        pass
    a = np.ascontiguousarray(t)
    return a if dtype is None else a.astype(dtype, copy=False)


# ---------------------------------------------------------------------------------------------
# scalar / vector helpers
# ---------------------------------------------------------------------------------------------
def bf16_to_f64(bits):
    L = lib()
    return np.array([L.oracle_bf16_to_f64(int(b)) for b in np.ravel(bits)]).reshape(np.shape(bits))


def f64_to_bf16(vals):
    L = lib()
    return np.array([L.oracle_f64_to_bf16(float(v)) for v in np.ravel(vals)], dtype=np.uint16).reshape(np.shape(vals))


def e4m3_to_f64(codes):
    L = lib()
    return np.array([L.oracle_e4m3_to_f64(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def f64_to_e4m3(vals):
    L = lib()
    return np.array([L.oracle_f64_to_e4m3(float(v)) for v in np.ravel(vals)], dtype=np.uint8).reshape(np.shape(vals))


def mean_square(s32):
    s32 = np.ascontiguousarray(s32, dtype=np.float32)
    return float(lib().oracle_mean_square(len(s32), s32.ctypes.data))


def norm_token(x, r, g, eps=1e-6):
    """-> (xn bf16 bits, residual_out bf16 bits, xn64, xn32) for one token."""
    x, r, g = _np(x), _np(r), _np(g, np.float32)
    d = x.shape[-1]
    xn = np.empty(d, np.uint16)
    ro = np.empty(d, np.uint16)
    x64 = np.empty(d, np.float64)
    x32 = np.empty(d, np.float32)
    lib().oracle_norm_token(d, _p(x), _p(r), _p(g), eps, _p(xn), _p(ro), _p(x64), _p(x32))
    return xn, ro, x64, x32


def act_quant(v):
    """v: float64 values (multiple of 128) -> (codes u8, scales f32, dequantised f64)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    n = len(v)
    q = np.empty(n, np.uint8)
    sc = np.empty(n // 128, np.float32)
    dq = np.empty(n, np.float64)
    lib().oracle_act_quant(n, _p(v), _p(q), _p(sc), _p(dq))
    return q, sc, dq


def swiglu(a, w1, w3, w2, s1=None, s3=None, s2=None, act_fp8=False):
    """One SwiGLU on activation vector a (float64); weights [I,d],[I,d],[d,I]."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    w1, w3, w2 = _np(w1), _np(w3), _np(w2)
    fp8 = w1.dtype == np.uint8
    I, d = w1.shape
    s1, s3, s2 = _np(s1, np.float32), _np(s3, np.float32), _np(s2, np.float32)
    y = np.empty(d, np.float64)
    lib().oracle_swiglu(d, I, int(fp8), int(act_fp8), _p(a), _p(w1), _p(s1), _p(w3), _p(s3), _p(w2), _p(s2), _p(y))
    return y


def gate_token(xn_bits, gate_w, bias, k):
    xn, gw, b = _np(xn_bits), _np(gate_w), _np(bias, np.float32)
    E, d = gw.shape
    sc = np.empty(E, np.float64)
    idx = np.empty(k, np.int32)
    w = np.empty(k, np.float64)
    m = np.empty(1, np.float64)
    lib().oracle_gate_token(d, E, k, _p(xn), _p(gw), _p(b), _p(sc), _p(idx), _p(w), _p(m))
    return sc, idx, w, float(m[0])


def gate_scores(xn_bits, gate_w, bias=None, nthreads=0):
    xn, gw, b = _np(xn_bits), _np(gate_w), _np(bias, np.float32)
    n, d = xn.shape
    E = gw.shape[0]
    sc = np.empty((n, E), np.float64)
    lib().oracle_gate_scores(n, d, E, _p(xn), _p(gw), _p(b), _p(sc), nthreads)
    return sc


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class Oracle:
    """Holds host copies of one layer's inputs and evaluates the oracle on token subsets."""

    def __init__(self, shape, inputs: dict, act_fp8: bool | None = None):
        self.shape = shape
        fp8 = shape.wtype == "fp8"
        self.act_fp8 = fp8 if act_fp8 is None else act_fp8
        self.a = {k: _np(v) for k, v in inputs.items()}
        for k in ("norm_w", "gate_bias", "s1", "s3", "s2", "ss1", "ss3", "ss2"):
            if self.a.get(k) is not None:
                self.a[k] = np.ascontiguousarray(self.a[k], dtype=np.float32)
        self.cfg = Cfg(shape.T, shape.d, shape.I, shape.E, shape.k, shape.Is, int(fp8), int(self.act_fp8), shape.eps)
        inp = Inputs()
        for n, _ in Inputs._fields_:
            setattr(inp, n, _p(self.a.get(n)))
        self.inp = inp

    def forward(self, tokens=None, route_only=False, nthreads=0):
        s = self.shape
        tokens = np.arange(s.T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        n = len(tokens)
        r = {
            "out": None if route_only else np.empty((n, s.d), np.uint16),
            "residual_out": np.empty((n, s.d), np.uint16),
            "xn": np.empty((n, s.d), np.uint16),
            "xn64": np.empty((n, s.d), np.float64),
            "idx": np.empty((n, s.k), np.int32),
            "w": np.empty((n, s.k), np.float64),
            "margin": np.empty(n, np.float64),
        }
        lib().oracle_forward(C.byref(self.cfg), C.byref(self.inp), n, _p(tokens), int(route_only),
                             _p(r["out"]), _p(r["residual_out"]), _p(r["xn"]), _p(r["xn64"]), _p(r["idx"]),
                             _p(r["w"]), _p(r["margin"]), nthreads or default_threads())
        r["tokens"] = tokens
        return r


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Vectorised bf16 bits -> float64 (exact widening by bit shift; used by tests to compare)."""
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)
