"""ctypes binding of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain statement of what the Flint
MoE block computes (see ``oracle.h`` for the definitions and readings).  Only
the test suite, the smoke check and the benchmark's CPU-baseline leg import
this package; the CUDA library never does.  This file only marshals arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (plain C, IEEE fp64, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.oracle_bf16_to_double.restype = C.c_double
        _lib.oracle_double_to_bf16.restype = C.c_uint16
        _lib.oracle_double_to_bf16.argtypes = [C.c_double]
        _lib.oracle_fp16_to_double.restype = C.c_double
        _lib.oracle_fp16_to_double.argtypes = [C.c_uint16]
        _lib.oracle_e2m1_to_double.restype = C.c_double
        _lib.oracle_e2m1_to_double.argtypes = [C.c_uint8]
        _lib.oracle_e4m3_to_double.restype = C.c_double
        _lib.oracle_e4m3_to_double.argtypes = [C.c_uint8]
        _lib.oracle_get_threads.restype = C.c_int
        set_threads(os.cpu_count() or 1)
    return _lib


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return lib().oracle_get_threads()


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


class _LayerC(C.Structure):
    _fields_ = [("n_experts", C.c_int), ("top_k", C.c_int), ("hidden", C.c_int),
                ("expert_i", C.c_int), ("shared_i", C.c_int)] + [
        (n, C.c_void_p) for n in ("router_w", "router_b", "w13_q", "w13_s", "w2_q", "w2_s",
                                  "sh13_q", "sh13_s", "sh2_q", "sh2_s")] + [
        ("expert_interm_div", C.c_double), ("format", C.c_int)] + [
        (n, C.c_void_p) for n in ("w13_m", "w2_m", "sh13_m", "sh2_m",
                                  "w13_g", "w2_g", "sh13_g", "sh2_g")]


_DT = {"router_w": np.uint16, "router_b": np.float32, "w13_q": np.uint8, "w13_s": np.uint16,
       "w2_q": np.uint8, "w2_s": np.uint16, "sh13_q": np.uint8, "sh13_s": np.uint16,
       "sh2_q": np.uint8, "sh2_s": np.uint16}


_OFFSETS = ("w13_m", "w2_m", "sh13_m", "sh2_m")
_GLOBALS = ("w13_g", "w2_g", "sh13_g", "sh2_g")
_SCALES = ("w13_s", "w2_s", "sh13_s", "sh2_s")


class Layer:
    """A MoE layer's host tensors (the dict ``synth.layer_host`` returns;
    ``synth.affine_layer_host``: with the *_m offset arrays the expert
    matrices are read as group-64 affine int4; ``synth.nvfp4_layer_host``:
    with the *_g global scales they are NVFP4, the *_s arrays E4M3 bytes)."""

    def __init__(self, t: dict, top_k: int = 6, expert_interm_div: float = 0.0):
        self.affine = "w13_m" in t
        self.nvfp4 = "w13_g" in t
        self.t = {k: np.ascontiguousarray(t[k], dtype=np.uint8 if (self.nvfp4 and k in _SCALES)
                                          else _DT[k]) for k in _DT}
        if self.affine:
            self.t.update({k: np.ascontiguousarray(t[k], dtype=np.uint16) for k in _OFFSETS})
        if self.nvfp4:
            self.t.update({k: np.ascontiguousarray(t[k], dtype=np.float32) for k in _GLOBALS})
        E, H = self.t["router_w"].shape
        self.E, self.H, self.k = E, H, top_k
        self.I = self.t["w13_s"].shape[1] // 2
        self.Is = self.t["sh13_s"].shape[0] // 2
        offs = [_p(self.t[n]).value if self.affine else None for n in _OFFSETS]
        gls = [_p(self.t[n]).value if self.nvfp4 else None for n in _GLOBALS]
        fmt = 1 if self.affine else (2 if self.nvfp4 else 0)
        self.c = _LayerC(E, top_k, H, self.I, self.Is, *[_p(self.t[n]).value for n in _DT],
                         float(expert_interm_div), fmt, *offs, *gls)


def unpack_int4(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    out = np.empty(2 * q.size, np.int8)
    lib().oracle_unpack_int4(_p(q), C.c_int64(out.size), _p(out))
    return out


def dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    N, K = q.shape[0], 2 * q.shape[1]
    W = np.empty((N, K), np.float64)
    lib().oracle_dequant(_p(q), _p(s), C.c_int64(N), C.c_int64(K), _p(W))
    return W


def bf16_from_double(v: float) -> int:
    return int(lib().oracle_double_to_bf16(float(v)))


def int4_gemv(q: np.ndarray, s: np.ndarray, x: np.ndarray):
    """(y[B,N] fp64, argmax[B] int32, top1-top2 gap[B])."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    N, K = q.shape[0], 2 * q.shape[1]
    B = x.shape[0]
    y = np.empty((B, N), np.float64)
    am = np.empty(B, np.int32)
    gap = np.empty(B, np.float64)
    lib().oracle_int4_gemv(_p(q), _p(s), C.c_int64(N), C.c_int64(K), _p(x), C.c_int(B),
                           _p(y), _p(am), _p(gap))
    return y, am, gap


def fp16_to_double(v: int) -> float:
    return float(lib().oracle_fp16_to_double(C.c_uint16(int(v))))


def dequant_affine(q: np.ndarray, s: np.ndarray, m: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    m = np.ascontiguousarray(m, dtype=np.uint16)
    N, K = q.shape[0], 2 * q.shape[1]
    W = np.empty((N, K), np.float64)
    lib().oracle_dequant_affine(_p(q), _p(s), _p(m), C.c_int64(N), C.c_int64(K), _p(W))
    return W


def int4_gemv_affine(q: np.ndarray, s: np.ndarray, m: np.ndarray, x: np.ndarray):
    """Group-64 affine int4 GEMV: (y[B,N] fp64, argmax[B] int32, top1-top2 gap[B])."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    m = np.ascontiguousarray(m, dtype=np.uint16)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    N, K = q.shape[0], 2 * q.shape[1]
    B = x.shape[0]
    y = np.empty((B, N), np.float64)
    am = np.empty(B, np.int32)
    gap = np.empty(B, np.float64)
    lib().oracle_int4_gemv_affine(_p(q), _p(s), _p(m), C.c_int64(N), C.c_int64(K), _p(x),
                                  C.c_int(B), _p(y), _p(am), _p(gap))
    return y, am, gap


def e2m1_to_double(v: int) -> float:
    return float(lib().oracle_e2m1_to_double(C.c_uint8(int(v))))


def e4m3_to_double(v: int) -> float:
    return float(lib().oracle_e4m3_to_double(C.c_uint8(int(v))))


def dequant_nvfp4(q: np.ndarray, s: np.ndarray, global_scale: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    N, K = q.shape[0], 2 * q.shape[1]
    W = np.empty((N, K), np.float64)
    lib().oracle_dequant_nvfp4(_p(q), _p(s), C.c_float(global_scale), C.c_int64(N), C.c_int64(K),
                               _p(W))
    return W


def int4_gemv_nvfp4(q: np.ndarray, s: np.ndarray, global_scale: float, x: np.ndarray):
    """NVFP4 weight-only GEMV: (y[B,N] fp64, argmax[B] int32, top1-top2 gap[B])."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    N, K = q.shape[0], 2 * q.shape[1]
    B = x.shape[0]
    y = np.empty((B, N), np.float64)
    am = np.empty(B, np.int32)
    gap = np.empty(B, np.float64)
    lib().oracle_int4_gemv_nvfp4(_p(q), _p(s), C.c_float(global_scale), C.c_int64(N),
                                 C.c_int64(K), _p(x), C.c_int(B), _p(y), _p(am), _p(gap))
    return y, am, gap


def route(L: Layer, x: np.ndarray):
    """dict of z, sig, biased [B,E]; idx [B,k]; w [B,k]; gap [B]."""
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    B = x.shape[0]
    r = {n: np.empty((B, L.E), np.float64) for n in ("z", "sig", "biased")}
    r["idx"] = np.empty((B, L.k), np.int32)
    r["w"] = np.empty((B, L.k), np.float64)
    r["gap"] = np.empty(B, np.float64)
    lib().oracle_route(C.byref(L.c), _p(x), C.c_int(B), _p(r["z"]), _p(r["sig"]),
                       _p(r["biased"]), _p(r["idx"]), _p(r["w"]), _p(r["gap"]))
    return r


def swiglu_expert(q13, s13, q2, s2, x: np.ndarray) -> np.ndarray:
    q13 = np.ascontiguousarray(q13, dtype=np.uint8)
    q2 = np.ascontiguousarray(q2, dtype=np.uint8)
    s13 = np.ascontiguousarray(s13, dtype=np.uint16)
    s2 = np.ascontiguousarray(s2, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    H, I = x.size, q13.shape[0] // 2
    y = np.empty(H, np.float64)
    lib().oracle_swiglu_expert(_p(q13), _p(s13), _p(q2), _p(s2), C.c_int(H), C.c_int(I),
                               _p(x), _p(y))
    return y


def moe_layer(L: Layer, x: np.ndarray):
    """(out[B,H] fp64, idx[B,k], w[B,k], gap[B])."""
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    B = x.shape[0]
    out = np.empty((B, L.H), np.float64)
    idx = np.empty((B, L.k), np.int32)
    w = np.empty((B, L.k), np.float64)
    gap = np.empty(B, np.float64)
    lib().oracle_moe_layer(C.byref(L.c), _p(x), C.c_int(B), _p(out), _p(idx), _p(w), _p(gap))
    return out, idx, w, gap


def moe_layer_partial(L: Layer, x: np.ndarray, e_lo: int, e_hi: int, with_shared: bool):
    """out[B,H] fp64: the block's terms from routed experts [e_lo, e_hi) and,
    with with_shared, the shared expert."""
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
    B = x.shape[0]
    out = np.empty((B, L.H), np.float64)
    lib().oracle_moe_layer_partial(C.byref(L.c), _p(x), C.c_int(B), C.c_int(e_lo), C.c_int(e_hi),
                                   C.c_int(1 if with_shared else 0), _p(out))
    return out


def rmsnorm_bf16(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    h = np.ascontiguousarray(np.atleast_2d(h), dtype=np.float32)
    x = np.empty(h.shape, np.uint16)
    lib().oracle_rmsnorm_bf16(_p(h), C.c_int(h.shape[0]), C.c_int(h.shape[1]),
                              C.c_double(eps), _p(x))
    return x


def stack_layer(L: Layer, h: np.ndarray, eps: float = 1e-6):
    """Returns (h_next fp32 [B,H], idx, w, gap); the input is not modified."""
    h = np.array(np.atleast_2d(h), dtype=np.float32, copy=True, order="C")
    B = h.shape[0]
    idx = np.empty((B, L.k), np.int32)
    w = np.empty((B, L.k), np.float64)
    gap = np.empty(B, np.float64)
    lib().oracle_stack_layer(C.byref(L.c), _p(h), C.c_int(B), C.c_double(eps), _p(idx),
                             _p(w), _p(gap))
    return h, idx, w, gap
