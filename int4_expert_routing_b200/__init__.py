"""Python binding of libflint (the Flint int4 MoE block for B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libflint.so``.  Each function has the name and argument order of
its C entry point (see ``include/flint.h``); device buffers are torch CUDA
tensors (their data pointers are passed), and ``stream`` defaults to torch's
current stream.  A missing or unloadable library raises: there is no fallback.
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libflint.so")
# the bounds-checked build (FLINT_DEBUG): same ABI, every index the kernels
# read back from device memory checked before use (FLINT_EDEVICE on failure)
DEBUG_LIB_PATH = os.path.join(HERE, "libflint_debug.so")

FLINT_OK, FLINT_EINVAL, FLINT_ECUDA, FLINT_ETIMEOUT, FLINT_EDEVICE = range(5)
FLINT_OP_ROUTE, FLINT_OP_DECODE, FLINT_OP_PREFILL, FLINT_OP_GEMV = range(4)
HIDDEN, EXPERTS, TOP_K, EXPERT_I, SHARED_I, GROUP, MAX_DECODE_B = 2048, 256, 6, 512, 1024, 128, 8

EXPORTS = ("flint_version", "flint_strerror", "flint_last_cuda_error", "flint_workspace_bytes",
           "flint_gemv_workspace_bytes", "flint_workspace_init", "flint_read_status",
           "flint_moe_route", "flint_moe_decode", "flint_moe_decode_residual", "flint_moe_decode_stack",
           "flint_moe_decode_partial", "flint_moe_combine_partials",
           "flint_moe_prefill", "flint_int4_gemv", "flint_int4_gemv_affine", "flint_int4_gemv_nvfp4",
           "flint_int4_gemv_noalloc",
           "flint_int4_gemv_noalloc_status",
           "flint_debug_set_wait_polls", "flint_debug_prefill_events",
           "flint_debug_prefill_stage_ms")

_lib = None
_loaded = {}  # path -> CDLL with its signatures set


class FlintError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = f" [{lib().flint_last_cuda_error().decode()}]" if code == FLINT_ECUDA else ""
        super().__init__(f"{where}: {strerror(code)} ({code}){detail}")


_WEIGHTS = ("router_w", "router_b", "w13_q", "w13_s", "w2_q", "w2_s",
            "sh13_q", "sh13_s", "sh2_q", "sh2_s")
_OFFSETS = ("w13_m", "w2_m", "sh13_m", "sh2_m")
_GLOBALS = ("w13_g", "w2_g", "sh13_g", "sh2_g")
FLINT_FMT_SYM_INT4 = 0
FLINT_FMT_AFFINE_INT4 = 1
FLINT_FMT_NVFP4 = 2
FLINT_MAX_DECODE_B_AFFINE = 7  # decode batch limit of affine and NVFP4 layers (flint.h)


class flint_moe_layer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _WEIGHTS] + [
        ("expert_interm_div", C.c_int), ("format", C.c_int)] + [
        (n, C.c_void_p) for n in _OFFSETS + _GLOBALS]


def build(force: bool = False, debug: bool = False) -> str:
    from . import buildlib
    return buildlib.build(force=force, debug=debug)


def lib() -> C.CDLL:
    """Load libflint.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Route the calls made inside the block to the library at ``path`` (for
    instance DEBUG_LIB_PATH, built by ``build(debug=True)``); the default
    library afterwards."""
    global _lib
    saved = lib()
    _lib = _load(path)
    try:
        yield _lib
    finally:
        _lib = saved


def _load(path: str) -> C.CDLL:
    if path not in _loaded:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built: run int4_expert_routing_b200.build()")
        L = C.CDLL(path)
        vp, i, sz = C.c_void_p, C.c_int, C.c_size_t
        L.flint_version.restype = i
        L.flint_strerror.restype = C.c_char_p
        L.flint_strerror.argtypes = [i]
        L.flint_last_cuda_error.restype = C.c_char_p
        L.flint_workspace_bytes.restype = sz
        L.flint_workspace_bytes.argtypes = [i, i]
        L.flint_gemv_workspace_bytes.restype = sz
        L.flint_gemv_workspace_bytes.argtypes = [i, i]
        L.flint_workspace_init.argtypes = [vp, sz, vp]
        L.flint_read_status.argtypes = [vp, C.POINTER(C.c_int), vp]
        L.flint_debug_set_wait_polls.argtypes = [C.c_uint32]
        L.flint_debug_prefill_events.argtypes = [C.c_int]
        L.flint_debug_prefill_stage_ms.argtypes = [C.POINTER(C.c_float), C.c_int]
        lp = C.POINTER(flint_moe_layer)
        L.flint_moe_route.argtypes = [lp, vp, i, vp, vp, vp, sz, vp]
        L.flint_moe_decode.argtypes = [lp, vp, i, vp, vp, sz, vp]
        L.flint_moe_decode_residual.argtypes = [lp, vp, i, vp, vp, vp, sz, vp]
        L.flint_moe_decode_stack.argtypes = [lp, i, vp, i, vp, vp, vp, vp, sz, vp]
        L.flint_moe_decode_partial.argtypes = [lp, vp, vp, i, i, i, i, vp, vp, sz, vp]
        L.flint_moe_combine_partials.argtypes = [vp, i, vp, vp, vp]
        L.flint_moe_prefill.argtypes = [lp, vp, i, vp, vp, sz, vp]
        L.flint_int4_gemv.argtypes = [vp, vp, i, i, vp, i, vp, vp, vp, sz, vp]
        L.flint_int4_gemv_affine.argtypes = [vp, vp, vp, i, i, vp, i, vp, vp, vp, sz, vp]
        L.flint_int4_gemv_nvfp4.argtypes = [vp, vp, C.c_float, i, i, vp, i, vp, vp, vp, sz, vp]
        L.flint_int4_gemv_noalloc.argtypes = [vp, vp, i, i, vp, i, vp, vp, vp]
        L.flint_int4_gemv_noalloc_status.argtypes = [C.POINTER(C.c_int), vp]
        for name in EXPORTS:
            getattr(L, name).restype = getattr(L, name).restype or i
        _loaded[path] = L
    return _loaded[path]


def strerror(code: int) -> str:
    return lib().flint_strerror(int(code)).decode()


def version() -> int:
    return lib().flint_version()


# ------------------------------------------------------------- marshalling
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(code: int, where: str):
    if code != FLINT_OK:
        raise FlintError(code, where)


def make_layer(t: dict, expert_interm_div: int = 0) -> flint_moe_layer:
    """The C layer struct from a dict of device tensors (keys as in flint.h)
    and the divisor of the routed up projections (0: not divided).  With the
    *_m offset tensors the experts are group-64 affine int4
    (FLINT_FMT_AFFINE_INT4); with the *_g global-scale tensors they are NVFP4
    (FLINT_FMT_NVFP4).  The struct keeps a reference to the tensors, so their
    memory stays allocated while the struct is alive."""
    affine, nvfp4 = "w13_m" in t, "w13_g" in t
    fmt = FLINT_FMT_AFFINE_INT4 if affine else (FLINT_FMT_NVFP4 if nvfp4 else FLINT_FMT_SYM_INT4)
    layer = flint_moe_layer(*[_ptr(t[n]) for n in _WEIGHTS], int(expert_interm_div), fmt,
                            *[_ptr(t[n]) if affine else None for n in _OFFSETS],
                            *[_ptr(t[n]) if nvfp4 else None for n in _GLOBALS])
    layer._tensors = t
    return layer


def flint_workspace_bytes(op: int, n: int) -> int:
    return lib().flint_workspace_bytes(op, n)


def flint_gemv_workspace_bytes(N: int, B: int) -> int:
    return lib().flint_gemv_workspace_bytes(N, B)


def flint_workspace_init(ws, ws_bytes: int, stream=None):
    _check(lib().flint_workspace_init(_ptr(ws), ws_bytes, _stream(stream)), "flint_workspace_init")


def flint_debug_set_wait_polls(polls: int) -> None:
    """Poll bound of the decode kernels' first barrier waits (test hook for
    the timeout path); 0xFFFFFFFF restores the default."""
    _check(lib().flint_debug_set_wait_polls(polls), "flint_debug_set_wait_polls")


PREFILL_STAGES = ("routing", "sort", "scaling+gather", "gemm1", "gemm2", "combine")


def flint_debug_prefill_events(enable: bool) -> None:
    """Record CUDA events between the stages of flint_moe_prefill (measurement)."""
    _check(lib().flint_debug_prefill_events(1 if enable else 0), "flint_debug_prefill_events")


def flint_debug_prefill_stage_ms() -> dict:
    """Stage times (ms) of the last flint_moe_prefill call made with events on."""
    buf = (C.c_float * 6)()
    _check(lib().flint_debug_prefill_stage_ms(buf, 6), "flint_debug_prefill_stage_ms")
    return dict(zip(PREFILL_STAGES, list(buf)))


def flint_read_status(ws, stream=None) -> int:
    st = C.c_int(0)
    _check(lib().flint_read_status(_ptr(ws), C.byref(st), _stream(stream)), "flint_read_status")
    return st.value


def flint_moe_route(layer: flint_moe_layer, x, B: int, idx, w, ws, ws_bytes: int, stream=None):
    _check(lib().flint_moe_route(C.byref(layer), _ptr(x), B, _ptr(idx), _ptr(w), _ptr(ws),
                                 ws_bytes, _stream(stream)), "flint_moe_route")


def flint_moe_decode(layer: flint_moe_layer, x, B: int, out, ws, ws_bytes: int, stream=None):
    _check(lib().flint_moe_decode(C.byref(layer), _ptr(x), B, _ptr(out), _ptr(ws), ws_bytes,
                                  _stream(stream)), "flint_moe_decode")


def flint_moe_decode_residual(layer: flint_moe_layer, h, B: int, idx, w, ws, ws_bytes: int,
                              stream=None):
    _check(lib().flint_moe_decode_residual(C.byref(layer), _ptr(h), B, _ptr(idx), _ptr(w),
                                           _ptr(ws), ws_bytes, _stream(stream)),
           "flint_moe_decode_residual")


def layer_array(layers) -> C.Array:
    """A contiguous host array of layer structs (for flint_moe_decode_stack);
    keeps the structs' tensors alive."""
    arr = (flint_moe_layer * len(layers))(*layers)
    arr._keep = list(layers)
    return arr


def flint_moe_decode_stack(layers, L: int, h, B: int, idx, w, h_trace, ws, ws_bytes: int,
                           stream=None):
    """``layers``: an array from ``layer_array`` (or a list of structs)."""
    if not isinstance(layers, C.Array):
        layers = layer_array(layers)
    _check(lib().flint_moe_decode_stack(layers, L, _ptr(h), B, _ptr(idx), _ptr(w), _ptr(h_trace),
                                        _ptr(ws), ws_bytes, _stream(stream)),
           "flint_moe_decode_stack")


def flint_moe_decode_partial(layer: flint_moe_layer, x, h, B: int, expert_lo: int,
                             expert_hi: int, with_shared: bool, partial, ws, ws_bytes: int,
                             stream=None):
    """One expert shard's fp32 share of the decode block (exactly one of x, h)."""
    _check(lib().flint_moe_decode_partial(C.byref(layer), _ptr(x), _ptr(h), B, expert_lo,
                                          expert_hi, 1 if with_shared else 0, _ptr(partial),
                                          _ptr(ws), ws_bytes, _stream(stream)),
           "flint_moe_decode_partial")


def flint_moe_combine_partials(total, B: int, out, h, stream=None):
    """out = bf16(total) and / or h += bf16(total)."""
    _check(lib().flint_moe_combine_partials(_ptr(total), B, _ptr(out), _ptr(h), _stream(stream)),
           "flint_moe_combine_partials")


def flint_moe_prefill(layer: flint_moe_layer, x, T: int, out, ws, ws_bytes: int, stream=None):
    _check(lib().flint_moe_prefill(C.byref(layer), _ptr(x), T, _ptr(out), _ptr(ws), ws_bytes,
                                   _stream(stream)), "flint_moe_prefill")


def flint_int4_gemv(q, s, N: int, K: int, x, B: int, y, argmax, ws, ws_bytes: int, stream=None):
    _check(lib().flint_int4_gemv(_ptr(q), _ptr(s), N, K, _ptr(x), B, _ptr(y), _ptr(argmax),
                                 _ptr(ws), ws_bytes, _stream(stream)), "flint_int4_gemv")


def flint_int4_gemv_affine(q, s, m, N: int, K: int, x, B: int, y, argmax, ws, ws_bytes: int,
                           stream=None):
    _check(lib().flint_int4_gemv_affine(_ptr(q), _ptr(s), _ptr(m), N, K, _ptr(x), B, _ptr(y),
                                        _ptr(argmax), _ptr(ws), ws_bytes, _stream(stream)),
           "flint_int4_gemv_affine")


def flint_int4_gemv_nvfp4(q, s, global_scale: float, N: int, K: int, x, B: int, y, argmax, ws,
                          ws_bytes: int, stream=None):
    _check(lib().flint_int4_gemv_nvfp4(_ptr(q), _ptr(s), float(global_scale), N, K, _ptr(x), B,
                                       _ptr(y), _ptr(argmax), _ptr(ws), ws_bytes, _stream(stream)),
           "flint_int4_gemv_nvfp4")


def flint_int4_gemv_noalloc(q, s, N: int, K: int, x, B: int, y, argmax, stream=None):
    """flint_int4_gemv with the library's own static scratch (no workspace)."""
    _check(lib().flint_int4_gemv_noalloc(_ptr(q), _ptr(s), N, K, _ptr(x), B, _ptr(y),
                                         _ptr(argmax), _stream(stream)), "flint_int4_gemv_noalloc")


def flint_int4_gemv_noalloc_status(stream=None) -> int:
    """Status word of the allocation-free GEMV's static array on the current
    device (synchronizes the stream)."""
    st = C.c_int(0)
    _check(lib().flint_int4_gemv_noalloc_status(C.byref(st), _stream(stream)),
           "flint_int4_gemv_noalloc_status")
    return st.value
