"""The bounds-checked build (libflint_debug.so, FLINT_DEBUG): the same sources
with every index the kernels read back from device memory (slot words, expert
indices, sorted token rows, GEMM tile descriptors) checked before it addresses
memory, a failed check reported as FLINT_EDEVICE in the call's status word.

On valid inputs the checks must neither fire nor change a result: every call
here runs through both libraries on the same inputs and workspaces, and the
debug library's outputs must equal the release library's bit for bit with the
status word clear.  Decode (batch 1, 4 and the residual form) and prefill
(5, 300 and 2,048 tokens) in the three expert formats, an expert shard,
routing, and the head GEMV."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import synth
from gpu_util import dev_bf16, host_bf16, torch, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    F.build()
    F.build(debug=True)
    sym = synth.layer_device(0, "cuda", host=synth.layer_host(0))
    aff = synth.to_device(synth.affine_layer_host(0), "cuda")
    nv = synth.nvfp4_layer_device(0, "cuda")
    return {"sym": F.make_layer(sym), "aff": F.make_layer(aff), "nv": F.make_layer(nv),
            "keep": (sym, aff, nv)}


def both(run):
    """run() through the release library, then through the debug library;
    the debug run's status words must be clear."""
    a = run()
    with F.using_library(F.DEBUG_LIB_PATH):
        b = run()
    return a, b


def decode(L, xbits):
    B = xbits.shape[0]
    out = torch().empty((B, 2048), dtype=torch().int16, device="cuda")
    idx = torch().empty((B, 6), dtype=torch().int32, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode(L, dev_bf16(xbits), B, out, ws, nb)
    w = torch().empty((B, 6), dtype=torch().float32, device="cuda")
    F.flint_moe_route(L, dev_bf16(xbits), B, idx, w, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == F.FLINT_OK
    return host_bf16(out), idx.cpu().numpy()


@pytest.mark.parametrize("fmt", ["sym", "aff", "nv"])
@pytest.mark.parametrize("seeds", [[0], [1, 2, 3, 4]])
def test_debug_decode_bitwise(env, fmt, seeds):
    x = synth.decode_x(seeds)
    (o1, i1), (o2, i2) = both(lambda: decode(env[fmt], x))
    assert np.array_equal(o1, o2) and np.array_equal(i1, i2)


def test_debug_residual_and_shard_bitwise(env):
    h0 = synth.residual_h([5, 6, 7])

    def run():
        h = torch().from_numpy(h0.copy()).cuda()
        ws, nb = workspace(F.FLINT_OP_DECODE, 3)
        F.flint_moe_decode_residual(env["sym"], h, 3, None, None, ws, nb)
        part = torch().empty((3, 2048), dtype=torch().float32, device="cuda")
        x = dev_bf16(synth.decode_x([5, 6, 7]))
        F.flint_moe_decode_partial(env["sym"], x, None, 3, 64, 192, 1, part, ws, nb)
        torch().cuda.synchronize()
        assert F.flint_read_status(ws) == F.FLINT_OK
        return h.cpu().numpy(), part.cpu().numpy()

    (h1, p1), (h2, p2) = both(run)
    assert np.array_equal(h1, h2) and np.array_equal(p1, p2)


def prefill(L, xbits):
    T = xbits.shape[0]
    out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
    idx = torch().empty((T, 6), dtype=torch().int32, device="cuda")
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_moe_prefill(L, dev_bf16(xbits), T, out, ws, nb)
    w = torch().empty((T, 6), dtype=torch().float32, device="cuda")
    F.flint_moe_route(L, dev_bf16(xbits), T, idx, w, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == F.FLINT_OK
    return host_bf16(out), idx.cpu().numpy()


@pytest.mark.parametrize("fmt,T", [("sym", 5), ("sym", 300), ("sym", 2048), ("aff", 300),
                                   ("nv", 300)])
def test_debug_prefill_bitwise(env, fmt, T):
    x = synth.prefill_x(T, T)
    (o1, i1), (o2, i2) = both(lambda: prefill(env[fmt], x))
    assert np.array_equal(o1, o2) and np.array_equal(i1, i2)


def test_debug_gemv_bitwise():
    F.build(debug=True)
    N, K, B = 20011, 2048, 3
    q = torch().from_numpy(synth.random_bytes(N, 41, N * K // 2).reshape(N, K // 2)).cuda()
    s = torch().from_numpy(synth.scale_bits(N, 42, N * K // 128).reshape(N, K // 128)
                           .view(np.int16)).cuda()
    x = dev_bf16(np.stack([synth.bf16_bits(synth.normals(300 + r, 43, K)) for r in range(B)]))

    def run():
        y = torch().empty((B, N), dtype=torch().float32, device="cuda")
        am = torch().empty((B,), dtype=torch().int32, device="cuda")
        nb = F.flint_gemv_workspace_bytes(N, B)
        ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
        F.flint_workspace_init(ws, nb)
        F.flint_int4_gemv(q, s, N, K, x, B, y, am, ws, nb)
        torch().cuda.synchronize()
        assert F.flint_read_status(ws) == F.FLINT_OK
        return y.cpu().numpy(), am.cpu().numpy()

    (y1, a1), (y2, a2) = both(run)
    assert np.array_equal(y1, y2) and np.array_equal(a1, a2)
