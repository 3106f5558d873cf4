"""Routed up projections stored divided by 128 (the packs' expert_interm_div of
TandemLLM "21 Flint" section 21.2 "The packs"; the routing weights are
multiplied back).  Every step of the block scales by a power of two, so decode
(plain and residual) and prefill on the divided weights give bitwise the
outputs of the undivided ones; the oracle on the divided layer agrees within
the bound."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layers():
    F.build()
    host = synth.layer_host(0)
    hdiv = synth.divide_routed_up(host, 7)
    d0 = synth.layer_device(0, "cuda", host=host)
    d1 = synth.layer_device(0, "cuda", host=hdiv)
    return {"plain": F.make_layer(d0), "div": F.make_layer(d1, expert_interm_div=128),
            "O": oracle.Layer(hdiv, expert_interm_div=128.0), "keep": (d0, d1)}


def decode(L, x):
    B = x.shape[0]
    out = torch().empty((B, 2048), dtype=torch().int16, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode(L, dev_bf16(x), B, out, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return host_bf16(out)


def test_decode_divided_equals_undivided_bitwise(layers):
    x = synth.decode_x([1, 2, 3, 4])
    a = decode(layers["plain"], x)
    b = decode(layers["div"], x)
    assert np.array_equal(a, b)
    ref, idx, w, gap = oracle.moe_layer(layers["O"], x)
    rows = [r for r in range(4) if gap[r] >= 1e-6]
    check_close(bf16_to_f64(b), ref, rows, what="decode, divided up rows")


def test_residual_divided_equals_undivided_bitwise(layers):
    h0 = synth.residual_h([3000, 3001, 3002])
    out = []
    for key in ("plain", "div"):
        h = torch().from_numpy(h0.copy()).cuda()
        ws, nb = workspace(F.FLINT_OP_DECODE, 3)
        F.flint_moe_decode_residual(layers[key], h, 3, None, None, ws, nb)
        torch().cuda.synchronize()
        out.append(h.cpu().numpy())
    assert np.array_equal(out[0], out[1])


@pytest.mark.parametrize("T", [300, 4096])
def test_prefill_divided_equals_undivided_bitwise(layers, T):
    x = synth.prefill_x(T, T)
    res = []
    for key in ("plain", "div"):
        out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
        ws, nb = workspace(F.FLINT_OP_PREFILL, T)
        F.flint_moe_prefill(layers[key], dev_bf16(x), T, out, ws, nb)
        torch().cuda.synchronize()
        assert F.flint_read_status(ws) == 0
        res.append(host_bf16(out))
    assert np.array_equal(res[0], res[1])
    if T == 300:
        ref, idx, w, gap = oracle.moe_layer(layers["O"], x)
        rows = [r for r in range(T) if gap[r] >= 1e-6]
        check_close(bf16_to_f64(res[1]), ref, rows, what="prefill, divided up rows")
