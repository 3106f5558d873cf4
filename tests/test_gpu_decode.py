"""Decode path on the GPU, through the C ABI, against the fp64 oracle.

Full-size Flint MoE layers (256 experts, hidden 2,048), seeded synthetic
weights and inputs as in the workload recipe: layer 0 with x from seed 0
(batch 1) and seeds 1-4 (batch 4), batch 8, residual stack layers, and the
large-activation regime of TandemLLM "21 Flint" section 21.2.
"""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import (bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch,
                      workspace)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer0():
    F.build()
    assert torch().cuda.is_available(), "GPU tests need a CUDA device"
    host = synth.layer_host(0)
    dev = synth.layer_device(0, "cuda", host=host)
    return {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}


def decode(env, xbits):
    B = xbits.shape[0]
    x = dev_bf16(xbits)
    out = torch().empty((B, 2048), dtype=torch().int16, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode(env["L"], x, B, out, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return host_bf16(out)


def route(env, xbits):
    B = xbits.shape[0]
    x = dev_bf16(xbits)
    idx = torch().empty((B, 6), dtype=torch().int32, device="cuda")
    w = torch().empty((B, 6), dtype=torch().float32, device="cuda")
    ws, nb = workspace(F.FLINT_OP_ROUTE, B)
    F.flint_moe_route(env["L"], x, B, idx, w, ws, nb)
    torch().cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("seeds", [[0], [1, 2, 3, 4], list(range(20, 28))])
def test_route_matches_oracle(layer0, seeds):
    x = synth.decode_x(seeds)
    idx, w = route(layer0, x)
    r = oracle.route(layer0["O"], x)
    rows = routing_rows(idx, r["idx"], r["gap"])
    assert len(rows) >= len(seeds) - 1
    for b in rows:
        np.testing.assert_allclose(w[b], r["w"][b], rtol=0, atol=1e-6)
        assert abs(w[b].astype(np.float64).sum() - 1.0) < 1e-6


@pytest.mark.parametrize("seeds", [[0], [1, 2, 3, 4]])
def test_decode_matches_oracle(layer0, seeds):
    x = synth.decode_x(seeds)
    out = decode(layer0, x)
    ref, idx, w, gap = oracle.moe_layer(layer0["O"], x)
    ridx, _ = route(layer0, x)
    rows = routing_rows(ridx, idx, gap)
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"decode B={len(seeds)}: worst |err|/bound = {worst:.3e}")


@pytest.mark.parametrize("seeds", [[1, 2, 3, 4], list(range(30, 38)), [5, 5, 6]])
def test_decode_batch_invariance_bitwise(layer0, seeds):
    x = synth.decode_x(seeds)
    out = decode(layer0, x)
    for b in range(len(seeds)):
        alone = decode(layer0, x[b:b + 1])
        assert np.array_equal(out[b], alone[0]), f"row {b} differs from its batch-1 run"


def test_decode_deterministic(layer0):
    x = synth.decode_x([7, 8, 9])
    a = decode(layer0, x)
    b = decode(layer0, x)
    assert np.array_equal(a, b)


def test_decode_batch8_matches_oracle(layer0):
    x = synth.decode_x(list(range(40, 48)))
    out = decode(layer0, x)
    ref, idx, w, gap = oracle.moe_layer(layer0["O"], x)
    ridx, _ = route(layer0, x)
    rows = routing_rows(ridx, idx, gap)
    check_close(bf16_to_f64(out), ref, rows)


def test_decode_large_activations_stay_in_range(layer0):
    """x scaled by 512 (exact in bf16): routed SwiGLU intermediates reach ~1e5,
    past fp16; fp32 intermediates keep the output within tolerance."""
    x = synth.decode_x([3, 11])
    xs = synth.bf16_bits(bf16_to_f64(x) * 512.0)
    out = decode(layer0, xs)
    ref, idx, w, gap = oracle.moe_layer(layer0["O"], xs)
    assert np.all(np.isfinite(bf16_to_f64(out)))
    ridx, _ = route(layer0, xs)
    rows = routing_rows(ridx, idx, gap)
    check_close(bf16_to_f64(out), ref, rows)


def test_workspace_reused_across_layers(layer0):
    """Two different layers back to back on one workspace (the completion
    counter resets itself) give the same bytes as fresh workspaces."""
    host1 = synth.layer_host(1)
    dev1 = synth.layer_device(1, "cuda", host=host1)
    L1 = F.make_layer(dev1)
    x = dev_bf16(synth.decode_x([2, 3]))
    ws, nb = workspace(F.FLINT_OP_DECODE, 2)
    o0 = torch().empty((2, 2048), dtype=torch().int16, device="cuda")
    o1 = torch().empty_like(o0)
    F.flint_moe_decode(layer0["L"], x, 2, o0, ws, nb)
    F.flint_moe_decode(L1, x, 2, o1, ws, nb)
    F.flint_moe_decode(layer0["L"], x, 2, o0, ws, nb)
    torch().cuda.synchronize()
    env1 = {"L": L1}
    assert np.array_equal(host_bf16(o1), decode(env1, synth.decode_x([2, 3])))
    assert np.array_equal(host_bf16(o0), decode(layer0, synth.decode_x([2, 3])))


@pytest.mark.parametrize("layer_seed", [0, 46])
def test_residual_layer_matches_oracle(layer0, layer_seed):
    """One stacked layer on a seeded fp32 residual h: RMSNorm -> block ->
    h + bf16(out).  Compared per element on the block output h_out - h_in."""
    if layer_seed == 0:
        env = layer0
    else:
        host = synth.layer_host(layer_seed)
        dev = synth.layer_device(layer_seed, "cuda", host=host)
        env = {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}
    h0 = synth.residual_h([1000 + layer_seed, 1001 + layer_seed, 1002, 1003])
    B = h0.shape[0]
    h = torch().from_numpy(h0.copy()).cuda()
    idx = torch().empty((B, 6), dtype=torch().int32, device="cuda")
    w = torch().empty((B, 6), dtype=torch().float32, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode_residual(env["L"], h, B, idx, w, ws, nb)
    torch().cuda.synchronize()
    hg = h.cpu().numpy()
    href, ridx, rw, gap = oracle.stack_layer(env["O"], h0)
    rows = routing_rows(idx.cpu().numpy(), ridx, gap)
    check_close(hg.astype(np.float64) - h0, href.astype(np.float64) - h0, rows, "block output")
    np.testing.assert_allclose(w.cpu().numpy()[rows], rw[rows], rtol=0, atol=1e-6)


def test_residual_batch_invariance(layer0):
    h0 = synth.residual_h([2000, 2001, 2002])
    outs = []
    for rows in ([0, 1, 2], [0], [1], [2]):
        h = torch().from_numpy(h0[rows].copy()).cuda()
        ws, nb = workspace(F.FLINT_OP_DECODE, len(rows))
        F.flint_moe_decode_residual(layer0["L"], h, len(rows), None, None, ws, nb)
        torch().cuda.synchronize()
        outs.append(h.cpu().numpy())
    for b in range(3):
        assert np.array_equal(outs[0][b], outs[b + 1][0])


def test_device_code_generator_matches_host():
    t = synth.random_bytes_torch(9, synth.T_W2_Q, 1 << 20, "cuda", byte_offset=8 * 12345)
    assert np.array_equal(t.cpu().numpy(), synth.random_bytes(9, synth.T_W2_Q, 1 << 20, 8 * 12345))
