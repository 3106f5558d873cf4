"""Decode with group-64 affine int4 experts ("How to Run Flint Locally",
section "Every build and its size": the MLX int4 build and the Q4_1 GGUF's
codes with FP16 scales and offsets), through the C ABI, against the fp64
oracle's affine block: full-size layer (256 experts, hidden 2,048), the
synthetic affine recipe, decode inputs as in the workload."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def aff():
    F.build()
    host = synth.affine_layer_host(0)
    dev = synth.to_device(host, "cuda")
    return {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}


def decode(L, xbits):
    B = xbits.shape[0]
    x = dev_bf16(xbits)
    out = torch().empty((B, 2048), dtype=torch().int16, device="cuda")
    idx = torch().empty((B, 6), dtype=torch().int32, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode(L, x, B, out, ws, nb)
    F.flint_moe_route(L, x, B, idx, torch().empty((B, 6), dtype=torch().float32, device="cuda"),
                      ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return host_bf16(out), idx.cpu().numpy()


@pytest.mark.parametrize("seeds", [[0], [1, 2, 3, 4], list(range(40, 47))])
def test_affine_decode_matches_oracle(aff, seeds):
    x = synth.decode_x(seeds)
    out, gidx = decode(aff["L"], x)
    ref, idx, w, gap = oracle.moe_layer(aff["O"], x)
    rows = routing_rows(gidx, idx, gap)
    assert len(rows) >= len(seeds) - 1
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"affine decode B={len(seeds)}: worst |err|/bound = {worst:.3e}")


@pytest.mark.parametrize("seeds", [[1, 2, 3, 4], list(range(50, 57))])
def test_affine_decode_batch_invariance_bitwise(aff, seeds):
    x = synth.decode_x(seeds)
    out, _ = decode(aff["L"], x)
    for b in range(len(seeds)):
        alone, _ = decode(aff["L"], x[b:b + 1])
        assert np.array_equal(out[b], alone[0]), f"row {b} differs from its batch-1 run"


def test_affine_residual_layer_matches_oracle(aff):
    """One stack layer (RMSNorm -> affine block -> fp32 residual add)."""
    h0 = synth.residual_h([60, 61, 62])
    h = torch().from_numpy(h0.copy()).cuda()
    ws, nb = workspace(F.FLINT_OP_DECODE, 3)
    idx = torch().empty((3, 6), dtype=torch().int32, device="cuda")
    F.flint_moe_decode_residual(aff["L"], h, 3, idx, None, ws, nb)
    torch().cuda.synchronize()
    got = h.cpu().numpy()
    ref, ridx, _, gap = oracle.stack_layer(aff["O"], h0)
    rows = routing_rows(idx.cpu().numpy(), ridx, gap)
    check_close(got.astype(np.float64) - h0, ref.astype(np.float64) - h0, rows, "affine residual")


def test_affine_form_of_a_symmetric_layer_matches_its_oracle():
    """The symmetric layer 0 rewritten exactly in the affine format (codes +
    8, scales split per 64, offsets -8 x scale) is the same function: the GPU
    affine path on it meets the bound of the symmetric oracle."""
    F.build()
    sym = synth.layer_host(0)
    dev = synth.to_device(synth.affine_from_symmetric(sym), "cuda")
    x = synth.decode_x([70, 71, 72, 73])
    out, gidx = decode(F.make_layer(dev), x)
    ref, idx, w, gap = oracle.moe_layer(oracle.Layer(sym), x)
    rows = routing_rows(gidx, idx, gap)
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"affine form of the symmetric layer: worst |err|/bound = {worst:.3e}")


def test_affine_batch_limit(aff):
    """Affine layers decode up to FLINT_MAX_DECODE_B_AFFINE = 7 rows; 8 is
    refused before any launch (routing alone still takes 8)."""
    x = dev_bf16(synth.decode_x(list(range(8))))
    out = torch().empty((8, 2048), dtype=torch().int16, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, 8)
    with pytest.raises(F.FlintError) as e:
        F.flint_moe_decode(aff["L"], x, 8, out, ws, nb)
    assert e.value.code == F.FLINT_EINVAL
    idx = torch().empty((8, 6), dtype=torch().int32, device="cuda")
    F.flint_moe_route(aff["L"], x, 8, idx, torch().empty((8, 6), dtype=torch().float32,
                                                         device="cuda"), ws, nb)
    torch().cuda.synchronize()

