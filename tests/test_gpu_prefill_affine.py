"""Prefill with group-64 affine int4 experts ("How to Run Flint Locally",
section "Every build and its size": the MLX int4 build and the Q4_1 GGUF's
codes with FP16 scales and offsets), through the C ABI, against the fp64
oracle's affine block.  The grouped GEMMs round each weight code x scale +
offset (times the matrix's power of two) once to fp16; everything else is the
symmetric prefill path.  Full-size layer (256 experts, hidden 2,048), the
synthetic affine recipe, prefill inputs as in the workload (x ~ N(0, 1) bf16,
seed T)."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def aff():
    F.build()
    host = synth.affine_layer_host(0)
    dev = synth.to_device(host, "cuda")
    return {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}


def prefill(L, xbits):
    T = xbits.shape[0]
    x = dev_bf16(xbits)
    out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_moe_prefill(L, x, T, out, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return host_bf16(out)


def route(L, xbits):
    T = xbits.shape[0]
    idx = torch().empty((T, 6), dtype=torch().int32, device="cuda")
    w = torch().empty((T, 6), dtype=torch().float32, device="cuda")
    nb = F.flint_workspace_bytes(F.FLINT_OP_ROUTE, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_moe_route(L, dev_bf16(xbits), T, idx, w, ws, nb)
    torch().cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("T", [1, 5, 300])
def test_affine_prefill_matches_oracle(aff, T):
    x = synth.prefill_x(T, T)
    out = prefill(aff["L"], x)
    ref, idx, w, gap = oracle.moe_layer(aff["O"], x)
    rows = routing_rows(route(aff["L"], x), idx, gap)
    assert len(rows) >= T - 2
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"affine prefill T={T}: worst |err|/bound = {worst:.3e}")


def test_affine_prefill_2048_group_edges(aff):
    """The 2,048-token workload on affine experts: the first and the last
    token of every expert's group (each group's first and partial last tile)
    against the oracle."""
    T = 2048
    x = synth.prefill_x(T, T)
    out = prefill(aff["L"], x)
    ridx = route(aff["L"], x)
    rows = {0, T - 1}
    for e in range(256):
        toks = np.nonzero((ridx == e).any(axis=1))[0]
        if toks.size:
            rows.update((int(toks[0]), int(toks[-1])))
    rows = sorted(rows)
    ref, idx, w, gap = oracle.moe_layer(aff["O"], x[rows])
    keep = routing_rows(ridx[rows], idx, gap)
    assert len(keep) >= len(rows) - 2
    worst = check_close(bf16_to_f64(out[rows]), ref, keep)
    print(f"affine prefill T=2048: {len(rows)} group-edge rows, worst |err|/bound = {worst:.3e}")


@pytest.mark.parametrize("T", [300, 4096])
def test_affine_form_of_a_symmetric_layer_prefills_bitwise(T):
    """The symmetric layer 0 rewritten exactly in the affine format (codes +
    8, each bf16 scale as two fp16 scales, offsets -8 x scale) gives the
    same fp16 weights (the bound max(|m|, |15 s + m|) = 8 s puts the shift
    where the symmetric path puts it), so prefill on it gives bitwise the
    symmetric prefill's output."""
    F.build()
    sym = synth.layer_host(0)
    ds = synth.to_device(sym, "cuda")
    da = synth.to_device(synth.affine_from_symmetric(sym), "cuda")
    x = synth.prefill_x(T, T)
    a = prefill(F.make_layer(ds), x)
    b = prefill(F.make_layer(da), x)
    assert np.array_equal(a, b)


def test_affine_prefill_divided_up_rows_bitwise(aff):
    """Routed up projections stored divided by 4 (expert_interm_div = 4;
    fp16 scales and offsets both divided, exactly): the same output bits as
    the undivided layer, and within the bound of the oracle's divided layer."""
    T = 300
    hdiv = synth.divide_routed_up_affine(aff["host"], 2)
    ddiv = synth.to_device(hdiv, "cuda")
    x = synth.prefill_x(T, T)
    a = prefill(aff["L"], x)
    b = prefill(F.make_layer(ddiv, expert_interm_div=4), x)
    assert np.array_equal(a, b)
    ref, idx, w, gap = oracle.moe_layer(oracle.Layer(hdiv, expert_interm_div=4.0), x)
    rows = [r for r in range(T) if gap[r] >= 1e-6]
    check_close(bf16_to_f64(b), ref, rows, what="affine prefill, divided up rows")


def test_affine_prefill_repeat_runs_bitwise(aff):
    """Repeated runs of 4,096 tokens on one workspace give the same bits."""
    T = 4096
    x = dev_bf16(synth.prefill_x(T, T))
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    outs = []
    for _ in range(3):
        out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
        F.flint_moe_prefill(aff["L"], x, T, out, ws, nb)
        torch().cuda.synchronize()
        assert F.flint_read_status(ws) == 0
        outs.append(host_bf16(out))
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
