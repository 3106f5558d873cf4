"""Prefill with NVFP4 experts ("How to Run Flint Locally", section "What vLLM
changed": the NVFP4 checkpoint runs weight-only with BF16 activations),
through the C ABI, against the fp64 oracle's NVFP4 block.  The grouped GEMMs
take each E2M1 value times its E4M3 block scale as an exact fp16 weight and
the global scales in their read-out; everything else is the symmetric
prefill path.  Full-size layer, the synthetic NVFP4 recipe, prefill inputs as
in the workload (x ~ N(0, 1) bf16, seed T)."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    F.build()
    host = synth.nvfp4_layer_host(0)
    dev = synth.to_device(host, "cuda")
    return {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}


def prefill(L, xbits):
    T = xbits.shape[0]
    out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_moe_prefill(L, dev_bf16(xbits), T, out, ws, nb)
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
def test_nvfp4_prefill_matches_oracle(nv, T):
    x = synth.prefill_x(T, T)
    out = prefill(nv["L"], x)
    ref, idx, w, gap = oracle.moe_layer(nv["O"], x)
    rows = routing_rows(route(nv["L"], x), idx, gap)
    assert len(rows) >= T - 2
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"NVFP4 prefill T={T}: worst |err|/bound = {worst:.3e}")


def test_nvfp4_prefill_2048_group_edges(nv):
    """The 2,048-token workload on NVFP4 experts: the first and the last token
    of every expert's group (each group's first and partial last tile)."""
    T = 2048
    x = synth.prefill_x(T, T)
    out = prefill(nv["L"], x)
    ridx = route(nv["L"], x)
    rows = {0, T - 1}
    for e in range(256):
        toks = np.nonzero((ridx == e).any(axis=1))[0]
        if toks.size:
            rows.update((int(toks[0]), int(toks[-1])))
    rows = sorted(rows)
    ref, idx, w, gap = oracle.moe_layer(nv["O"], x[rows])
    keep = routing_rows(ridx[rows], idx, gap)
    assert len(keep) >= len(rows) - 2
    worst = check_close(bf16_to_f64(out[rows]), ref, keep)
    print(f"NVFP4 prefill T=2048: {len(rows)} group-edge rows, worst |err|/bound = {worst:.3e}")


def test_nvfp4_prefill_divided_up_rows_bitwise(nv):
    """Routed up projections stored divided by 4 (expert_interm_div = 4, here
    the up rows' global scales divided exactly): the same output bits as the
    undivided layer, and within the bound of the oracle's divided layer."""
    T = 300
    hdiv = dict(nv["host"])
    g = np.array(nv["host"]["w13_g"], np.float32).copy()
    g[:, 1] /= 4
    hdiv["w13_g"] = g
    ddiv = synth.to_device(hdiv, "cuda")
    x = synth.prefill_x(T, T)
    a = prefill(nv["L"], x)
    b = prefill(F.make_layer(ddiv, expert_interm_div=4), x)
    assert np.array_equal(a, b)
    ref, idx, w, gap = oracle.moe_layer(oracle.Layer(hdiv, expert_interm_div=4.0), x)
    check_close(bf16_to_f64(b), ref, [r for r in range(T) if gap[r] >= 1e-6],
                what="NVFP4 prefill, divided up rows")


def test_nvfp4_prefill_repeat_runs_bitwise(nv):
    """Repeated runs of 4,096 tokens on one workspace give the same bits."""
    T = 4096
    x = dev_bf16(synth.prefill_x(T, T))
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    outs = []
    for _ in range(3):
        out = torch().empty((T, 2048), dtype=torch().int16, device="cuda")
        F.flint_moe_prefill(nv["L"], x, T, out, ws, nb)
        torch().cuda.synchronize()
        assert F.flint_read_status(ws) == 0
        outs.append(host_bf16(out))
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
