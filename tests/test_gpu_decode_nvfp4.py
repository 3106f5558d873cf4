"""Decode with NVFP4 experts ("How to Run Flint Locally", section "What vLLM
changed": the NVFP4 checkpoint runs weight-only with BF16 activations):
E2M1 codes, E4M3 scales per 16 elements, fp32 global scales per matrix,
through the C ABI, against the fp64 oracle's NVFP4 block.  Full-size layer
(256 experts, hidden 2,048), the synthetic NVFP4 recipe, decode inputs as in
the workload."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, routing_rows, torch, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    F.build()
    host = synth.nvfp4_layer_host(0)
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
def test_nvfp4_decode_matches_oracle(nv, seeds):
    x = synth.decode_x(seeds)
    out, gidx = decode(nv["L"], x)
    ref, idx, w, gap = oracle.moe_layer(nv["O"], x)
    rows = routing_rows(gidx, idx, gap)
    assert len(rows) >= len(seeds) - 1
    worst = check_close(bf16_to_f64(out), ref, rows)
    print(f"NVFP4 decode B={len(seeds)}: worst |err|/bound = {worst:.3e}")


@pytest.mark.parametrize("seeds", [[1, 2, 3, 4], list(range(50, 57))])
def test_nvfp4_decode_batch_invariance_bitwise(nv, seeds):
    x = synth.decode_x(seeds)
    out, _ = decode(nv["L"], x)
    for b in range(len(seeds)):
        alone, _ = decode(nv["L"], x[b:b + 1])
        assert np.array_equal(out[b], alone[0]), f"row {b} differs from its batch-1 run"


def test_nvfp4_residual_layer_and_stack(nv):
    """One stack layer (RMSNorm -> NVFP4 block -> fp32 residual add) against
    the oracle, and the stack call over two NVFP4 layers bitwise equal to two
    residual calls in turn."""
    h0 = synth.residual_h([60, 61, 62])
    h = torch().from_numpy(h0.copy()).cuda()
    ws, nb = workspace(F.FLINT_OP_DECODE, 3)
    idx = torch().empty((3, 6), dtype=torch().int32, device="cuda")
    F.flint_moe_decode_residual(nv["L"], h, 3, idx, None, ws, nb)
    torch().cuda.synchronize()
    got = h.cpu().numpy()
    ref, ridx, _, gap = oracle.stack_layer(nv["O"], h0)
    rows = routing_rows(idx.cpu().numpy(), ridx, gap)
    check_close(got.astype(np.float64) - h0, ref.astype(np.float64) - h0, rows, "NVFP4 residual")
    F.flint_moe_decode_residual(nv["L"], h, 3, None, None, ws, nb)
    hs = torch().from_numpy(h0.copy()).cuda()
    arr = F.layer_array([nv["L"], nv["L"]])
    F.flint_moe_decode_stack(arr, 2, hs, 3, None, None, None, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    assert np.array_equal(hs.cpu().numpy(), h.cpu().numpy())


def test_nvfp4_full_range_partial_is_the_block(nv):
    """Expert parallelism on NVFP4 experts: the share of all 256 experts and
    the shared one, combined, is bitwise the block output; two shards sum to
    it within the bound."""
    x = synth.decode_x([5, 6])
    out, _ = decode(nv["L"], x)
    ws, nb = workspace(F.FLINT_OP_DECODE, 2)
    parts = []
    for lo, hi, shr in ((0, 256, 1), (0, 100, 1), (100, 256, 0)):
        p = torch().empty((2, 2048), dtype=torch().float32, device="cuda")
        F.flint_moe_decode_partial(nv["L"], dev_bf16(x), None, 2, lo, hi, shr, p, ws, nb)
        parts.append(p)
    comb = torch().empty((2, 2048), dtype=torch().int16, device="cuda")
    F.flint_moe_combine_partials(parts[0], 2, comb, None)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    assert np.array_equal(host_bf16(comb), out)
    ref, idx, w, gap = oracle.moe_layer(nv["O"], x)
    total = (parts[1] + parts[2]).cpu().numpy().astype(np.float64)
    check_close(total, ref, [r for r in range(2) if gap[r] >= 1e-6], "NVFP4 shards summed")


def test_nvfp4_form_of_exactly_shared_weights_decodes_bitwise():
    """Weights both formats hold exactly (values in {0, +-1, +-2, +-3, +-4,
    +-6}): symmetric int4 codes with every bf16 scale 2^-7, and E2M1 codes
    with every E4M3 scale 1.0 and every global scale 2^-7.  Both decodes
    multiply the same bf16 weights and scale by powers of two, so their
    outputs agree bit for bit."""
    F.build()
    base = synth.layer_host(0)
    vals = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    enc = {0: 0x0, 1: 0x2, 2: 0x4, 3: 0x5, 4: 0x6, 6: 0x7}
    v = vals[np.arange(16) % 11]                     # nibble n -> value
    sym_nib = (v & 0xF).astype(np.uint8)
    nv_nib = np.array([enc[abs(a)] | (0x8 if a < 0 else 0) for a in v], np.uint8)
    byte = np.arange(256)
    sym_lut = (sym_nib[byte & 15] | (sym_nib[byte >> 4] << 4)).astype(np.uint8)
    nv_lut = (nv_nib[byte & 15] | (nv_nib[byte >> 4] << 4)).astype(np.uint8)
    sym, nvl = dict(base), dict(base)
    for name in ("w13", "w2", "sh13", "sh2"):
        q = np.asarray(base[name + "_q"], np.uint8)
        sym[name + "_q"], nvl[name + "_q"] = sym_lut[q], nv_lut[q]
        ss = base[name + "_s"].shape
        sym[name + "_s"] = np.full(ss, 0x3C00, np.uint16)                   # bf16 2^-7
        nvl[name + "_s"] = np.full(ss[:-1] + (ss[-1] * 8,), 0x38, np.uint8)  # E4M3 1.0
    nvl["w13_g"] = np.full((256, 2), 2.0 ** -7, np.float32)
    nvl["w2_g"] = np.full(256, 2.0 ** -7, np.float32)
    nvl["sh13_g"] = np.full(2, 2.0 ** -7, np.float32)
    nvl["sh2_g"] = np.full(1, 2.0 ** -7, np.float32)
    ds, dn = synth.to_device(sym, "cuda"), synth.to_device(nvl, "cuda")
    x = synth.decode_x([70, 71, 72, 73])
    a, ia = decode(F.make_layer(ds), x)
    b, ib = decode(F.make_layer(dn), x)
    assert np.array_equal(ia, ib) and np.array_equal(a, b)


def test_nvfp4_batch_limit(nv):
    """NVFP4 layers decode up to FLINT_MAX_DECODE_B_AFFINE = 7 rows; 8 is
    refused before any launch."""
    x = dev_bf16(synth.decode_x(list(range(8))))
    out = torch().empty((8, 2048), dtype=torch().int16, device="cuda")
    ws, nb = workspace(F.FLINT_OP_DECODE, 8)
    with pytest.raises(F.FlintError) as e:
        F.flint_moe_decode(nv["L"], x, 8, out, ws, nb)
    assert e.value.code == F.FLINT_EINVAL
