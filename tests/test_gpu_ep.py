"""Expert parallelism on one GPU: every rank's shard computed in turn
(flint_moe_decode_partial), each against the oracle's partial of the same
experts, and the shares summed in rank order (the all-reduce's sum) and
finished by flint_moe_combine_partials, against the single-GPU block and the
oracle.  A rank may hold only its experts' weights: base pointers offset to
the shard give the same bits."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import bf16_to_f64, check_close, dev_bf16, host_bf16, torch, workspace
from int4_expert_routing_b200.ep import shard_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer0():
    F.build()
    host = synth.layer_host(0)
    dev = synth.layer_device(0, "cuda", host=host)
    return {"host": host, "dev": dev, "L": F.make_layer(dev), "O": oracle.Layer(host)}


def partials(env, x=None, h=None, world=2):
    B = (x if x is not None else h).shape[0]
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    out = []
    for r in range(world):
        lo, hi = shard_range(r, world)
        p = torch().full((B, 2048), float("nan"), dtype=torch().float32, device="cuda")
        F.flint_moe_decode_partial(env["L"], None if x is None else dev_bf16(x),
                                   None if h is None else torch().from_numpy(h.copy()).cuda(),
                                   B, lo, hi, r == 0, p, ws, nb)
        out.append(p)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return out


@pytest.mark.parametrize("world,seeds", [(2, [0]), (4, [1, 2, 3, 4]), (8, [1, 2, 3, 4]),
                                         (3, list(range(40, 48)))])
def test_shards_match_oracle_and_sum_to_the_block(layer0, world, seeds):
    x = synth.decode_x(seeds)
    B = len(seeds)
    ps = partials(layer0, x=x, world=world)
    for r, p in enumerate(ps):
        lo, hi = shard_range(r, world)
        ref = oracle.moe_layer_partial(layer0["O"], x, lo, hi, r == 0)
        got = p.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        for b in range(B):
            if not ref[b].any():
                assert not got[b].any()
        rows = [b for b in range(B) if ref[b].any()]
        check_close(got, ref, rows, what=f"shard {r} of {world}")
    total = ps[0].clone()
    for p in ps[1:]:
        total += p
    out = torch().empty((B, 2048), dtype=torch().int16, device="cuda")
    F.flint_moe_combine_partials(total, B, out, None)
    full = torch().empty_like(out)
    ws, nb = workspace(F.FLINT_OP_DECODE, B)
    F.flint_moe_decode(layer0["L"], dev_bf16(x), B, full, ws, nb)
    torch().cuda.synchronize()
    ref, idx, w, gap = oracle.moe_layer(layer0["O"], x)
    rows = [b for b in range(B) if gap[b] >= 1e-6]
    check_close(bf16_to_f64(host_bf16(out)), ref, rows, what=f"sum of {world} shards")
    check_close(bf16_to_f64(host_bf16(out)), bf16_to_f64(host_bf16(full)), rows,
                what="sharded vs single-GPU block")


def test_residual_form_matches_decode_residual(layer0):
    h0 = synth.residual_h([5000, 5001, 5002, 5003])
    ps = partials(layer0, h=h0, world=4)
    total = ps[0] + ps[1] + ps[2] + ps[3]
    h = torch().from_numpy(h0.copy()).cuda()
    F.flint_moe_combine_partials(total, 4, None, h)
    ref = torch().from_numpy(h0.copy()).cuda()
    ws, nb = workspace(F.FLINT_OP_DECODE, 4)
    F.flint_moe_decode_residual(layer0["L"], ref, 4, None, None, ws, nb)
    torch().cuda.synchronize()
    href, ridx, rw, gap = oracle.stack_layer(layer0["O"], h0)
    rows = [b for b in range(4) if gap[b] >= 1e-6]
    hs = h.cpu().numpy().astype(np.float64)
    check_close(hs - h0, href.astype(np.float64) - h0, rows, "sharded residual")
    check_close(hs - h0, ref.cpu().numpy().astype(np.float64) - h0, rows, "sharded vs single")


def test_rank_holding_only_its_experts(layer0):
    """Rank 1 of 4 with only experts 64..127 resident: base pointers offset so
    that expert 64's block sits at the first byte of the rank's copy; the
    partial is bitwise the one computed with all experts resident."""
    world, r = 4, 1
    lo, hi = shard_range(r, world)
    d = layer0["dev"]
    own = {k: d[k][lo:hi].clone() for k in ("w13_q", "w13_s", "w2_q", "w2_s")}
    t = dict(d)
    L = F.make_layer(t)
    for k in own:
        per = d[k][0].numel() * d[k].element_size()
        setattr(L, k, own[k].data_ptr() - lo * per)
    L._own = own
    x = synth.decode_x([1, 2, 3, 4])
    ws, nb = workspace(F.FLINT_OP_DECODE, 4)
    a = torch().empty((4, 2048), dtype=torch().float32, device="cuda")
    b = torch().empty_like(a)
    F.flint_moe_decode_partial(layer0["L"], dev_bf16(x), None, 4, lo, hi, False, a, ws, nb)
    F.flint_moe_decode_partial(L, dev_bf16(x), None, 4, lo, hi, False, b, ws, nb)
    torch().cuda.synchronize()
    assert torch().equal(a, b)


def test_full_range_partial_is_the_block_before_rounding(layer0):
    x = synth.decode_x([1, 2, 3, 4])
    ps = partials(layer0, x=x, world=1)
    out = torch().empty((4, 2048), dtype=torch().int16, device="cuda")
    F.flint_moe_combine_partials(ps[0], 4, out, None)
    full = torch().empty_like(out)
    ws, nb = workspace(F.FLINT_OP_DECODE, 4)
    F.flint_moe_decode(layer0["L"], dev_bf16(x), 4, full, ws, nb)
    torch().cuda.synchronize()
    assert torch().equal(out, full)
