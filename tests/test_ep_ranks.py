"""The expert-parallel plumbing on CPU: gloo ranks each take their shard of the
experts (int4_expert_routing_b200.ep.shard_range), compute the shard's partial
(the oracle stands in for the GPU kernel here), and sum the partials with the
same all-reduce the GPU path calls (ep.all_reduce_partials); every rank then
holds the block output of the oracle."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out, fmt="sym"):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from int4_expert_routing_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dims = synth.Dims(hidden=128, n_experts=256, top_k=6, expert_i=128, shared_i=128)
        make = {"sym": synth.layer_host, "affine": synth.affine_layer_host,
                "nvfp4": synth.nvfp4_layer_host}[fmt]
        L = oracle.Layer(make(3, dims))
        x = synth.bf16_bits(np.random.default_rng(4).normal(size=(3, 128)))
        lo, hi = ep.shard_range(rank, world)
        part = torch.from_numpy(oracle.moe_layer_partial(L, x, lo, hi, rank == 0))
        ep.all_reduce_partials(part)
        full, *_ = oracle.moe_layer(L, x)
        out.put((rank, (lo, hi), float(np.abs(part.numpy() - full).max()),
                 float(np.abs(full).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,fmt", [(2, "sym"), (4, "sym"), (2, "affine"), (3, "nvfp4")])
def test_ranks_sum_their_shards_to_the_block(world, fmt):
    """Each weight format: the shards' partials, all-reduced over gloo ranks,
    are the block output."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out, fmt))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=10) for _ in range(world))
    spans = [s for _, s, _, _ in res]
    assert spans[0][0] == 0 and spans[-1][1] == 256
    assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    for _, _, err, scale in res:
        assert err <= 1e-12 * scale


def test_shard_ranges_partition_the_experts():
    from int4_expert_routing_b200.ep import shard_range
    for world in (1, 2, 3, 4, 7, 8, 256):
        spans = [shard_range(r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 256
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        assert max(h - l for l, h in spans) - min(h - l for l, h in spans) <= 1
    with pytest.raises(ValueError):
        shard_range(2, 2)
