"""Expert-parallel decode of the Flint MoE block over ranks (torch.distributed).

Each rank holds the router and a contiguous block of the 256 routed experts
(rank 0 also the shared expert); every rank computes the same routing, its
experts' weighted share of the block output in fp32 (flint_moe_decode_partial),
one all-reduce sums the shares, and flint_moe_combine_partials rounds the sum
to bf16 (or adds it to the residual stream).  Argument marshalling and the
collective only: the arithmetic runs in libflint's kernels, the sum in the
process group's all-reduce.
"""
from __future__ import annotations

from . import flint_moe_combine_partials, flint_moe_decode_partial

N_EXPERTS = 256


def shard_range(rank: int, world: int, n_experts: int = N_EXPERTS) -> tuple[int, int]:
    """[lo, hi) of the routed experts rank `rank` of `world` owns (contiguous
    blocks whose sizes differ by at most one)."""
    if not (0 <= rank < world <= n_experts):
        raise ValueError(f"rank {rank} of {world} over {n_experts} experts")
    return rank * n_experts // world, (rank + 1) * n_experts // world


def all_reduce_partials(partial, group=None) -> None:
    """Sum the ranks' partials in place on every rank."""
    import torch.distributed as dist
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)


def decode_ep(layer, x, h, B: int, partial, ws, ws_bytes: int, rank: int, world: int,
              out=None, group=None, stream=None) -> None:
    """One expert-parallel decode step of one layer on this rank.

    Exactly one of x (bf16 [B][2048] block input; the result goes to `out`)
    and h (fp32 [B][2048] residual stream; updated in place: h += bf16(block))
    is given.  `partial` is fp32 [B][2048] scratch that ends holding the sum.
    Every rank of the group makes the same call with its own layer shard."""
    import torch
    lo, hi = shard_range(rank, world)
    st = stream if stream is not None else torch.cuda.current_stream()
    flint_moe_decode_partial(layer, x, h, B, lo, hi, rank == 0, partial, ws, ws_bytes, stream=st)
    with torch.cuda.stream(st):
        all_reduce_partials(partial, group)
    flint_moe_combine_partials(partial, B, out if x is not None else None,
                               h if h is not None else None, stream=st)
