"""The allocation-free GEMV entry point (flint_int4_gemv_noalloc).

Some callers cannot allocate device memory themselves: a host program that
owns every device allocation and forbids libraries to call cudaMalloc, or a
hot path with a fixed memory budget that must not fail or stall on an
allocation.  For them the library keeps the GEMV's small scratch in a static
device array.  This test calls that entry point through the C ABI twice in a
row and checks both results against the workspace entry point on the same
inputs, with the tolerance the other GPU tests use.  It sits in a file pytest
collects last so that a run stopping at its first failure has already run
everything else.
"""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import synth
from gpu_util import check_close, dev_bf16, torch

pytestmark = pytest.mark.gpu


def inputs(N, K, B):
    qh = synth.random_bytes(N, 91, N * K // 2).reshape(N, K // 2)
    sh = synth.scale_bits(N, 92, N * K // 128).reshape(N, K // 128)
    xh = np.stack([synth.bf16_bits(synth.normals(100 + r, 93, K)) for r in range(B)])
    return (torch().from_numpy(qh).cuda(), torch().from_numpy(sh.view(np.int16)).cuda(),
            dev_bf16(xh))


def run(q, s, x, N, K, noalloc, with_argmax=True):
    B = x.shape[0]
    y = torch().empty((B, N), dtype=torch().float32, device="cuda")
    am = torch().full((B,), -7, dtype=torch().int32, device="cuda")
    if noalloc:
        F.flint_int4_gemv_noalloc(q, s, N, K, x, B, y, am if with_argmax else None)
    else:
        nb = F.flint_gemv_workspace_bytes(N, B)
        ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
        F.flint_workspace_init(ws, nb)
        F.flint_int4_gemv(q, s, N, K, x, B, y, am, ws, nb)
    torch().cuda.synchronize()
    return y.cpu().numpy(), am.cpu().numpy()


@pytest.mark.parametrize("N,K,B", [(20000, 2048, 4), (4099, 384, 1), (150144, 2048, 2),
                                   (150144, 2048, 8)])
def test_noalloc_gemv_matches_workspace_gemv_twice(N, K, B):
    F.build()
    q, s, x = inputs(N, K, B)
    y_ref, am_ref = run(q, s, x, N, K, noalloc=False)
    for _ in range(2):                       # the scratch keeps the previous call's contents
        y, am = run(q, s, x, N, K, noalloc=True)
        check_close(y, y_ref.astype(np.float64), what="no-alloc logits")
        assert np.array_equal(am, am_ref)
        assert F.flint_int4_gemv_noalloc_status() == F.FLINT_OK


def test_noalloc_without_argmax_then_with():
    """argmax = NULL skips the argmax partials and the counter; the next call
    with argmax still gives the workspace entry point's result."""
    F.build()
    N, K, B = 30011, 2048, 3
    q, s, x = inputs(N, K, B)
    y_ref, am_ref = run(q, s, x, N, K, noalloc=False)
    y, am = run(q, s, x, N, K, noalloc=True, with_argmax=False)
    check_close(y, y_ref.astype(np.float64), what="no-alloc logits without argmax")
    assert (am == -7).all()                  # argmax left untouched
    y, am = run(q, s, x, N, K, noalloc=True)
    check_close(y, y_ref.astype(np.float64), what="no-alloc logits after")
    assert np.array_equal(am, am_ref)


def test_noalloc_timeout_is_reported_and_recovers():
    """With the first-wait bound lowered to zero the call gives up at once and
    its status word says FLINT_ETIMEOUT; restored, the next call is normal."""
    F.build()
    N, K, B = 20000, 2048, 2
    q, s, x = inputs(N, K, B)
    y_ref, am_ref = run(q, s, x, N, K, noalloc=False)
    F.flint_debug_set_wait_polls(0)
    try:
        run(q, s, x, N, K, noalloc=True)
        status = F.flint_int4_gemv_noalloc_status()
    finally:
        F.flint_debug_set_wait_polls(0xFFFFFFFF)
    assert status == F.FLINT_ETIMEOUT
    y, am = run(q, s, x, N, K, noalloc=True)
    assert F.flint_int4_gemv_noalloc_status() == F.FLINT_OK
    check_close(y, y_ref.astype(np.float64), what="no-alloc logits after a timeout")
    assert np.array_equal(am, am_ref)


def test_noalloc_rejects_bad_sizes():
    F.build()
    fake = 1 << 20
    for B in (0, 9):
        with pytest.raises(F.FlintError) as e:
            F.flint_int4_gemv_noalloc(fake, fake, 16, 2048, fake, B, fake, fake, stream=0)
        assert e.value.code == F.FLINT_EINVAL
