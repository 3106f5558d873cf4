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


def run(q, s, x, N, K, noalloc):
    B = x.shape[0]
    y = torch().empty((B, N), dtype=torch().float32, device="cuda")
    am = torch().empty(B, dtype=torch().int32, device="cuda")
    if noalloc:
        F.flint_int4_gemv_noalloc(q, s, N, K, x, B, y, am)
    else:
        nb = F.flint_gemv_workspace_bytes(N, B)
        ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
        F.flint_workspace_init(ws, nb)
        F.flint_int4_gemv(q, s, N, K, x, B, y, am, ws, nb)
    torch().cuda.synchronize()
    return y.cpu().numpy(), am.cpu().numpy()


@pytest.mark.parametrize("N,K,B", [(20000, 2048, 4), (4099, 384, 1), (150144, 2048, 2)])
def test_noalloc_gemv_matches_workspace_gemv_twice(N, K, B):
    F.build()
    qh = synth.random_bytes(N, 91, N * K // 2).reshape(N, K // 2)
    sh = synth.scale_bits(N, 92, N * K // 128).reshape(N, K // 128)
    xh = np.stack([synth.bf16_bits(synth.normals(100 + r, 93, K)) for r in range(B)])
    q = torch().from_numpy(qh).cuda()
    s = torch().from_numpy(sh.view(np.int16)).cuda()
    x = dev_bf16(xh)
    y_ref, am_ref = run(q, s, x, N, K, noalloc=False)
    for _ in range(2):                       # the scratch keeps the previous call's contents
        y, am = run(q, s, x, N, K, noalloc=True)
        check_close(y, y_ref.astype(np.float64), what="no-alloc logits")
        assert np.array_equal(am, am_ref)


def test_noalloc_rejects_bad_sizes():
    F.build()
    fake = 1 << 20
    for B in (0, 9):
        with pytest.raises(F.FlintError) as e:
            F.flint_int4_gemv_noalloc(fake, fake, 16, 2048, fake, B, fake, fake, stream=0)
        assert e.value.code == F.FLINT_EINVAL
