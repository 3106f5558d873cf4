"""The decode kernels' timeout path, driven without a GPU fault: the bound of
their first barrier waits is lowered to zero polls, so every CTA gives up at
once, records FLINT_ETIMEOUT in the workspace status word and returns (the
waits on the error path keep the full bound, so the copies already issued land
first).  The call must end promptly, report the status, and leave the library
usable: with the bound restored, the same workspace gives the normal result."""
import time

import numpy as np
import pytest

import int4_expert_routing_b200 as F
import synth
from gpu_util import dev_bf16, host_bf16, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer0():
    F.build()
    return F.make_layer(synth.layer_device(0, "cuda"))


def run_decode(L, x, ws, nb):
    B = x.shape[0]
    out = torch().full((B, 2048), 0x1234, dtype=torch().int16, device="cuda")
    F.flint_moe_decode(L, dev_bf16(x), B, out, ws, nb)
    torch().cuda.synchronize()
    return host_bf16(out)


def test_decode_timeout_reports_status_and_recovers(layer0):
    B = 3
    x = synth.decode_x([21, 22, 23])
    nb = F.flint_workspace_bytes(F.FLINT_OP_DECODE, B)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    good = run_decode(layer0, x, ws, nb)
    assert F.flint_read_status(ws) == F.FLINT_OK

    F.flint_workspace_init(ws, nb)
    F.flint_debug_set_wait_polls(0)
    try:
        t0 = time.time()
        failed = run_decode(layer0, x, ws, nb)
        elapsed = time.time() - t0
        status = F.flint_read_status(ws)
    finally:
        F.flint_debug_set_wait_polls(0xFFFFFFFF)
    assert status == F.FLINT_ETIMEOUT
    assert elapsed < 5.0
    assert (failed == np.uint16(0x1234)).all()  # no result was written

    F.flint_workspace_init(ws, nb)
    again = run_decode(layer0, x, ws, nb)
    assert F.flint_read_status(ws) == F.FLINT_OK
    assert np.array_equal(again, good)
