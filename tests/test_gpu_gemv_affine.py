"""Group-64 affine int4 GEMV + argmax on the GPU (the MLX int4 / Q4_1 weight
format of "How to Run Flint Locally", section "Every build and its size"),
through the C ABI, against the fp64 oracle: the 150,144 x 2,048 head shape and
ragged ones."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import check_close, dev_bf16, torch

pytestmark = pytest.mark.gpu

ARGMAX_GAP = 1e-5


def gemv_affine(w, xbits):
    N, K = w["q"].shape[0], 2 * w["q"].shape[1]
    B = xbits.shape[0]
    d = synth.to_device({"q": w["q"], "s": w["s"], "m": w["m"]}, "cuda")
    y = torch().empty((B, N), dtype=torch().float32, device="cuda")
    am = torch().empty(B, dtype=torch().int32, device="cuda")
    nb = F.flint_gemv_workspace_bytes(N, B)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_int4_gemv_affine(d["q"], d["s"], d["m"], N, K, dev_bf16(xbits), B, y, am, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return y.cpu().numpy(), am.cpu().numpy()


@pytest.fixture(scope="module")
def head():
    F.build()
    return synth.affine_head_host()


@pytest.mark.parametrize("rows", [[0], [1, 2, 3, 4]])
def test_affine_head_matches_oracle(head, rows):
    x = synth.head_x(rows)
    y, am = gemv_affine(head, x)
    yr, amr, gap = oracle.int4_gemv_affine(head["q"], head["s"], head["m"], x)
    worst = check_close(y, yr, what="affine logits")
    for b in range(len(rows)):
        if gap[b] >= ARGMAX_GAP:
            assert am[b] == amr[b]
    print(f"affine head B={len(rows)}: worst |err|/bound {worst:.3e}, "
          f"max |y - oracle| {np.abs(y - yr).max():.3e}")


@pytest.mark.parametrize("N,K,B", [(1007, 384, 3), (16, 128, 8), (5, 2048, 1), (4099, 8192, 2)])
def test_affine_ragged_shapes(N, K, B):
    F.build()
    w = synth.affine_head_host(N, K, seed=N)
    x = np.stack([synth.bf16_bits(synth.normals(500 + r, 93, K)) for r in range(B)])
    y, am = gemv_affine(w, x)
    yr, amr, gap = oracle.int4_gemv_affine(w["q"], w["s"], w["m"], x)
    check_close(y, yr, what=f"affine {N}x{K}")
    for b in range(B):
        if gap[b] >= ARGMAX_GAP:
            assert am[b] == amr[b]


def test_affine_batch_invariance_bitwise(head):
    x = synth.head_x([7, 8, 9])
    y3, am3 = gemv_affine(head, x)
    for b in range(3):
        y1, am1 = gemv_affine(head, x[b:b + 1])
        assert np.array_equal(y1[0], y3[b]) and am1[0] == am3[b]


def test_affine_argmax_ties_go_to_lowest_row():
    """Rows 3, 70 and 1000 identical and the largest: the lowest wins."""
    F.build()
    N, K = 1024 + 7, 256
    w = synth.affine_head_host(N, K, seed=77)
    w["q"][:] = 0
    for r in (3, 70, 1000):
        w["q"][r] = 0xFF
    w["s"][:] = synth.fp16_bits(0.01)
    w["m"][:] = synth.fp16_bits(0.0)
    x = np.full((1, K), synth.bf16_bits(np.array([1.0]))[0], np.uint16)
    y, am = gemv_affine(w, x)
    assert am[0] == 3
    assert y[0, 3] == y[0, 70] == y[0, 1000]
