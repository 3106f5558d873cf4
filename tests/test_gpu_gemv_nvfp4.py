"""NVFP4 weight-only GEMV + argmax on the GPU (E2M1 codes, E4M3 scale per 16
elements, fp32 global scale, bf16 activations: the checkpoint format of the
vLLM path in "How to Run Flint Locally", section "What vLLM changed"),
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


def gemv_nvfp4(w, xbits):
    N, K = w["q"].shape[0], 2 * w["q"].shape[1]
    B = xbits.shape[0]
    d = synth.to_device({"q": w["q"], "s": w["s"]}, "cuda")
    y = torch().empty((B, N), dtype=torch().float32, device="cuda")
    am = torch().empty(B, dtype=torch().int32, device="cuda")
    nb = F.flint_gemv_workspace_bytes(N, B)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_int4_gemv_nvfp4(d["q"], d["s"], w["g"], N, K, dev_bf16(xbits), B, y, am, ws, nb)
    torch().cuda.synchronize()
    assert F.flint_read_status(ws) == 0
    return y.cpu().numpy(), am.cpu().numpy()


@pytest.fixture(scope="module")
def head():
    F.build()
    return synth.nvfp4_head_host()


@pytest.mark.parametrize("rows", [[0], [1, 2, 3, 4]])
def test_nvfp4_head_matches_oracle(head, rows):
    x = synth.head_x(rows)
    y, am = gemv_nvfp4(head, x)
    yr, amr, gap = oracle.int4_gemv_nvfp4(head["q"], head["s"], head["g"], x)
    worst = check_close(y, yr, what="nvfp4 logits")
    for b in range(len(rows)):
        if gap[b] >= ARGMAX_GAP:
            assert am[b] == amr[b]
    print(f"nvfp4 head B={len(rows)}: worst |err|/bound {worst:.3e}, "
          f"max |y - oracle| {np.abs(y - yr).max():.3e}")


@pytest.mark.parametrize("N,K,B", [(1007, 384, 3), (16, 128, 8), (5, 2048, 1), (4099, 8192, 2)])
def test_nvfp4_ragged_shapes(N, K, B):
    F.build()
    w = synth.nvfp4_head_host(N, K, seed=N)
    x = np.stack([synth.bf16_bits(synth.normals(700 + r, 93, K)) for r in range(B)])
    y, am = gemv_nvfp4(w, x)
    yr, amr, gap = oracle.int4_gemv_nvfp4(w["q"], w["s"], w["g"], x)
    check_close(y, yr, what=f"nvfp4 {N}x{K}")
    for b in range(B):
        if gap[b] >= ARGMAX_GAP:
            assert am[b] == amr[b]


def test_nvfp4_wide_activation_range():
    """Rows whose largest element is 2^20 and 2^-20 (the per-row f16 shift
    takes each into range): still within the bound."""
    F.build()
    N, K = 512, 1024
    w = synth.nvfp4_head_host(N, K, seed=5)
    base = synth.normals(900, 93, K)
    x = np.stack([synth.bf16_bits(base * 2.0 ** 20), synth.bf16_bits(base * 2.0 ** -20)])
    y, am = gemv_nvfp4(w, x)
    yr, amr, gap = oracle.int4_gemv_nvfp4(w["q"], w["s"], w["g"], x)
    check_close(y, yr, what="nvfp4 wide range")


def test_nvfp4_batch_invariance_bitwise(head):
    x = synth.head_x([7, 8, 9])
    y3, am3 = gemv_nvfp4(head, x)
    for b in range(3):
        y1, am1 = gemv_nvfp4(head, x[b:b + 1])
        assert np.array_equal(y1[0], y3[b]) and am1[0] == am3[b]


def test_nvfp4_argmax_ties_go_to_lowest_row():
    F.build()
    N, K = 1024 + 5, 256
    w = synth.nvfp4_head_host(N, K, seed=78)
    w["q"][:] = 0
    w["s"][:] = 0x68              # one E4M3 scale (96) everywhere
    for r in (9, 400, 1000):
        w["q"][r] = 0x77          # +6 in every element
    x = np.full((1, K), synth.bf16_bits(np.array([1.0]))[0], np.uint16)
    y, am = gemv_nvfp4(w, x)
    assert am[0] == 9
    assert y[0, 9] == y[0, 400] == y[0, 1000] > 0
