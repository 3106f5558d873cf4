"""Int4 GEMV + argmax on the GPU (the 150,144 x 2,048 output head and ragged
shapes), through the C ABI, against the fp64 oracle."""
import numpy as np
import pytest

import int4_expert_routing_b200 as F
import oracle
import synth
from gpu_util import check_close, dev_bf16, torch

pytestmark = pytest.mark.gpu

# Rows whose oracle top-1/top-2 gap is below this are excluded from the exact
# argmax check (fp32 accumulation error of a 2,048-term sum at these
# magnitudes is ~1e-6).
ARGMAX_GAP = 1e-5


def gemv(q, s, xbits, N, K):
    B = xbits.shape[0]
    qd = torch().from_numpy(np.ascontiguousarray(q)).cuda()
    sd = torch().from_numpy(np.ascontiguousarray(s).view(np.int16)).cuda()
    x = dev_bf16(xbits)
    y = torch().empty((B, N), dtype=torch().float32, device="cuda")
    am = torch().empty(B, dtype=torch().int32, device="cuda")
    nb = F.flint_gemv_workspace_bytes(N, B)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")
    F.flint_workspace_init(ws, nb)
    F.flint_int4_gemv(qd, sd, N, K, x, B, y, am, ws, nb)
    torch().cuda.synchronize()
    return y.cpu().numpy(), am.cpu().numpy()


@pytest.fixture(scope="module")
def head():
    F.build()
    return synth.head_host()


@pytest.mark.parametrize("rows", [[0], [0, 1, 2, 3]])
def test_head_gemv_matches_oracle(head, rows):
    x = synth.head_x(rows)
    y, am = gemv(head["q"], head["s"], x, synth.VOCAB, synth.HIDDEN)
    ref, ram, gap = oracle.int4_gemv(head["q"], head["s"], x)
    check_close(y, ref, what="logits")
    for b in range(len(rows)):
        if gap[b] < ARGMAX_GAP:
            print(f"row {b}: top-1/top-2 gap {gap[b]:.3e}: argmax excluded")
            continue
        assert am[b] == ram[b]
    print("max |y - oracle|:", float(np.max(np.abs(y - ref))))


def test_head_batch_invariance(head):
    x = synth.head_x([0, 1, 2, 3])
    y4, a4 = gemv(head["q"], head["s"], x, synth.VOCAB, synth.HIDDEN)
    for b in range(4):
        y1, a1 = gemv(head["q"], head["s"], x[b:b + 1], synth.VOCAB, synth.HIDDEN)
        assert np.array_equal(y4[b], y1[0]) and a4[b] == a1[0]


# K = 512, 1,024 and 2,048 take the kernel that holds the activation fragment
# in registers (with full tiles and a ragged last tile); the others the
# shared-memory fragment
@pytest.mark.parametrize("N,K,B", [(1007, 384, 3), (16, 128, 8), (5, 2048, 1), (4099, 8192, 2),
                                   (1000, 512, 2), (2049, 1024, 5), (3001, 2048, 8)])
def test_ragged_shapes(N, K, B):
    q = synth.random_bytes(N, 77, N * K // 2).reshape(N, K // 2)
    s = synth.scale_bits(N, 78, N * K // 128).reshape(N, K // 128)
    x = np.stack([synth.bf16_bits(synth.normals(r, 79, K)) for r in range(B)])
    y, am = gemv(q, s, x, N, K)
    ref, ram, gap = oracle.int4_gemv(q, s, x)
    check_close(y, ref, what="y")
    for b in range(B):
        if gap[b] >= ARGMAX_GAP:
            assert am[b] == ram[b]


def test_argmax_ties_go_to_lowest_row():
    N, K = 4000, 256
    q = np.zeros((N, K // 2), np.uint8)
    s = np.full((N, K // 128), synth.bf16_bits(np.array([0.5]))[0], np.uint16)
    for r in (3001, 17, 2500):          # three identical maxima
        q[r, 0] = 0x07
    q[100, 0] = 0x05
    x = np.zeros((2, K), np.uint16)
    x[:, 0] = synth.bf16_bits(np.array([1.0]))[0]
    y, am = gemv(q, s, x, N, K)
    assert list(am) == [17, 17]
    assert y[0, 17] == 3.5 and y[0, 100] == 2.5


def test_gemv_timeout_reports_status_and_recovers():
    """The GEMV's timeout path, driven without a GPU fault: with the first-wait
    bound lowered to zero every CTA gives up at once, records FLINT_ETIMEOUT in
    the workspace status word and returns after the copies it issued have
    landed; with the bound restored the same workspace gives the normal,
    bitwise-equal result."""
    import time
    F.build()
    N, K, B = 150144, 2048, 2
    q = synth.random_bytes_torch(0, synth.T_HEAD_Q, N * K // 2, "cuda").view(N, K // 2)
    s = synth.to_device({"s": synth.head_host(with_codes=False)["s"]}, "cuda")["s"]
    x = synth.to_device({"x": synth.head_x([0, 1])}, "cuda")["x"]
    nb = F.flint_gemv_workspace_bytes(N, B)
    ws = torch().zeros(nb, dtype=torch().uint8, device="cuda")

    def call():
        F.flint_workspace_init(ws, nb)
        y = torch().full((B, N), 7.0, dtype=torch().float32, device="cuda")
        am = torch().full((B,), -7, dtype=torch().int32, device="cuda")
        F.flint_int4_gemv(q, s, N, K, x, B, y, am, ws, nb)
        torch().cuda.synchronize()
        return y.cpu().numpy(), am.cpu().numpy(), F.flint_read_status(ws)

    y0, am0, st0 = call()
    assert st0 == F.FLINT_OK
    F.flint_debug_set_wait_polls(0)
    try:
        t0 = time.time()
        y1, am1, st1 = call()
        elapsed = time.time() - t0
    finally:
        F.flint_debug_set_wait_polls(0xFFFFFFFF)
    assert st1 == F.FLINT_ETIMEOUT
    assert elapsed < 5.0
    assert (am1 == -7).all() and (y1 == 7.0).all()   # nothing written
    y2, am2, st2 = call()
    assert st2 == F.FLINT_OK
    assert np.array_equal(y2, y0) and np.array_equal(am2, am0)
