"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

Every test here runs on the CPU.  Each checks the oracle against something
other than itself: values the pages print, hand-computed cases, brute force on
tiny inputs, numpy's fp64 matmul, and invariants of the definition (routing
weights sum to one, selection is invariant to a common bias shift, the block is
linear in the down-projection scales).
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ helpers
def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Independent packer: even element -> low nibble, two's complement."""
    c = np.asarray(codes, np.int64).reshape(-1, 2)
    lo = c[:, 0] & 0xF
    hi = c[:, 1] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_codes(q: np.ndarray) -> np.ndarray:
    """Independent unpacker by arithmetic: ((nibble ^ 8) - 8)."""
    q = np.asarray(q, np.int64)
    lo = ((q & 0xF) ^ 8) - 8
    hi = (((q >> 4) & 0xF) ^ 8) - 8
    return np.stack([lo, hi], axis=-1).reshape(*q.shape[:-1], 2 * q.shape[-1])


def dequant_np(q, s):
    codes = unpack_codes(q).astype(np.float64)
    sc = synth.bf16_to_f64(s)
    return codes * np.repeat(sc, 128, axis=-1)


def bf16(v):
    return synth.bf16_bits(np.asarray(v, np.float64))


def silu(v):
    return v / (1.0 + math.exp(-v))


def sigm(v):
    return 1.0 / (1.0 + math.exp(-v))


def tiny_layer(E=8, H=128, I=128, Is=128, seed=7, k=6):
    dims = synth.Dims(hidden=H, n_experts=E, top_k=k, expert_i=I, shared_i=Is)
    return synth.layer_host(seed, dims), dims


# ------------------------------------------------------------------ format
def test_unpack_every_byte_value():
    q = np.arange(256, dtype=np.uint8)
    codes = oracle.unpack_int4(q).reshape(256, 2)
    for b in range(256):
        lo, hi = b & 15, b >> 4
        assert codes[b, 0] == (lo - 16 if lo >= 8 else lo)
        assert codes[b, 1] == (hi - 16 if hi >= 8 else hi)


def test_pack_unpack_round_trip_all_codes_both_positions():
    codes = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)], np.int8).reshape(-1)
    q = pack_codes(codes)
    assert np.array_equal(oracle.unpack_int4(q), codes)
    assert np.array_equal(pack_codes(oracle.unpack_int4(q)), q)


def test_dequant_is_code_times_group_scale_exactly():
    rng = np.random.default_rng(0)
    q = rng.integers(0, 256, size=(5, 192), dtype=np.uint8)  # K = 384: three groups
    s = bf16(rng.uniform(1e-3, 5e-3, size=(5, 3)))
    W = oracle.dequant(q, s)
    assert np.array_equal(W, dequant_np(q, s))
    # group boundary: element 127 uses scale 0, element 128 uses scale 1
    c = unpack_codes(q)
    sc = synth.bf16_to_f64(s)
    assert W[2, 127] == c[2, 127] * sc[2, 0]
    assert W[2, 128] == c[2, 128] * sc[2, 1]


def test_bf16_rounding_ties_to_even():
    f = oracle.bf16_from_double
    assert f(1.0) == 0x3F80
    assert f(1.0 + 2 ** -8) == 0x3F80            # tie -> even (mantissa 0)
    assert f(1.0 + 3 * 2 ** -8) == 0x3F82        # tie -> even (mantissa 2)
    assert f(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81  # just above the tie
    assert f(-2.0) == 0xC000
    assert f(0.0) == 0x0000
    rng = np.random.default_rng(1)
    v = rng.normal(size=2000) * np.exp(rng.uniform(-20, 20, size=2000))
    assert all(f(x) == int(b) for x, b in zip(v, synth.bf16_bits(v)))


# ------------------------------------------------------------------ GEMV
def test_int4_gemv_matches_numpy_fp64_matmul():
    rng = np.random.default_rng(2)
    N, K, B = 37, 384, 3
    q = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = bf16(rng.uniform(1e-3, 5e-3, size=(N, K // 128)))
    x = bf16(rng.normal(size=(B, K)))
    y, am, gap = oracle.int4_gemv(q, s, x)
    ref = synth.bf16_to_f64(x) @ dequant_np(q, s).T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(am, ref.argmax(axis=1))
    srt = np.sort(ref, axis=1)
    np.testing.assert_allclose(gap, srt[:, -1] - srt[:, -2], rtol=1e-9, atol=1e-15)


def test_int4_gemv_argmax_ties_go_to_lowest_index():
    K = 128
    q = np.zeros((6, K // 2), np.uint8)
    # rows 1 and 4 identical and largest
    q[1, 0] = q[4, 0] = 0x07   # code 7 at element 0
    q[2, 0] = 0x03
    s = np.full((6, 1), bf16(0.5), np.uint16)
    x = np.zeros((1, K), np.uint16)
    x[0, 0] = bf16(1.0)
    y, am, gap = oracle.int4_gemv(q, s, x)
    assert am[0] == 1 and gap[0] == 0.0
    assert y[0, 1] == 3.5 and y[0, 2] == 1.5


# ------------------------------------------------------------------ group-64 affine int4
def fp16(v):
    return np.asarray(v, np.float64).astype(np.float16).view(np.uint16)


def test_fp16_decode_every_finite_bit_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    got = np.array([oracle.fp16_to_double(int(b)) for b in bits[finite]])
    assert np.array_equal(got, ref[finite])
    assert math.isinf(oracle.fp16_to_double(0x7C00)) and math.isnan(oracle.fp16_to_double(0x7E00))


def dequant_affine_np(q, s, m):
    """Independent statement: unsigned nibbles (low = even element) times the
    fp16 scale of the element's 64-group, plus that group's fp16 offset."""
    q = np.asarray(q, np.int64)
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(q.shape[0], -1).astype(np.float64)
    sd = np.repeat(np.asarray(s, np.uint16).view(np.float16).astype(np.float64), 64, axis=1)
    md = np.repeat(np.asarray(m, np.uint16).view(np.float16).astype(np.float64), 64, axis=1)
    return codes * sd + md


def test_affine_hand_case():
    """One row of 128: group 0 has scale 0.5 and offset -1, group 1 scale 0.25
    and offset 2; codes 0..15 then 15..0 in each group (all exact in binary)."""
    codes = np.concatenate([np.arange(64) % 16, 15 - np.arange(64) % 16])
    q = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
    s = fp16([[0.5, 0.25]])
    m = fp16([[-1.0, 2.0]])
    W = oracle.dequant_affine(q, s, m)
    expect = np.concatenate([(np.arange(64) % 16) * 0.5 - 1.0, (15 - np.arange(64) % 16) * 0.25 + 2.0])
    assert np.array_equal(W[0], expect)
    x = np.zeros((1, 128), np.uint16)
    x[0, 3], x[0, 70] = bf16(1.0), bf16(-2.0)   # 3 * 0.5 - 1 = 0.5; -2 * ((15 - 6) * 0.25 + 2) = -8.5
    y, am, gap = oracle.int4_gemv_affine(q, s, m, x)
    assert y[0, 0] == 0.5 - 8.5


def test_affine_gemv_matches_numpy_fp64_matmul():
    rng = np.random.default_rng(12)
    N, K, B = 41, 448, 3
    q = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = fp16(rng.uniform(1e-3, 5e-3, size=(N, K // 64)))
    m = fp16(-rng.uniform(1e-2, 4e-2, size=(N, K // 64)))
    x = bf16(rng.normal(size=(B, K)))
    assert np.array_equal(oracle.dequant_affine(q, s, m), dequant_affine_np(q, s, m))
    y, am, gap = oracle.int4_gemv_affine(q, s, m, x)
    ref = synth.bf16_to_f64(x) @ dequant_affine_np(q, s, m).T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(am, ref.argmax(axis=1))


def test_affine_argmax_ties_go_to_lowest_index():
    K = 64
    q = np.zeros((5, K // 2), np.uint8)
    q[1, 0] = q[3, 0] = 0x0F   # code 15 at element 0
    s = fp16(np.full((5, 1), 0.5))
    m = fp16(np.zeros((5, 1)))
    x = np.zeros((1, K), np.uint16)
    x[0, 0] = bf16(1.0)
    y, am, gap = oracle.int4_gemv_affine(q, s, m, x)
    assert am[0] == 1 and gap[0] == 0.0 and y[0, 1] == 7.5


# ------------------------------------------------------------------ NVFP4
def test_e2m1_values_match_the_published_table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e2m1_values.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_to_double(int(code, 16))
        assert got == float(val) and math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_e4m3_decode_every_code_against_torch():
    import torch
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_double(v) for v in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


def nvfp4_dequant_np(q, s, g):
    """Independent statement: E2M1 value of each nibble (low = even element) from
    the published table, times the E4M3 scale of its 16-block (torch's decoder),
    times the global scale."""
    import torch
    table = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
    q = np.asarray(q, np.int64)
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(q.shape[0], -1)
    sv = torch.from_numpy(np.ascontiguousarray(s, np.uint8)).view(torch.float8_e4m3fn)
    sv = sv.to(torch.float64).numpy()
    return table[codes] * np.repeat(sv, 16, axis=1) * float(np.float32(g))


def test_nvfp4_gemv_matches_numpy_fp64_matmul():
    rng = np.random.default_rng(31)
    N, K, B = 29, 256, 3
    q = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = rng.integers(0x30, 0x70, size=(N, K // 16), dtype=np.uint8)   # finite E4M3 codes
    g = 2.0 ** -9
    x = bf16(rng.normal(size=(B, K)))
    W = oracle.dequant_nvfp4(q, s, g)
    assert np.array_equal(W, nvfp4_dequant_np(q, s, g))
    y, am, gap = oracle.int4_gemv_nvfp4(q, s, g, x)
    ref = synth.bf16_to_f64(x) @ W.T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(am, ref.argmax(axis=1))


def test_nvfp4_hand_case():
    """One row of 32: block 0 scale 2 (E4M3 0x40), block 1 scale 0.25 (0x28);
    global 0.5; x picks element 1 (code 0x3 = 1.5) with 1 and element 17 (code
    0xF = -6) with 0.5: 1.5 * 2 * 0.5 * 1 - 6 * 0.25 * 0.5 * 0.5 = 1.125."""
    q = np.zeros((1, 16), np.uint8)
    q[0, 0] = 0x30          # element 1: 1.5
    q[0, 8] = 0xF0          # element 17: -6
    s = np.array([[0x40, 0x28]], np.uint8)
    x = np.zeros((1, 32), np.uint16)
    x[0, 1], x[0, 17] = bf16(1.0), bf16(0.5)
    y, am, gap = oracle.int4_gemv_nvfp4(q, s, 0.5, x)
    assert y[0, 0] == 1.125


# ------------------------------------------------------------------ routing
def brute_force_topk(b, k):
    """The unique k-subset whose members all rank above every non-member
    (rank: larger score, then lower index)."""
    E = len(b)
    found = []
    for S in itertools.combinations(range(E), k):
        inside = set(S)
        ok = all((b[i] > b[j]) or (b[i] == b[j] and i < j)
                 for i in inside for j in range(E) if j not in inside)
        if ok:
            found.append(S)
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("E", [8, 10, 12])
def test_route_top6_matches_brute_force(E):
    rng = np.random.default_rng(E)
    H = 128
    for trial in range(6):
        t, dims = tiny_layer(E=E, H=H, seed=100 + trial)
        if trial >= 3:   # plant exact ties in the biased score
            t["router_w"][:] = 0
            t["router_b"][:] = np.float32(0.0)
            t["router_b"][[1, 3, 5, 7]] = np.float32(0.25)
        L = oracle.Layer(t)
        x = bf16(rng.normal(size=(3, H)))
        r = oracle.route(L, x)
        for row in range(3):
            sel = brute_force_topk(list(r["biased"][row]), 6)
            assert set(r["idx"][row]) == sel
            # selection order: biased score descending, index ascending on ties
            key = sorted(range(E), key=lambda e: (-r["biased"][row][e], e))
            assert list(r["idx"][row]) == key[:6]
            assert r["gap"][row] == r["biased"][row][key[5]] - r["biased"][row][key[6]]


def test_route_scores_closed_form():
    t, _ = tiny_layer()
    L = oracle.Layer(t)
    x = bf16(np.random.default_rng(3).normal(size=(2, 128)))
    r = oracle.route(L, x)
    Wr = synth.bf16_to_f64(t["router_w"])
    z = synth.bf16_to_f64(x) @ Wr.T
    np.testing.assert_allclose(r["z"], z, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r["sig"], 1 / (1 + np.exp(-z)), rtol=1e-14)
    np.testing.assert_allclose(r["biased"], r["sig"] + t["router_b"].astype(np.float64), rtol=1e-14)


def test_route_weights_positive_and_sum_to_one_full_size():
    L = oracle.Layer(synth.layer_host(0, with_codes=False) | {
        k: np.zeros(1, np.uint8) for k in ("w13_q", "w2_q", "sh13_q", "sh2_q")})
    x = synth.decode_x([0, 1, 2, 3, 4])
    r = oracle.route(L, x)
    assert np.all(r["w"] > 0)
    np.testing.assert_allclose(r["w"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # weights are the unbiased scores of the chosen experts, renormalized
    for row in range(5):
        s = r["sig"][row][r["idx"][row]]
        np.testing.assert_allclose(r["w"][row], s / s.sum(), rtol=1e-15)


def test_route_invariant_to_common_bias_shift_and_bias_zero_is_top_z():
    t, _ = tiny_layer(E=12, seed=9)
    x = bf16(np.random.default_rng(4).normal(size=(4, 128)))
    r0 = oracle.route(oracle.Layer(t), x)
    t2 = dict(t)
    t2["router_b"] = (t["router_b"] + np.float32(0.5)).astype(np.float32)  # exact in fp32 here
    r1 = oracle.route(oracle.Layer(t2), x)
    assert np.array_equal(r0["idx"], r1["idx"])
    np.testing.assert_array_equal(r0["w"], r1["w"])
    t3 = dict(t)
    t3["router_b"] = np.zeros_like(t["router_b"])
    r3 = oracle.route(oracle.Layer(t3), x)
    for row in range(4):   # sigmoid is monotone: top-6 of sigmoid(z) is top-6 of z
        assert list(r3["idx"][row]) == list(np.argsort(-r3["z"][row], kind="stable")[:6])


# ------------------------------------------------------------------ hand case
def test_hand_computed_one_token_eight_experts():
    """1 token, 8 experts, H = I = Is = 128.  Every weight is a small integer
    code times a power-of-two scale; the expected output is written out below
    from the definition: z = W_r x, s = sigmoid(z), selection by s + bias,
    w = s / sum(s) over the chosen six, expert = W2 (silu(W1 x) * W3 x),
    out = sum_j w_j y_j + y_shared."""
    E, H, I = 8, 128, 128
    t, _ = tiny_layer(E=E, H=H, I=I, Is=I)
    for k in ("w13_q", "w2_q", "sh13_q", "sh2_q"):
        t[k] = np.zeros_like(t[k])
    for k in ("w13_s", "w2_s", "sh13_s", "sh2_s"):
        t[k] = np.full_like(t[k], bf16(1.0))
    # router: z_e = Wr[e,0]*1 + Wr[e,1]*0.5
    wr0 = [0.0, 0.5, -0.5, 1.0, -1.0, 0.25, 2.0, -2.0]
    wr1 = [0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 1.0]   # z_7 = -2 + 0.5 = -1.5
    t["router_w"] = np.zeros((E, H), np.uint16)
    t["router_w"][:, 0] = bf16(wr0)
    t["router_w"][:, 1] = bf16(wr1)
    t["router_w"][:, 5] = bf16(3.0)   # multiplies x[5] = 0
    t["router_b"] = np.array([0, 0, 0, -1.0, 0, 0, 0, 1.0], np.float32)
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = bf16(1.0)
    x[0, 1] = bf16(0.5)

    g0 = [1, 2, -1, 3, 0, -2, 1, 2]
    g1 = [2, 0, 1, -1, 1, 2, -2, 2]
    u0 = [3, -1, 2, 1, 1, 1, -3, 2]
    d = [[1, -2, 3], [2, 1, 0], [-1, -1, 1], [4, 0, -4], [1, 1, 1], [0, 2, -2], [3, -3, 1], [-2, 1, 2]]

    def set_expert(q13, s13, q2, s2, gg0, gg1, uu0, dd):
        q13[0, 0] = pack_codes([gg0, gg1])[0]     # gate row 0, elements 0, 1
        s13[0, 0] = bf16(0.25)
        q13[I, 0] = pack_codes([uu0, 0])[0]        # up row 0 (row I), element 0
        s13[I, 0] = bf16(0.5)
        for n in range(3):                          # down rows 0..2, column 0
            q2[n, 0] = pack_codes([dd[n], 0])[0]
            s2[n, 0] = bf16(0.125)
        q2[0, 0] |= pack_codes([0, 5])[0]           # W2[0,1]: multiplies h_1 = 0
        q2[0, 1] = pack_codes([-3, 0])[0]           # W2[0,2]: multiplies h_2 = 0

    for e in range(E):
        set_expert(t["w13_q"][e], t["w13_s"][e], t["w2_q"][e], t["w2_s"][e], g0[e], g1[e], u0[e], d[e])
    set_expert(t["sh13_q"], t["sh13_s"], t["sh2_q"], t["sh2_s"], 2, -1, 1, [1, 0, -1])

    out, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)

    z = [wr0[e] + 0.5 * wr1[e] for e in range(E)]
    s = [sigm(v) for v in z]
    b = [s[e] + [0, 0, 0, -1.0, 0, 0, 0, 1.0][e] for e in range(E)]
    # by hand: b = [.5, .6225, .3775, -.2689, .2689, .5622, .8808, 1.1824]
    assert list(idx[0]) == [7, 6, 1, 5, 0, 2]
    assert gap[0] == pytest.approx(b[2] - b[4], abs=1e-15)
    ssum = sum(s[e] for e in (7, 6, 1, 5, 0, 2))
    expect = np.zeros(H)
    for e in (7, 6, 1, 5, 0, 2):
        g = (g0[e] * 1.0 + g1[e] * 0.5) * 0.25
        u = u0[e] * 0.5
        h0 = silu(g) * u
        for n in range(3):
            expect[n] += (s[e] / ssum) * d[e][n] * 0.125 * h0
    hs = silu((2 * 1.0 - 1 * 0.5) * 0.25) * (1 * 0.5)
    expect[0] += 1 * 0.125 * hs
    expect[2] += -1 * 0.125 * hs
    np.testing.assert_allclose(out[0], expect, rtol=1e-14, atol=1e-17)
    np.testing.assert_allclose(w[0], [s[e] / ssum for e in (7, 6, 1, 5, 0, 2)], rtol=1e-15)


# ------------------------------------------------------------------ layer invariants
def numpy_expert(q13, s13, q2, s2, x):
    W13 = dequant_np(q13, s13)
    I = W13.shape[0] // 2
    g, u = W13[:I] @ x, W13[I:] @ x
    return dequant_np(q2, s2) @ (g / (1 + np.exp(-g)) * u)


def test_expert_matches_numpy_definition():
    t, _ = tiny_layer(E=4, H=256, I=128, Is=256, seed=11)
    x = synth.bf16_to_f64(bf16(np.random.default_rng(5).normal(size=256)))
    for e in range(4):
        y = oracle.swiglu_expert(t["w13_q"][e], t["w13_s"][e], t["w2_q"][e], t["w2_s"][e], x)
        np.testing.assert_allclose(y, numpy_expert(t["w13_q"][e], t["w13_s"][e], t["w2_q"][e],
                                                   t["w2_s"][e], x), rtol=1e-11, atol=1e-14)


def test_identical_experts_make_routing_irrelevant():
    t, _ = tiny_layer(E=10, H=256, I=128, Is=128, seed=12)
    for k in ("w13_q", "w13_s", "w2_q", "w2_s"):
        t[k] = np.ascontiguousarray(np.broadcast_to(t[k][3], t[k].shape))
    x = bf16(np.random.default_rng(6).normal(size=(3, 256)))
    out, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)
    for row in range(3):
        xd = synth.bf16_to_f64(x[row])
        expect = numpy_expert(t["w13_q"][3], t["w13_s"][3], t["w2_q"][3], t["w2_s"][3], xd) + \
            numpy_expert(t["sh13_q"], t["sh13_s"], t["sh2_q"], t["sh2_s"], xd)
        np.testing.assert_allclose(out[row], expect, rtol=1e-11, atol=1e-13)


def test_doubling_down_scales_doubles_output_exactly():
    t, _ = tiny_layer(E=10, H=256, I=128, Is=256, seed=13)
    x = bf16(np.random.default_rng(7).normal(size=(2, 256)))
    out0, idx0, _, _ = oracle.moe_layer(oracle.Layer(t), x)
    t2 = dict(t)
    for k in ("w2_s", "sh2_s"):
        t2[k] = (t[k].astype(np.uint32) + 0x80).astype(np.uint16)   # exponent + 1
    out1, idx1, _, _ = oracle.moe_layer(oracle.Layer(t2), x)
    assert np.array_equal(idx0, idx1)
    assert np.array_equal(out1, 2 * out0)


def test_layer_matches_numpy_definition_random():
    t, _ = tiny_layer(E=16, H=256, I=128, Is=256, seed=14)
    x = bf16(np.random.default_rng(8).normal(size=(3, 256)))
    out, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)
    Wr = synth.bf16_to_f64(t["router_w"])
    for row in range(3):
        xd = synth.bf16_to_f64(x[row])
        z = Wr @ xd
        s = 1 / (1 + np.exp(-z))
        b = s + t["router_b"].astype(np.float64)
        sel = np.lexsort((np.arange(16), -b))[:6]
        assert list(sel) == list(idx[row])
        expect = sum(s[e] / s[sel].sum() * numpy_expert(t["w13_q"][e], t["w13_s"][e], t["w2_q"][e],
                                                         t["w2_s"][e], xd) for e in sel)
        expect = expect + numpy_expert(t["sh13_q"], t["sh13_s"], t["sh2_q"], t["sh2_s"], xd)
        np.testing.assert_allclose(out[row], expect, rtol=1e-10, atol=1e-13)


def dequant_affine_np(q, s, m):
    """Group-64 affine weights from their definition, in numpy: unsigned
    nibbles (low nibble = even element) x fp16 scale + fp16 offset."""
    q = np.asarray(q, np.uint8)
    u = np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1).astype(np.float64)
    sc = np.asarray(s, np.uint16).view(np.float16).astype(np.float64)
    off = np.asarray(m, np.uint16).view(np.float16).astype(np.float64)
    return u * np.repeat(sc, 64, axis=1) + np.repeat(off, 64, axis=1)


def test_affine_layer_matches_numpy_definition_random():
    """The block with group-64 affine experts ("How to Run Flint Locally",
    section "Every build and its size"), against a numpy statement of the
    same definition."""
    dims = synth.Dims(hidden=256, n_experts=16, top_k=6, expert_i=128, shared_i=256)
    t = synth.affine_layer_host(15, dims)
    x = bf16(np.random.default_rng(9).normal(size=(2, 256)))
    out, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)

    def expert(q13, s13, m13, q2, s2, m2, xd):
        W13 = dequant_affine_np(q13, s13, m13)
        I = W13.shape[0] // 2
        g, u = W13[:I] @ xd, W13[I:] @ xd
        return dequant_affine_np(q2, s2, m2) @ (g / (1 + np.exp(-g)) * u)

    for row in range(2):
        xd = synth.bf16_to_f64(x[row])
        s = 1 / (1 + np.exp(-(synth.bf16_to_f64(t["router_w"]) @ xd)))
        sel = np.lexsort((np.arange(16), -(s + t["router_b"].astype(np.float64))))[:6]
        assert list(sel) == list(idx[row])
        expect = sum(s[e] / s[sel].sum() * expert(t["w13_q"][e], t["w13_s"][e], t["w13_m"][e],
                                                  t["w2_q"][e], t["w2_s"][e], t["w2_m"][e], xd)
                     for e in sel)
        expect = expect + expert(t["sh13_q"], t["sh13_s"], t["sh13_m"], t["sh2_q"], t["sh2_s"],
                                 t["sh2_m"], xd)
        np.testing.assert_allclose(out[row], expect, rtol=1e-10, atol=1e-13)


def test_affine_layer_equals_symmetric_layer_exactly():
    """A symmetric layer rewritten in the affine format (codes + 8, each bf16
    scale as two fp16 scales, offsets -8 x scale) has the same weights, so
    the affine block output equals the symmetric one bit for bit."""
    t, _ = tiny_layer(E=8, H=256, I=128, Is=256, seed=23)
    x = bf16(np.random.default_rng(24).normal(size=(3, 256)))
    ref, idx, *_ = oracle.moe_layer(oracle.Layer(t), x)
    got, idx2, *_ = oracle.moe_layer(oracle.Layer(synth.affine_from_symmetric(t)), x)
    assert np.array_equal(got, ref) and np.array_equal(idx, idx2)


def test_nvfp4_layer_matches_numpy_definition_random():
    """The block with NVFP4 experts ("How to Run Flint Locally", section "What
    vLLM changed": NVFP4 weights with BF16 activations): E2M1 codes, E4M3
    scales per 16, a global scale per matrix (gate and up rows each their own),
    against a numpy statement built on the published E2M1 table and torch's
    E4M3 decoder (nvfp4_dequant_np)."""
    dims = synth.Dims(hidden=256, n_experts=16, top_k=6, expert_i=128, shared_i=256)
    t = synth.nvfp4_layer_host(17, dims)
    x = bf16(np.random.default_rng(11).normal(size=(2, 256)))
    out, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)

    def expert(q13, s13, g13, q2, s2, g2, xd):
        I = q13.shape[0] // 2
        Wg = nvfp4_dequant_np(q13[:I], s13[:I], g13[0])
        Wu = nvfp4_dequant_np(q13[I:], s13[I:], g13[1])
        g, u = Wg @ xd, Wu @ xd
        return nvfp4_dequant_np(q2, s2, g2) @ (g / (1 + np.exp(-g)) * u)

    for row in range(2):
        xd = synth.bf16_to_f64(x[row])
        s = 1 / (1 + np.exp(-(synth.bf16_to_f64(t["router_w"]) @ xd)))
        sel = np.lexsort((np.arange(16), -(s + t["router_b"].astype(np.float64))))[:6]
        assert list(sel) == list(idx[row])
        expect = sum(s[e] / s[sel].sum() * expert(t["w13_q"][e], t["w13_s"][e], t["w13_g"][e],
                                                  t["w2_q"][e], t["w2_s"][e], t["w2_g"][e], xd)
                     for e in sel)
        expect = expect + expert(t["sh13_q"], t["sh13_s"], t["sh13_g"], t["sh2_q"], t["sh2_s"],
                                 t["sh2_g"][0], xd)
        np.testing.assert_allclose(out[row], expect, rtol=1e-10, atol=1e-13)


def test_nvfp4_layer_equals_symmetric_layer_exactly():
    """Weights that both formats hold exactly: values in {0, +-1, +-2, +-3,
    +-4, +-6}, as symmetric int4 codes with every bf16 scale 2^-7, and as E2M1
    codes with every E4M3 scale 1.0 and every global scale 2^-7.  The two
    blocks are the same function, so their outputs agree bit for bit."""
    t, dims = tiny_layer(E=8, H=256, I=128, Is=256, seed=27)
    rng = np.random.default_rng(28)
    vals = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    e2m1 = {0: 0x0, 1: 0x2, 2: 0x4, 3: 0x5, 4: 0x6, 6: 0x7}
    sym, nv = dict(t), dict(t)
    for name in ("w13", "w2", "sh13", "sh2"):
        shape = t[name + "_q"].shape
        v = rng.choice(vals, size=shape[:-1] + (2 * shape[-1],))
        sym_nib = (v & 0xF).astype(np.uint8)
        nv_nib = np.vectorize(lambda a: e2m1[abs(a)] | (0x8 if a < 0 else 0))(v).astype(np.uint8)
        sym[name + "_q"] = sym_nib[..., 0::2] | (sym_nib[..., 1::2] << 4)
        nv[name + "_q"] = nv_nib[..., 0::2] | (nv_nib[..., 1::2] << 4)
        ss = t[name + "_s"].shape
        sym[name + "_s"] = np.full(ss, bf16(2.0 ** -7), np.uint16)
        nv[name + "_s"] = np.full(ss[:-1] + (ss[-1] * 8,), 0x38, np.uint8)  # E4M3 1.0 per 16
    E = dims.n_experts
    nv["w13_g"] = np.full((E, 2), 2.0 ** -7, np.float32)
    nv["w2_g"] = np.full(E, 2.0 ** -7, np.float32)
    nv["sh13_g"] = np.full(2, 2.0 ** -7, np.float32)
    nv["sh2_g"] = np.full(1, 2.0 ** -7, np.float32)
    x = bf16(rng.normal(size=(3, 256)))
    ref, idx, *_ = oracle.moe_layer(oracle.Layer(sym), x)
    got, idx2, *_ = oracle.moe_layer(oracle.Layer(nv), x)
    assert np.array_equal(got, ref) and np.array_equal(idx, idx2)


# ------------------------------------------------------------------ stack
def test_interm_div_layer_equals_undivided_layer_exactly():
    """Routed up projections stored / 128 with the routing weights multiplied
    back (TandemLLM "21 Flint" section 21.2, expert_interm_div): every step is
    scaled by a power of two, so the block output equals the undivided one
    exactly; without multiplying back it is not."""
    t, _ = tiny_layer(E=8, H=128, I=128, Is=128, seed=21)
    x = bf16(np.random.default_rng(22).normal(size=(3, 128)))
    ref, idx, w, gap = oracle.moe_layer(oracle.Layer(t), x)
    td = synth.divide_routed_up(t, 7)
    got, idx2, w2, gap2 = oracle.moe_layer(oracle.Layer(td, expert_interm_div=128.0), x)
    assert np.array_equal(got, ref) and np.array_equal(idx, idx2)
    plain, *_ = oracle.moe_layer(oracle.Layer(td), x)
    assert not np.allclose(plain, ref)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_expert_partition_partials_sum_to_the_block(world):
    """Expert parallelism's decomposition: the partials of a partition of the
    experts (the shared expert in one of them) sum to the block output, and a
    shard's partial does not depend on the weights of experts outside it."""
    t, dims = tiny_layer(E=8, H=128, I=128, Is=128, seed=31)
    x = bf16(np.random.default_rng(32).normal(size=(4, 128)))
    L = oracle.Layer(t)
    full, idx, w, gap = oracle.moe_layer(L, x)
    bounds = [r * 8 // world for r in range(world + 1)]
    parts = [oracle.moe_layer_partial(L, x, bounds[r], bounds[r + 1], r == 0) for r in range(world)]
    np.testing.assert_allclose(sum(parts), full, rtol=1e-12, atol=1e-14)
    assert np.array_equal(oracle.moe_layer_partial(L, x, 0, 8, True), full)
    # experts outside shard 0 altered: shard 0's partial is unchanged
    t2 = dict(t)
    t2["w2_s"] = t["w2_s"].copy()
    t2["w2_s"][bounds[1]:] = 0
    assert np.array_equal(oracle.moe_layer_partial(oracle.Layer(t2), x, 0, bounds[1], True), parts[0])


def test_rmsnorm_closed_forms():
    h = np.zeros((2, 4), np.float32)
    h[0] = [3.0, 4.0, 0.0, 0.0]           # mean square 25/4
    h[1] = [-2.0, -2.0, -2.0, -2.0]       # mean square 4
    x = synth.bf16_to_f64(oracle.rmsnorm_bf16(h, eps=1e-6))
    r0 = 1 / math.sqrt(25 / 4 + 1e-6)
    assert x[0, 0] == synth.bf16_to_f64(bf16(3 * r0)) and x[0, 2] == 0.0
    assert x[0, 1] == synth.bf16_to_f64(bf16(4 * r0))
    assert np.all(x[1] == -1.0)           # -2/sqrt(4 + 1e-6) rounds to -1 in bf16


def test_stack_layer_is_norm_then_block_then_fp32_residual():
    t, _ = tiny_layer(E=12, H=256, I=128, Is=128, seed=15)
    L = oracle.Layer(t)
    h = (np.random.default_rng(9).normal(size=(2, 256)) * 3).astype(np.float32)
    hn, idx, w, gap = oracle.stack_layer(L, h, eps=1e-6)
    x = oracle.rmsnorm_bf16(h, 1e-6)
    out, idx2, _, _ = oracle.moe_layer(L, x)
    assert np.array_equal(idx, idx2)
    expect = (h.astype(np.float64) + synth.bf16_to_f64(bf16(out))).astype(np.float32)
    assert np.array_equal(hn, expect)


# ------------------------------------------------------------------ the pages' counts
def test_parameter_counts_match_the_pages():
    d = synth.FLINT
    golden = {}
    for line in open(os.path.join(GOLDEN, "flint_param_counts.txt")):
        if line.strip() and not line.startswith("#"):
            name, value = line.split()[:2]
            golden[name] = int(value)
    expert = 3 * d.hidden * d.expert_i
    # shapes of the packed tensors, in elements (two per byte)
    assert 2 * np.prod(d.w13_q()[1:]) + 2 * np.prod(d.w2_q()[1:]) == expert
    assert round(6 * expert * 47 / 1e5) * 1e5 == golden["routed_active_47_layers"]
    assert round(3 * d.hidden * d.shared_i * 47 / 1e5) * 1e5 == golden["shared_47_layers"]
    assert 2 * np.prod(d.sh13_q()) + 2 * np.prod(d.sh2_q()) == 3 * d.hidden * d.shared_i
    assert round(d.n_experts * d.hidden * 47 / 1e5) * 1e5 == golden["routers_47_layers"]
    assert synth.VOCAB * synth.HIDDEN == golden["lm_head"]
    assert round(expert / 1e5) * 1e5 == golden["routed_expert"]
    assert round(256 * expert / 1e6) * 1e6 == golden["routed_layer"]
    assert round(47 * 256 * expert / 1e8) * 1e8 == golden["routed_all_layers"]
