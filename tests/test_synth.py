"""The seeded generator: its SplitMix64 core against the published vector, the
host and torch implementations against each other, and the recipe's shapes and
value ranges."""
import os

import numpy as np
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_vector():
    want = [int(l) for l in open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt"))
            if l.strip() and not l.startswith("#")]
    got = [synth._mix64_int(1234567 + i * synth.GAMMA) for i in range(1, 6)]
    assert got == want
    # the numpy path computes the same mixing
    z = (np.uint64(1234567) + np.arange(1, 6, dtype=np.uint64) * np.uint64(synth.GAMMA))
    assert [int(v) for v in synth._mix64_np(z)] == want


def test_counter_based_slices_and_torch_agree():
    full = synth.random_bytes(5, synth.T_W13_Q, 4096)
    assert np.array_equal(synth.random_bytes(5, synth.T_W13_Q, 100, byte_offset=37), full[37:137])
    t = synth.random_bytes_torch(5, synth.T_W13_Q, 4096, "cpu", chunk_words=64)
    assert np.array_equal(t.numpy(), full)
    t2 = synth.random_bytes_torch(5, synth.T_W13_Q, 1024, "cpu", byte_offset=2048)
    assert np.array_equal(t2.numpy(), full[2048:3072])


def test_codes_uniform_over_int4_range():
    b = synth.random_bytes(0, synth.T_HEAD_Q, 1 << 20)
    lo = ((b.astype(np.int64) & 15) ^ 8) - 8
    hist = np.bincount(lo + 8, minlength=16)
    assert hist.min() > 0.97 * (1 << 20) / 16 and hist.max() < 1.03 * (1 << 20) / 16


def test_recipe_value_ranges():
    t = synth.layer_host(0, synth.Dims(n_experts=4), with_codes=False)
    s = synth.bf16_to_f64(t["w13_s"])
    assert s.min() >= 0.02 * 0.5 / 7 * (1 - 2 ** -8) and s.max() <= 0.02 * 1.5 / 7 * (1 + 2 ** -8)
    wr = synth.bf16_to_f64(t["router_w"])
    assert abs(wr.std() - 0.02) < 0.002
    x = synth.bf16_to_f64(synth.decode_x([0]))[0]
    ch = synth.outlier_channels()
    assert len(set(ch.tolist())) == 8
    assert np.abs(x[ch]).mean() > 5 * np.abs(np.delete(x, ch)).mean()
    n = synth.normals(3, 99, 200000)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1) < 0.01


def test_bf16_bits_matches_torch_on_float32_values():
    v = np.random.default_rng(0).normal(size=10000).astype(np.float32)
    ours = synth.bf16_bits(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_expert_slice_equals_full_array_slice():
    d = synth.Dims(n_experts=3)
    t = synth.layer_host(2, d)
    w13, w2 = synth.expert_codes_host(2, 1, d)
    assert np.array_equal(w13, t["w13_q"][1]) and np.array_equal(w2, t["w2_q"][1])


def _e2m1(nib):
    table = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6])
    return table[nib]


def test_affine_and_nvfp4_recipe_value_ranges():
    """The other two formats' synthetic layers hold what their recipes state:
    affine groups roughly centred on zero within the symmetric recipe's
    largest weight (offset -7.5 scale x U(0.9, 1.1)),
    NVFP4 weights within about +-0.055 with an rms near 0.013 (E4M3 block
    scales 64 .. 240, global scales 2^-15 x U(0.75, 1.25))."""
    d = synth.Dims(n_experts=4)
    a = synth.affine_layer_host(1, d)
    s = a["w13_s"].view(np.float16).astype(np.float64)
    m = a["w13_m"].view(np.float16).astype(np.float64)
    assert s.min() > 0.02 * 0.5 / 7.5 * 0.999 and s.max() < 0.02 * 1.5 / 7.5 * 1.001
    assert np.all(m < 0) and np.all(-m / s > 7.5 * 0.9 * 0.999) and np.all(-m / s < 7.5 * 1.1 * 1.001)
    lo, hi = m, m + 15 * s                      # a group's weights lie between these
    mid = np.abs(0.5 * (lo + hi)).max()         # groups roughly centred on zero
    sym_max = 8 * 0.02 * 1.5 / 7                # the symmetric recipe's largest |weight|
    assert np.abs(lo).max() < sym_max and np.abs(hi).max() < sym_max and mid < 0.005
    n = synth.nvfp4_layer_host(1, d)
    sc = n["w13_s"].astype(np.int64)
    assert set(np.unique(sc >> 3).tolist()) <= {13, 14}    # exponent fields, sign 0
    g = n["w13_g"].astype(np.float64)
    assert g.min() >= 2.0 ** -15 * 0.75 and g.max() <= 2.0 ** -15 * 1.25
    q = n["w13_q"][0].astype(np.int64)
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1)
    sv = torch.from_numpy(np.ascontiguousarray(n["w13_s"][0])).view(torch.float8_e4m3fn)
    W = _e2m1(codes) * np.repeat(sv.to(torch.float64).numpy(), 16, axis=1)
    W[:512] *= g[0, 0]
    W[512:] *= g[0, 1]
    assert np.abs(W).max() < 0.056 and 0.012 < np.sqrt((W ** 2).mean()) < 0.015
