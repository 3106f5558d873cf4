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
