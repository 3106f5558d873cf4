"""The exactness facts the NVFP4 kernels rest on, checked on the host over
every case (no GPU).  The kernels' own outputs are checked against the
oracle by the GPU tests; these pin the arithmetic reasons they can be exact:

- an E2M1 value times an E4M3 scale is representable exactly in bf16 (the
  decode's MMA operand) and in fp16 (the prefill's), for every pair of codes;
- an fp16 bit pattern of an E2M1 value, its magnitude bits moved three places
  right and read as bf16, is the value times 2^-112 exactly (zero stays
  zero), and the scale times 2^112 is an exact bf16;
- two masks and a shift-or put the nibble pairs (p, p + 4) of a 32-bit word
  into the low bytes that the hardware conversion reads.
"""
import numpy as np
import torch

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def e4m3_values():
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v[np.isfinite(v)]


def exact_in(v, dtype):
    t = torch.from_numpy(np.asarray(v, np.float64))
    return np.array_equal(t.to(dtype).to(torch.float64).numpy(), np.asarray(v, np.float64))


def test_every_e2m1_times_e4m3_product_is_exact_in_bf16_and_fp16():
    prod = np.outer(E2M1, e4m3_values()).ravel()
    assert exact_in(prod, torch.bfloat16) and exact_in(prod, torch.float16)
    nz = np.abs(prod[prod != 0])
    assert nz.min() == 2.0 ** -10 and nz.max() == 6 * 448   # inside fp16's normal range


def test_fp16_bits_moved_right_read_as_bf16_are_the_value_times_2_to_minus_112():
    h = np.array(E2M1, np.float16).view(np.uint16).astype(np.uint32)
    b = ((h >> 3) & 0x0FFF) | (h & 0x8000)
    got = torch.from_numpy(b.astype(np.uint16).view(np.int16)).view(torch.bfloat16)
    assert np.array_equal(got.to(torch.float64).numpy() * 2.0 ** 112, E2M1)
    s = e4m3_values() * 2.0 ** 112
    assert exact_in(s, torch.bfloat16)


def test_nibble_pairs_land_in_the_low_bytes():
    rng = np.random.default_rng(5)
    for w in rng.integers(0, 2 ** 32, size=2000, dtype=np.uint64).astype(np.uint32):
        n = [(int(w) >> (4 * k)) & 15 for k in range(8)]
        lo, hi = int(w) & 0x0F0F0F0F, (int(w) >> 4) & 0x0F0F0F0F
        X, Y = lo | (lo >> 12), hi | (hi >> 12)
        pairs = [X & 0xFF, Y & 0xFF, (X >> 8) & 0xFF, (Y >> 8) & 0xFF]   # p = 0, 1, 2, 3
        assert pairs == [n[p] | (n[p + 4] << 4) for p in range(4)]
