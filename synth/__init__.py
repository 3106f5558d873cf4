"""Seeded synthetic inputs for the Flint int4 MoE block.

This module is shared by the fp64 oracle (``oracle/``) and the CUDA path
(``int4_expert_routing_b200``).  It holds none of the method's arithmetic: it
only draws random bits and shapes them into the inputs the workloads describe
(bf16 activations and router weights, fp32 router bias, int4 codes as raw
packed bytes, bf16 group scales).  How packed bytes are read back as int4
codes, how a weight is dequantized and everything after that lives on each
side separately.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used as a counter-based generator.  Word i
of stream (seed, tensor_id) is ``mix64(key + (i + 1) * GAMMA)`` with
``key = mix64(mix64(seed) ^ (tensor_id * GAMMA))``, all mod 2**64.  A packed
int4 array is the stream's words written out as little-endian bytes, so every
code is uniform over [-8, 7] and any slice can be drawn on its own.  The same
integer-only definition is implemented twice below: with numpy ``uint64`` on
the host, and with torch ``int64`` ops (wrapping multiply, masked shifts) for
drawing the multi-GB stacked weights straight into device memory.

Floating draws are host-only (numpy fp64): uniform ``u = (w >> 11) * 2**-53``
and one Box-Muller normal per pair of words, ``sqrt(-2 ln(1 - u0)) * cos(2 pi
u1)``.  bf16 values are rounded to nearest-even directly from fp64.

Workload recipe (the Flint MoE layer of "How to Run Flint Locally", section
"The architecture, from config.json": hidden 2,048, 256 routed experts of
size 512, top 6, one shared expert of size 1,024; quantization format:
symmetric int4, group 128 along K, bf16 scale):

* router weight  W_r[256, 2048] bf16 ~ N(0, 0.02^2)
* router bias    b[256] fp32 ~ N(0, 0.1)   (0.1 read as the variance)
* expert codes   uniform in [-8, 7]; scales bf16(0.02 * U(0.5, 1.5) / 7)
* decode input   x[2048] bf16 ~ N(0, 1), 8 fixed outlier channels x 20
* head           W[150144, 2048] int4 with the same scales, x ~ N(0, 1)
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

# Flint MoE layer dimensions.
HIDDEN = 2048
N_EXPERTS = 256
TOP_K = 6
EXPERT_I = 512
SHARED_I = 1024
GROUP = 128
VOCAB = 150144
N_MOE_LAYERS = 47

# Stream ids (the second half of a stream's key).
T_ROUTER_W = 1
T_ROUTER_B = 2
T_W13_Q = 3
T_W13_S = 4
T_W2_Q = 5
T_W2_S = 6
T_SH13_Q = 7
T_SH13_S = 8
T_SH2_Q = 9
T_SH2_S = 10
T_X = 11
T_OUTLIER = 12
T_PREFILL_X = 13
T_RESID = 14
T_HEAD_Q = 20
T_HEAD_S = 21
T_HEAD_X = 22
T_AFF_Q = 30
T_AFF_S = 31
T_AFF_M = 32
T_NV_Q = 33
T_NV_S = 34
T_AFL_W13_S = 40
T_AFL_W13_M = 41
T_AFL_W2_S = 42
T_AFL_W2_M = 43
T_AFL_SH13_S = 44
T_AFL_SH13_M = 45
T_AFL_SH2_S = 46
T_AFL_SH2_M = 47
T_NVL_W13_S = 50
T_NVL_W2_S = 51
T_NVL_SH13_S = 52
T_NVL_SH2_S = 53
T_NVL_G = 54

N_OUTLIERS = 8
OUTLIER_GAIN = 20.0
ROUTER_W_STD = 0.02
ROUTER_B_STD = math.sqrt(0.1)


# ---------------------------------------------------------------- host (numpy)
def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix64_int(_mix64_int(seed) ^ ((tensor_id * GAMMA) & _MASK64))


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def words(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Words start .. start+count-1 of stream (seed, tensor_id), uint64."""
    key = np.uint64(stream_key(seed, tensor_id))
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64_np(key + i * np.uint64(GAMMA))


def random_bytes(seed: int, tensor_id: int, nbytes: int, byte_offset: int = 0) -> np.ndarray:
    """Bytes [byte_offset, byte_offset + nbytes) of the stream, uint8."""
    if nbytes == 0:
        return np.zeros(0, np.uint8)
    w0 = byte_offset // 8
    w1 = (byte_offset + nbytes + 7) // 8
    b = words(seed, tensor_id, w0, w1 - w0).astype("<u8").view(np.uint8)
    lo = byte_offset - 8 * w0
    return np.ascontiguousarray(b[lo:lo + nbytes])


def uniforms(seed: int, tensor_id: int, count: int, start: int = 0) -> np.ndarray:
    w = words(seed, tensor_id, start, count)
    return (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(seed: int, tensor_id: int, count: int, start: int = 0) -> np.ndarray:
    """One Box-Muller normal per pair of words; element i uses words 2i, 2i+1."""
    u = uniforms(seed, tensor_id, 2 * count, 2 * start)
    u0 = u[0::2]
    u1 = u[1::2]
    return np.sqrt(-2.0 * np.log1p(-u0)) * np.cos(2.0 * math.pi * u1)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even); returns uint16 bits."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(m * 256.0), e - 8)  # 8 significant bits, exact in fp64
    f = r.astype(np.float32)                # exact: r has 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def scale_bits(seed: int, tensor_id: int, count: int, start: int = 0) -> np.ndarray:
    """Group scales bf16(0.02 * U(0.5, 1.5) / 7)."""
    u = uniforms(seed, tensor_id, count, start)
    return bf16_bits(0.02 * (0.5 + u) / 7.0)


def fp16_bits(v: np.ndarray) -> np.ndarray:
    """fp16 bit patterns of fp64 values, rounded to nearest-even (numpy's IEEE
    half conversion)."""
    return np.asarray(v, np.float64).astype(np.float16).view(np.uint16)


def affine_head_host(rows: int = VOCAB, hidden: int = HIDDEN, seed: int = 0) -> dict:
    """A group-64 affine int4 matrix [rows, hidden] (the MLX int4 / Q4_1
    layout): unsigned codes uniform in 0..15 (raw random bytes), per 64-group
    fp16 scale 0.02 * U(0.5, 1.5) / 7.5 and fp16 offset -7.5 * scale * U(0.9,
    1.1), so each group spans about [-0.02, 0.02] like the symmetric recipe."""
    g = rows * (hidden // 64)
    sc = 0.02 * (0.5 + uniforms(seed, T_AFF_S, g)) / 7.5
    off = -7.5 * sc * (0.9 + 0.2 * uniforms(seed, T_AFF_M, g))
    return {"q": random_bytes(seed, T_AFF_Q, rows * hidden // 2).reshape(rows, hidden // 2),
            "s": fp16_bits(sc).reshape(rows, hidden // 64),
            "m": fp16_bits(off).reshape(rows, hidden // 64)}


NVFP4_GLOBAL = 2.0 ** -13


def nvfp4_head_host(rows: int = VOCAB, hidden: int = HIDDEN, seed: int = 0) -> dict:
    """An NVFP4 matrix [rows, hidden]: E2M1 codes uniform over the 16 codes
    (raw random bytes), one E4M3 block scale per 16 elements with exponent
    field 13 or 14 and any mantissa (values 64 .. 240), global scale 2^-13: the
    weights span about [-0.18, 0.18]."""
    r = random_bytes(seed, T_NV_S, rows * (hidden // 16)).astype(np.uint32)
    sc = (((13 + (r & 1)) << 3) | ((r >> 1) & 7)).astype(np.uint8)
    return {"q": random_bytes(seed, T_NV_Q, rows * hidden // 2).reshape(rows, hidden // 2),
            "s": sc.reshape(rows, hidden // 16), "g": NVFP4_GLOBAL}


def divide_routed_up(layer: dict, log2_div: int = 7) -> dict:
    """A copy of a layer whose routed experts' up-projection scales (rows I ..
    2I-1 of each expert's gate/up block) are divided by 2^log2_div: the bf16
    exponent field lowered, exact while the scales stay normal."""
    out = dict(layer)
    s = layer["w13_s"].copy()
    I = s.shape[1] // 2
    up = s[:, I:, :].astype(np.int32)
    assert ((up >> 7) & 0xFF).min() > log2_div, "scale would leave the normal range"
    s[:, I:, :] = (up - (log2_div << 7)).astype(np.uint16)
    out["w13_s"] = s
    return out


def divide_routed_up_affine(layer: dict, log2_div: int = 2) -> dict:
    """The affine-format counterpart of ``divide_routed_up``: the routed
    experts' up-projection fp16 scales and offsets (rows I .. 2I-1 of each
    gate/up block) divided by 2^log2_div by lowering their exponent fields,
    exact while they stay normal (zeros stay zero)."""
    out = dict(layer)
    for name in ("w13_s", "w13_m"):
        a = layer[name].copy()
        I = a.shape[1] // 2
        up = a[:, I:, :].astype(np.int32)
        nz = (up & 0x7FFF) != 0
        assert ((up[nz] >> 10) & 0x1F).min() > log2_div, "value would leave the normal range"
        a[:, I:, :] = np.where(nz, up - (log2_div << 10), up).astype(np.uint16)
        out[name] = a
    return out


def outlier_channels(hidden: int = HIDDEN, n: int = N_OUTLIERS) -> np.ndarray:
    """The fixed outlier channels: a partial Fisher-Yates shuffle of 0..hidden-1
    drawn from stream (0, T_OUTLIER); the first n entries, in draw order."""
    perm = np.arange(hidden)
    u = uniforms(0, T_OUTLIER, n)
    for i in range(n):
        j = i + int(u[i] * (hidden - i))
        perm[i], perm[j] = perm[j], perm[i]
    return perm[:n].copy()


def decode_x(seeds, hidden: int = HIDDEN, outliers: bool = True) -> np.ndarray:
    """bf16 bits [len(seeds), hidden]: row r ~ N(0,1) from stream (seeds[r], T_X),
    with the outlier channels multiplied by 20 before rounding."""
    rows = []
    ch = outlier_channels(hidden) if outliers else np.zeros(0, np.int64)
    for s in seeds:
        v = normals(s, T_X, hidden)
        v[ch] *= OUTLIER_GAIN
        rows.append(bf16_bits(v))
    return np.stack(rows).astype(np.uint16)


def prefill_x(T: int, seed: int, hidden: int = HIDDEN) -> np.ndarray:
    """bf16 bits [T, hidden] ~ N(0, 1), one stream (seed, T_PREFILL_X)."""
    return bf16_bits(normals(seed, T_PREFILL_X, T * hidden)).reshape(T, hidden)


def head_x(rows, hidden: int = HIDDEN) -> np.ndarray:
    return np.stack([bf16_bits(normals(r, T_HEAD_X, hidden)) for r in rows]).astype(np.uint16)


def residual_h(seeds, hidden: int = HIDDEN) -> np.ndarray:
    """fp32 [len(seeds), hidden] residual-stream rows for the stacked layers:
    the decode input recipe (outliers included), held in fp32."""
    return bf16_to_f64(decode_x(seeds, hidden)).astype(np.float32)


# ------------------------------------------------------------- layer weights
@dataclass(frozen=True)
class Dims:
    hidden: int = HIDDEN
    n_experts: int = N_EXPERTS
    top_k: int = TOP_K
    expert_i: int = EXPERT_I
    shared_i: int = SHARED_I

    def check(self):
        for v in (self.hidden, self.expert_i, self.shared_i):
            if v % GROUP:
                raise ValueError("every reduction length must be a multiple of 128")

    # shapes of the packed tensors, as (rows, bytes per row) / (rows, groups per row)
    def w13_q(self):
        return (self.n_experts, 2 * self.expert_i, self.hidden // 2)

    def w13_s(self):
        return (self.n_experts, 2 * self.expert_i, self.hidden // GROUP)

    def w2_q(self):
        return (self.n_experts, self.hidden, self.expert_i // 2)

    def w2_s(self):
        return (self.n_experts, self.hidden, self.expert_i // GROUP)

    def sh13_q(self):
        return (2 * self.shared_i, self.hidden // 2)

    def sh13_s(self):
        return (2 * self.shared_i, self.hidden // GROUP)

    def sh2_q(self):
        return (self.hidden, self.shared_i // 2)

    def sh2_s(self):
        return (self.hidden, self.shared_i // GROUP)


FLINT = Dims()


def _n(shape):
    return int(np.prod(shape))


def layer_host(seed: int, dims: Dims = FLINT, with_codes: bool = True) -> dict:
    """All tensors of one MoE layer on the host.

    Gate and up rows of an expert are stacked: rows 0 .. I-1 are the gate
    projection, rows I .. 2I-1 the up projection.  Packed byte j of a row holds
    element 2j in its low nibble and 2j+1 in its high nibble (two's complement).
    With with_codes=False the four code arrays are left out (drawn on the
    device instead, see ``layer_codes_torch``)."""
    dims.check()
    E, H = dims.n_experts, dims.hidden
    d = {
        "router_w": bf16_bits(ROUTER_W_STD * normals(seed, T_ROUTER_W, E * H)).reshape(E, H),
        "router_b": (ROUTER_B_STD * normals(seed, T_ROUTER_B, E)).astype(np.float32),
        "w13_s": scale_bits(seed, T_W13_S, _n(dims.w13_s())).reshape(dims.w13_s()),
        "w2_s": scale_bits(seed, T_W2_S, _n(dims.w2_s())).reshape(dims.w2_s()),
        "sh13_s": scale_bits(seed, T_SH13_S, _n(dims.sh13_s())).reshape(dims.sh13_s()),
        "sh2_s": scale_bits(seed, T_SH2_S, _n(dims.sh2_s())).reshape(dims.sh2_s()),
    }
    if with_codes:
        d["w13_q"] = random_bytes(seed, T_W13_Q, _n(dims.w13_q())).reshape(dims.w13_q())
        d["w2_q"] = random_bytes(seed, T_W2_Q, _n(dims.w2_q())).reshape(dims.w2_q())
        d["sh13_q"] = random_bytes(seed, T_SH13_Q, _n(dims.sh13_q())).reshape(dims.sh13_q())
        d["sh2_q"] = random_bytes(seed, T_SH2_Q, _n(dims.sh2_q())).reshape(dims.sh2_q())
    return d


def _affine_groups(seed: int, tid_s: int, tid_m: int, rows: int, k: int):
    """fp16 scale and offset bits [rows, k/64] of the affine recipe: scale
    0.02 * U(0.5, 1.5) / 7.5, offset -7.5 * scale * U(0.9, 1.1)."""
    g = rows * (k // 64)
    sc = 0.02 * (0.5 + uniforms(seed, tid_s, g)) / 7.5
    off = -7.5 * sc * (0.9 + 0.2 * uniforms(seed, tid_m, g))
    return fp16_bits(sc).reshape(rows, k // 64), fp16_bits(off).reshape(rows, k // 64)


def affine_layer_host(seed: int, dims: Dims = FLINT, with_codes: bool = True) -> dict:
    """A MoE layer whose expert matrices are group-64 affine int4 (the MLX
    int4 / Q4_1 layout): the router as in ``layer_host``; the same packed
    bytes as the symmetric layer of this seed, each nibble read as an unsigned
    code 0..15; per 64 elements along K an fp16 scale and an fp16 offset
    (``_affine_groups``).  Scale and offset arrays are [rows, K/64] per
    matrix (w13_s [E, 2I, H/64], w2_s [E, H, I/64], sh13_s [2Is, H/64],
    sh2_s [H, Is/64]), the offsets under the *_m names."""
    dims.check()
    E, H, I, Is = dims.n_experts, dims.hidden, dims.expert_i, dims.shared_i
    d = layer_host(seed, dims, with_codes=with_codes)
    for name, tid_s, tid_m, rows, k, shape in (
            ("w13", T_AFL_W13_S, T_AFL_W13_M, E * 2 * I, H, (E, 2 * I, H // 64)),
            ("w2", T_AFL_W2_S, T_AFL_W2_M, E * H, I, (E, H, I // 64)),
            ("sh13", T_AFL_SH13_S, T_AFL_SH13_M, 2 * Is, H, (2 * Is, H // 64)),
            ("sh2", T_AFL_SH2_S, T_AFL_SH2_M, H, Is, (H, Is // 64))):
        sc, off = _affine_groups(seed, tid_s, tid_m, rows, k)
        d[name + "_s"], d[name + "_m"] = sc.reshape(shape), off.reshape(shape)
    return d


NVFP4_LAYER_GLOBAL = 2.0 ** -15


def _nvfp4_scales(seed: int, tid: int, rows: int, k: int) -> np.ndarray:
    """E4M3 bytes [rows, k/16] with exponent field 13 or 14 and any mantissa
    (values 64 .. 240), as the NVFP4 head recipe."""
    r = random_bytes(seed, tid, rows * (k // 16)).astype(np.uint32)
    return (((13 + (r & 1)) << 3) | ((r >> 1) & 7)).astype(np.uint8).reshape(rows, k // 16)


def nvfp4_layer_host(seed: int, dims: Dims = FLINT, with_codes: bool = True) -> dict:
    """A MoE layer whose expert matrices are NVFP4 weight-only: the router as
    in ``layer_host``; the same packed bytes as the symmetric layer of this
    seed, each nibble read as an FP4 E2M1 code (uniform over the 16 codes);
    one E4M3 scale per 16 elements along K (values 64 .. 240) as bytes
    [rows, K/16] per matrix (w13_s [E, 2I, H/16], w2_s [E, H, I/16], sh13_s
    [2Is, H/16], sh2_s [H, Is/16]); fp32 global scales 2^-15 x U(0.75, 1.25)
    per expert matrix (w13_g [E, 2]: gate, up; w2_g [E]; sh13_g [2]; sh2_g
    [1]).  Weights span about [-0.055, 0.055], rms about 0.013 (E2M1 rms 2.93 x
    E4M3 rms 148 x 2^-15)."""
    dims.check()
    E, H, I, Is = dims.n_experts, dims.hidden, dims.expert_i, dims.shared_i
    d = layer_host(seed, dims, with_codes=with_codes)
    d["w13_s"] = _nvfp4_scales(seed, T_NVL_W13_S, E * 2 * I, H).reshape(E, 2 * I, H // 16)
    d["w2_s"] = _nvfp4_scales(seed, T_NVL_W2_S, E * H, I).reshape(E, H, I // 16)
    d["sh13_s"] = _nvfp4_scales(seed, T_NVL_SH13_S, 2 * Is, H)
    d["sh2_s"] = _nvfp4_scales(seed, T_NVL_SH2_S, H, Is)
    g = (NVFP4_LAYER_GLOBAL * (0.75 + 0.5 * uniforms(seed, T_NVL_G, 3 * E + 3))).astype(np.float32)
    d["w13_g"] = g[:2 * E].reshape(E, 2)
    d["w2_g"] = g[2 * E:3 * E].copy()
    d["sh13_g"] = g[3 * E:3 * E + 2].copy()
    d["sh2_g"] = g[3 * E + 2:].copy()
    return d


def affine_from_symmetric(t: dict) -> dict:
    """The same weights in the affine format, exactly: code c -> c + 8 (each
    nibble XOR 8), each bf16 scale -> two fp16 scales of the same value (one
    per 64-half of its 128-group), offset -8 x scale.  Both conversions are
    exact for the recipe's scales (normal fp16, 8 significant bits)."""
    out = dict(t)
    for name in ("w13", "w2", "sh13", "sh2"):
        out[name + "_q"] = np.asarray(t[name + "_q"], np.uint8) ^ np.uint8(0x88)
        b = np.asarray(t[name + "_s"], np.uint16).astype(np.uint32) << np.uint32(16)
        sc = np.repeat(b.view(np.float32).astype(np.float64), 2, axis=-1)
        out[name + "_s"] = fp16_bits(sc)
        out[name + "_m"] = fp16_bits(-8.0 * sc)
    return out


def expert_codes_host(seed: int, expert: int, dims: Dims = FLINT):
    """(w13_q[e], w2_q[e]) of one expert, drawn on their own (counter-based)."""
    n13 = 2 * dims.expert_i * dims.hidden // 2
    n2 = dims.hidden * dims.expert_i // 2
    w13 = random_bytes(seed, T_W13_Q, n13, expert * n13).reshape(2 * dims.expert_i, dims.hidden // 2)
    w2 = random_bytes(seed, T_W2_Q, n2, expert * n2).reshape(dims.hidden, dims.expert_i // 2)
    return w13, w2


def head_host(vocab: int = VOCAB, hidden: int = HIDDEN, with_codes: bool = True) -> dict:
    d = {"s": scale_bits(0, T_HEAD_S, vocab * (hidden // GROUP)).reshape(vocab, hidden // GROUP)}
    if with_codes:
        d["q"] = random_bytes(0, T_HEAD_Q, vocab * hidden // 2).reshape(vocab, hidden // 2)
    return d


# ------------------------------------------------------------- device (torch)
def _u64_to_i64(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr_torch(z, s: int):
    """Logical right shift of int64 bits."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64_torch(z):
    z = (z ^ _lsr_torch(z, 30)) * _u64_to_i64(_M1)
    z = (z ^ _lsr_torch(z, 27)) * _u64_to_i64(_M2)
    return z ^ _lsr_torch(z, 31)


def random_bytes_torch(seed: int, tensor_id: int, nbytes: int, device, byte_offset: int = 0,
                       chunk_words: int = 1 << 24):
    """Same bytes as ``random_bytes`` drawn with torch int64 ops on ``device``.
    byte_offset and nbytes must be multiples of 8."""
    import torch
    if nbytes % 8 or byte_offset % 8:
        raise ValueError("torch byte draw needs 8-byte aligned offset and size")
    out = torch.empty(nbytes // 8, dtype=torch.int64, device=device)
    key = _u64_to_i64(stream_key(seed, tensor_id))
    g = _u64_to_i64(GAMMA)
    w0 = byte_offset // 8
    for c0 in range(0, nbytes // 8, chunk_words):
        c1 = min(nbytes // 8, c0 + chunk_words)
        i = torch.arange(w0 + c0 + 1, w0 + c1 + 1, dtype=torch.int64, device=device)
        out[c0:c1] = _mix64_torch(i * g + key)
    return out.view(torch.uint8)


def layer_codes_torch(seed: int, device, dims: Dims = FLINT) -> dict:
    """The four packed code arrays of a layer, drawn on ``device``."""
    return {
        "w13_q": random_bytes_torch(seed, T_W13_Q, _n(dims.w13_q()), device).view(dims.w13_q()),
        "w2_q": random_bytes_torch(seed, T_W2_Q, _n(dims.w2_q()), device).view(dims.w2_q()),
        "sh13_q": random_bytes_torch(seed, T_SH13_Q, _n(dims.sh13_q()), device).view(dims.sh13_q()),
        "sh2_q": random_bytes_torch(seed, T_SH2_Q, _n(dims.sh2_q()), device).view(dims.sh2_q()),
    }


def to_device(arrays: dict, device) -> dict:
    """Upload a dict of host arrays to ``device`` as torch tensors holding the
    same bytes (uint16 travels as int16, uint8 as uint8)."""
    import torch
    out = {}
    for k, v in arrays.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(device)
    return out


def nvfp4_layer_device(seed: int, device, dims: Dims = FLINT) -> dict:
    """``nvfp4_layer_host`` on ``device``, the codes drawn on the device."""
    d = to_device(nvfp4_layer_host(seed, dims, with_codes=False), device)
    d.update(layer_codes_torch(seed, device, dims))
    return d


def affine_layer_device(seed: int, device, dims: Dims = FLINT) -> dict:
    """``affine_layer_host`` on ``device``, the codes drawn on the device."""
    d = to_device(affine_layer_host(seed, dims, with_codes=False), device)
    d.update(layer_codes_torch(seed, device, dims))
    return d


def layer_device(seed: int, device, dims: Dims = FLINT, host: dict | None = None) -> dict:
    """A layer's tensors on ``device``.  With ``host`` (from layer_host with
    codes) the bytes are uploaded; otherwise the codes are drawn on the device
    and only the floating tensors are drawn on the host."""
    if host is not None:
        return to_device(host, device)
    d = to_device(layer_host(seed, dims, with_codes=False), device)
    d.update(layer_codes_torch(seed, device, dims))
    return d
