"""The oracle's pins reject plausible mistakes.

Each case plants one mistake in a copy of ``oracle.c``: a wrong nibble sign or
order, a wrong scale group, a sign error in the sigmoid, the bias added before
it, biased or unnormalized weights, the wrong tie order, gate and up swapped, a
dropped shared expert or activation, RMSNorm without the mean, a residual
without the bf16 block output, a transposed router, truncating bf16 rounding,
the head's ties to the highest row.  It builds the copy with gcc into a
temporary directory, loads it in place of the oracle library, and runs the
pins of ``test_oracle.py`` against it: at least one must fail.  Nothing here
touches the oracle's own source or library.  CPU only.
"""
import inspect
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# name -> [(text in oracle.c, replacement)]; every text occurs exactly once,
# and every mutant keeps its indexes inside the arrays it reads
MUTANTS = {
    "affine layer read as symmetric": [("else if (m->fmt[j] == 1)", "else if (0)")],
    "affine layer with 128-groups": [("const int gs = aff ? 64 : (nv ? 16 : 128)",
                                      "const int gs = aff ? 128 : (nv ? 16 : 128)")],
    "nvfp4 layer read as symmetric": [("if (m->fmt[j] == 2)", "if (0)")],
    "nvfp4 down global from gate/up": [("nv ? (double)L->w2_g[e] : 0.0",
                                        "nv ? (double)L->w13_g[e] : 0.0")],
    "nvfp4 up rows with the gate's global scale": [
        ("NULL, (double)gl[1], inter, H, xd, g + go + inter);",
         "NULL, (double)gl[0], inter, H, xd, g + go + inter);")],
    "nvfp4 gate/up global scales of the wrong expert": [
        ("const float *gl = j < k ? L->w13_g + 2 * e : L->sh13_g;",
         "const float *gl = j < k ? L->w13_g + e : L->sh13_g;")],
    "affine down offsets from gate/up": [("aff ? L->w2_m + g2 : NULL", "aff ? L->w13_m + g2 : NULL")],
    "nibble as offset binary": [("return nib >= 8 ? nib - 16 : nib;", "return nib - 8;")],
    "nibble order swapped": [("int nib = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);",
                              "int nib = (k % 2 == 0) ? (byte >> 4) : (byte & 0x0F);")],
    "scale group of 64": [("s[n * (K / 128) + k / 128]", "s[n * (K / 128) + (k / 64) % (K / 128)]")],
    "scale ignored": [("return (double)code_of(row, k) * scale;",
                       "(void)scale;\n  return (double)code_of(row, k);")],
    "sigmoid sign": [("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));")],
    "bias inside the sigmoid": [("biased[e] = sig[e] + (double)L->router_b[e];",
                                 "biased[e] = sigmoid(acc + (double)L->router_b[e]);")],
    "weights from biased scores": [("ssum += sig[order[j]];", "ssum += biased[order[j]];"),
                                   ("w[j] = sig[order[j]] / ssum;", "w[j] = biased[order[j]] / ssum;")],
    "weights not normalized": [("w[j] = sig[order[j]] / ssum;", "w[j] = sig[order[j]];")],
    "ties to the higher expert": [("(bi == bj && i < j)", "(bi == bj && i > j)")],
    "router transposed": [("L->router_w[(int64_t)e * H + h]", "L->router_w[(int64_t)h * E + e]")],
    "gate and up swapped": [("hmid[r] = g[r] * sigmoid(g[r]) * g[inter + r];",
                             "hmid[r] = g[inter + r] * sigmoid(g[inter + r]) * g[r];")],
    "activation dropped": [("hmid[r] = g[r] * sigmoid(g[r]) * g[inter + r];",
                            "hmid[r] = g[r] * g[inter + r];")],
    "shared expert dropped": [("for (int n = 0; n < H; ++n) out[n] += ys[(size_t)H * k + n];",
                               "(void)0;")],
    "rmsnorm without the mean": [("1.0 / sqrt(ss / H + eps)", "1.0 / sqrt(ss + eps)")],
    "residual adds the fp64 block output": [
        ("double o = oracle_bf16_to_double(oracle_double_to_bf16(out[i]));", "double o = out[i];")],
    "bf16 rounding truncates": [("nearbyint(m * 256.0)", "trunc(m * 256.0)")],
    "head ties to the highest row": [("if (yb[n] > yb[best]) best = n;",
                                      "if (yb[n] >= yb[best]) best = n;")],
    "affine codes read as signed": [("return (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);",
                                     "return ((k % 2 == 0) ? (byte & 0x0F) : (byte >> 4)) ^ 8;")],
    "affine offset dropped": [("oracle_fp16_to_double(s[g]) +\n         oracle_fp16_to_double(m[g]);",
                               "oracle_fp16_to_double(s[g]);")],
    "affine group of 128": [("const int64_t g = n * (K / 64) + k / 64;",
                             "const int64_t g = n * (K / 64) + (k / 128) % (K / 64);")],
    "affine scale and offset swapped": [
        ("(double)ucode_of(q + n * (K / 2), k) * oracle_fp16_to_double(s[g]) +\n         oracle_fp16_to_double(m[g]);",
         "(double)ucode_of(q + n * (K / 2), k) * oracle_fp16_to_double(m[g]) +\n         oracle_fp16_to_double(s[g]);")],
    "interm_div not multiplied back": [("out[n] += (w[j] * div) * ys[(size_t)H * j + n];",
                                        "out[n] += w[j] * ys[(size_t)H * j + n];")],
    "e2m1 exponent bias 0": [("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)")],
    "e4m3 exponent bias 8": [("mag = ldexp(1.0 + m / 8.0, e - 7);", "mag = ldexp(1.0 + m / 8.0, e - 8);")],
    "nvfp4 scale block of 32": [("s[n * (K / 16) + k / 16]", "s[n * (K / 16) + (k / 32) % (K / 16)]")],
    "nvfp4 global scale dropped": [("oracle_e4m3_to_double(s[n * (K / 16) + k / 16]) * global;",
                                    "oracle_e4m3_to_double(s[n * (K / 16) + k / 16]);")],
    "fp16 exponent bias 16": [("mag = ldexp((double)(1024 + f), e - 25);", "mag = ldexp((double)(1024 + f), e - 26);")],
}


def _pin_calls():
    """(name, zero-argument call) for every pin in test_oracle.py."""
    calls = []
    for name, fn in vars(pins).items():
        if not name.startswith("test_") or not callable(fn):
            continue
        params = list(inspect.signature(fn).parameters)
        if not params:
            calls.append((name, fn))
        else:  # the parametrized brute-force pin: every expert count it lists
            for mark in getattr(fn, "pytestmark", []):
                if mark.name == "parametrize":
                    for v in mark.args[1]:
                        calls.append((f"{name}[{v}]", lambda fn=fn, v=v: fn(v)))
    return calls


def _build_mutant(tmp_path, edits):
    text = open(SRC).read()
    for old, new in edits:
        assert text.count(old) == 1, old
        text = text.replace(old, new)
    src = tmp_path / "oracle_mutant.c"
    src.write_text(text)
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread",
                           "-ffp-contract=off", "-fno-fast-math",
                           "-I", os.path.dirname(SRC), str(src), "-o", str(so), "-lm"])
    return str(so)


def test_every_pin_passes_on_the_oracle_itself():
    failed = []
    for name, call in _pin_calls():
        try:
            call()
        except Exception as e:  # noqa: BLE001 - any failure counts
            failed.append((name, repr(e)[:120]))
    assert not failed, failed


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_planted_mistake(mutant, tmp_path, monkeypatch):
    so = _build_mutant(tmp_path, MUTANTS[mutant])
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "build", lambda force=False: so)
    caught = []
    for name, call in _pin_calls():
        try:
            call()
        except Exception:  # noqa: BLE001 - an assertion or a shape/value error both catch it
            caught.append(name)
            break
    assert caught, f"no pin rejects the planted mistake: {mutant}"
