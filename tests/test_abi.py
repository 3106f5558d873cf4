"""The C ABI library without a GPU: it loads, exports every entry point the
header declares, and rejects bad arguments before touching the device."""
import os
import re

import pytest

import int4_expert_routing_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    F.build()
    return F.lib()


def declared_entry_points():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"FLINT_API\s+[\w\s\*]*?\b(flint_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(F.EXPORTS)


def test_bounds_checked_build_exports_the_same_symbols():
    """libflint_debug.so (FLINT_DEBUG) is the same ABI: it builds from the same
    sources and exports every declared entry point; its argument checks are
    the release library's."""
    F.build(debug=True)
    with F.using_library(F.DEBUG_LIB_PATH) as dbg:
        for n in declared_entry_points():
            assert hasattr(dbg, n), n
        assert F.lib() is dbg and F.version() >= 100
        with pytest.raises(F.FlintError) as e:
            F.flint_int4_gemv(1 << 20, 1 << 20, 16, 100, 1 << 20, 1, 1 << 20, None, 1 << 20,
                              1 << 20, stream=0)
        assert e.value.code == F.FLINT_EINVAL
    assert F.lib()._name == F.LIB_PATH  # the default library again


def test_decode_batch_limit_per_format_before_launch(lib):
    """B = 8 is refused for affine and NVFP4 layers (their down slots do not
    fit 48 in K3's shared memory) by every decode call, before any launch;
    the symmetric format's limit is 8, and B = 9 is refused for all."""
    fake = 1 << 20
    nb = F.flint_workspace_bytes(F.FLINT_OP_DECODE, 8)
    for fmt in (F.FLINT_FMT_AFFINE_INT4, F.FLINT_FMT_NVFP4):
        L = F.flint_moe_layer(*([fake] * 10), 0, fmt, *([fake] * 8))
        for call in (lambda: F.flint_moe_decode(L, fake, 8, fake + 65536, fake, nb, stream=0),
                     lambda: F.flint_moe_decode_residual(L, fake, 8, None, None, fake, nb,
                                                         stream=0)):
            with pytest.raises(F.FlintError) as e:
                call()
            assert e.value.code == F.FLINT_EINVAL
    for fmt in (F.FLINT_FMT_SYM_INT4, F.FLINT_FMT_AFFINE_INT4, F.FLINT_FMT_NVFP4):
        L = F.flint_moe_layer(*([fake] * 10), 0, fmt, *([fake] * 8))
        with pytest.raises(F.FlintError) as e:
            F.flint_moe_decode(L, fake, 9, fake + 65536, fake, 1 << 24, stream=0)
        assert e.value.code == F.FLINT_EINVAL


def test_using_library_restores_the_default_after_an_error():
    """An error raised inside the block still leaves the default library
    selected afterwards."""
    F.build(debug=True)
    with pytest.raises(F.FlintError):
        with F.using_library(F.DEBUG_LIB_PATH):
            F.flint_moe_route(F.flint_moe_layer(), 1 << 20, 1, None, None, 1 << 20, 1 << 20,
                              stream=0)
    assert F.lib()._name == F.LIB_PATH


def test_version_and_strerror(lib):
    assert F.version() >= 100
    assert "invalid" in F.strerror(F.FLINT_EINVAL)
    assert F.strerror(99) == "unknown flint status"


def test_workspace_sizes(lib):
    assert F.flint_workspace_bytes(F.FLINT_OP_DECODE, 0) == 0
    assert F.flint_workspace_bytes(F.FLINT_OP_DECODE, 9) == 0
    s1 = F.flint_workspace_bytes(F.FLINT_OP_DECODE, 1)
    s8 = F.flint_workspace_bytes(F.FLINT_OP_DECODE, 8)
    assert 0 < s1 < s8 and s8 % 256 == 0
    assert F.flint_gemv_workspace_bytes(150144, 4) > 256
    assert F.flint_gemv_workspace_bytes(150144, 9) == 0


def test_bad_arguments_rejected_before_launch(lib):
    layer = F.flint_moe_layer()                      # all NULL
    fake = 1 << 20                                   # aligned, never dereferenced
    with pytest.raises(F.FlintError) as e:
        F.flint_moe_decode(layer, fake, 1, fake, fake, 1 << 20, stream=0)
    assert e.value.code == F.FLINT_EINVAL
    good = F.flint_moe_layer(*([fake] * 10))
    for B in (0, 9):
        with pytest.raises(F.FlintError):
            F.flint_moe_decode(good, fake, B, fake + 4096, fake, 1 << 20, stream=0)
    with pytest.raises(F.FlintError):                # misaligned x
        F.flint_moe_decode(good, fake + 2, 1, fake + 4096, fake, 1 << 20, stream=0)
    with pytest.raises(F.FlintError):                # workspace too small
        F.flint_moe_decode(good, fake, 1, fake + 4096, fake, 64, stream=0)
    with pytest.raises(F.FlintError):                # x aliases out
        F.flint_moe_decode(good, fake, 1, fake, fake + 8192, 1 << 20, stream=0)
    with pytest.raises(F.FlintError):                # K not a multiple of 128
        F.flint_int4_gemv(fake, fake, 16, 100, fake, 1, fake, None, fake, 1 << 20, stream=0)
    with pytest.raises(F.FlintError):
        F.flint_moe_route(good, fake, 1, None, fake, fake, 1 << 20, stream=0)
    with pytest.raises(F.FlintError):
        F.flint_workspace_init(fake + 8, 16, stream=0)


def test_weight_format_rejected_before_launch(lib):
    """An unknown expert format, an affine layer without its offsets (or
    with a misaligned one) and an NVFP4 layer without its global scales (or
    with a misaligned one) are refused on the host, by decode and prefill."""
    fake = 1 << 20
    for fmt, offs in ((3, [fake] * 8), (-1, [fake] * 8), (1, [None] * 8),
                      (1, [fake, fake + 2, fake, fake] + [None] * 4),
                      (2, [fake] * 4 + [None] * 4), (2, [None] * 4 + [fake, fake + 2, fake, fake])):
        bad = F.flint_moe_layer(*([fake] * 10), 0, fmt, *offs)
        with pytest.raises(F.FlintError) as e:
            F.flint_moe_decode(bad, fake, 1, fake + 4096, fake, 1 << 20, stream=0)
        assert e.value.code == F.FLINT_EINVAL
    nb = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, 16)
    for fmt, offs in ((1, [fake, fake, None, fake]), (1, [fake, fake, fake, fake + 8]),
                      (2, [None] * 4 + [fake, None, fake, fake]),
                      (2, [None] * 4 + [fake, fake, fake + 1, fake])):
        bad = F.flint_moe_layer(*([fake] * 10), 0, fmt, *offs)
        with pytest.raises(F.FlintError) as e:
            F.flint_moe_prefill(bad, fake, 16, fake + (1 << 24), fake, nb, stream=0)
        assert e.value.code == F.FLINT_EINVAL
