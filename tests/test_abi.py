"""C ABI of libgdr.so, host side only (no CUDA work is launched): the library
loads, exports every function include/gdr.h declares, its enums match the
binding, and bad requests are rejected before anything reaches the GPU."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_141_b200 import build as gdr_build
from gated_delta_rule_141_b200 import gdr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")


@pytest.fixture(scope="module")
def lib():
    gdr_build.build()
    return gdr.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert declared == sorted(gdr.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_enums_match_header():
    text = open(HEADER).read()
    def val(name):
        return int(re.search(r"\b%s\s*=\s*(\d+)" % name, text).group(1))
    assert [val("GDR_OK"), val("GDR_ERR_ARG"), val("GDR_ERR_SHAPE"), val("GDR_ERR_DTYPE"),
            val("GDR_ERR_ALIGN"), val("GDR_ERR_UNSUPPORTED"), val("GDR_ERR_CUDA"),
            val("GDR_ERR_TIMEOUT"), val("GDR_ERR_NONFINITE")] == list(range(9))
    assert (val("GDR_F32"), val("GDR_BF16")) == (gdr.F32, gdr.BF16)
    assert (val("GDR_GATE_SCALAR"), val("GDR_GATE_GROUP64"), val("GDR_GATE_CHANNEL")) == (
        gdr.GATE_SCALAR, gdr.GATE_GROUP64, gdr.GATE_CHANNEL)
    assert (val("GDR_INV_EXACT"), val("GDR_INV_NEUMANN")) == (gdr.INV_EXACT, gdr.INV_NEUMANN)
    assert (val("GDR_KERNEL_AUTO"), val("GDR_KERNEL_SIMT"), val("GDR_KERNEL_TC")) == (
        gdr.KERNEL_AUTO, gdr.KERNEL_SIMT, gdr.KERNEL_TC)
    # struct layout: 11 ints
    assert ctypes.sizeof(gdr.GdrShape) == 44


def test_status_strings_and_version(lib):
    for s in range(9):
        assert gdr.status_string(s)
    assert gdr.status_string(123) == "unknown status"
    assert gdr.version() >= 100


def _call(shape, ptrs=None, chunk=64, gate=gdr.GATE_SCALAR, inv=gdr.INV_EXACT):
    # fake but 16-byte-aligned device addresses: validation fails before any use
    p = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)] if ptrs is None else ptrs
    return gdr.load().gdr_chunk_fwd(ctypes.byref(shape), p[0], p[1], p[2], p[3], p[4], p[5],
                                    chunk, gate, inv, p[6], p[7], None)


def test_rejects_bad_shapes(lib):
    ok = dict(B=1, T=64, Hk=2, Hv=4, dk=64, dv=64)
    bad = [dict(ok, B=-1), dict(ok, T=-5), dict(ok, Hk=0), dict(ok, Hv=3), dict(ok, dk=0),
           dict(ok, dk=257), dict(ok, dv=300)]
    for kw in bad:
        assert _call(gdr.make_shape(**kw)) == gdr.ERR_SHAPE, kw
    assert _call(gdr.make_shape(**ok), chunk=0) == gdr.ERR_SHAPE
    assert _call(gdr.make_shape(**ok), chunk=129) == gdr.ERR_SHAPE
    # GROUP64 needs dk % 64 == 0
    assert _call(gdr.make_shape(**dict(ok, dk=96)), gate=gdr.GATE_GROUP64) == gdr.ERR_SHAPE
    # Neumann parameters
    assert _call(gdr.make_shape(**ok, neumann_order=-1), inv=gdr.INV_NEUMANN) == gdr.ERR_SHAPE
    assert _call(gdr.make_shape(**ok, neumann_residual_steps=-1),
                 inv=gdr.INV_NEUMANN) == gdr.ERR_SHAPE


def test_rejects_bad_enums_and_dtypes(lib):
    ok = dict(B=1, T=64, Hk=2, Hv=4, dk=64, dv=64)
    assert _call(gdr.make_shape(**ok), gate=7) == gdr.ERR_ARG
    assert _call(gdr.make_shape(**ok), inv=9) == gdr.ERR_ARG
    assert _call(gdr.make_shape(**ok, in_dtype=5)) == gdr.ERR_DTYPE
    assert _call(gdr.make_shape(**ok, out_dtype=5)) == gdr.ERR_DTYPE
    assert _call(gdr.make_shape(**ok, kernel=9)) == gdr.ERR_ARG
    assert gdr.load().gdr_chunk_fwd(None, None, None, None, None, None, None, 64, 0, 0,
                                    None, None, None) == gdr.ERR_ARG


def test_rejects_null_and_misaligned(lib):
    shape = gdr.make_shape(1, 64, 2, 4, 64, 64)
    good = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)]
    for i in (0, 1, 2, 3, 4, 6):   # q k v g beta o are required
        p = list(good)
        p[i] = None
        assert _call(shape, p) == gdr.ERR_ARG, i
    for i in range(8):
        p = list(good)
        p[i] = ctypes.c_void_p(0x10000 * (i + 1) + 4)
        assert _call(shape, p) == gdr.ERR_ALIGN, i


def test_empty_batch_is_a_no_op(lib):
    # B == 0: validated, nothing launched, nothing touched
    assert _call(gdr.make_shape(0, 64, 2, 4, 64, 64), ptrs=[None] * 8) == gdr.OK


def test_kernel_selection(lib):
    bf = gdr.make_shape(4, 4096, 16, 16, 128, 128)
    assert gdr.select_kernel(bf, 64, gdr.GATE_SCALAR) in (gdr.KERNEL_TC, gdr.KERNEL_SIMT)
    f32 = gdr.make_shape(1, 256, 2, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert gdr.select_kernel(f32, 64, gdr.GATE_SCALAR) == gdr.KERNEL_SIMT
    forced = gdr.make_shape(1, 256, 2, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32,
                            kernel="tc")
    assert gdr.select_kernel(forced, 64, gdr.GATE_SCALAR) == -gdr.ERR_UNSUPPORTED
    bad = gdr.make_shape(1, 256, 2, 3, 64, 64)
    assert gdr.select_kernel(bad, 64, gdr.GATE_SCALAR) == -gdr.ERR_SHAPE


def test_kernel_chunk(lib):
    # Exact mode: chunk 128 on the tensor-core kernel blocks by 64 (same function);
    # the Neumann inverse depends on C and keeps the requested blocking.
    kda = gdr.make_shape(2, 8192, 32, 32, 128, 128)
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL) == gdr.KERNEL_TC
    assert gdr.kernel_chunk(kda, 128, gdr.GATE_CHANNEL) == 64
    assert gdr.kernel_chunk(kda, 64, gdr.GATE_CHANNEL) == 64
    assert gdr.kernel_chunk(kda, 128, gdr.GATE_CHANNEL, "neumann") == 128
    simt = gdr.make_shape(1, 256, 2, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert gdr.kernel_chunk(simt, 128, gdr.GATE_SCALAR) == 128
    assert gdr.kernel_chunk(simt, 32, gdr.GATE_SCALAR) == 32
    assert gdr.kernel_chunk(gdr.make_shape(1, 256, 2, 3, 64, 64), 64,
                            gdr.GATE_SCALAR) == -gdr.ERR_SHAPE


def test_host_entry_validates(lib):
    shape = gdr.make_shape(1, 64, 2, 4, 64, 64)
    io = gdr.GdrIO()
    assert gdr.load().gdr_chunk_fwd_host(ctypes.byref(shape), None, ctypes.byref(io), 64, 0, 0,
                                         None) == gdr.ERR_ARG
    assert gdr.load().gdr_chunk_fwd_host(ctypes.byref(shape), ctypes.byref(io),
                                         ctypes.byref(io), 64, 0, 0, None) == gdr.ERR_ARG
