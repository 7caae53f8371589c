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
            val("GDR_ERR_TIMEOUT"), val("GDR_ERR_NONFINITE"), val("GDR_ERR_WORKSPACE"),
            val("GDR_ERR_SCRATCH_LIMIT")] == list(range(11))
    assert int(re.search(r"GDR_STATIC_SCRATCH_BYTES \((\d+)u \* 1024u \* 1024u\)", text).group(1)) \
        * 1024 * 1024 == gdr.STATIC_SCRATCH_BYTES
    assert val("GDR_ERR_WORKSPACE") == gdr.ERR_WORKSPACE
    assert (val("GDR_F32"), val("GDR_BF16")) == (gdr.F32, gdr.BF16)
    assert (val("GDR_GATE_SCALAR"), val("GDR_GATE_GROUP64"), val("GDR_GATE_CHANNEL")) == (
        gdr.GATE_SCALAR, gdr.GATE_GROUP64, gdr.GATE_CHANNEL)
    assert (val("GDR_INV_EXACT"), val("GDR_INV_NEUMANN")) == (gdr.INV_EXACT, gdr.INV_NEUMANN)
    assert (val("GDR_KERNEL_AUTO"), val("GDR_KERNEL_SIMT"), val("GDR_KERNEL_TC"),
            val("GDR_KERNEL_TC2"), val("GDR_KERNEL_SIMT2"), val("GDR_KERNEL_TC2W")) == (
        gdr.KERNEL_AUTO, gdr.KERNEL_SIMT, gdr.KERNEL_TC, gdr.KERNEL_TC2, gdr.KERNEL_SIMT2,
        gdr.KERNEL_TC2W)
    # struct layout: 11 ints
    assert ctypes.sizeof(gdr.GdrShape) == 44


def test_status_strings_and_version(lib):
    for s in range(11):
        assert gdr.status_string(s) != "unknown status"
    assert gdr.status_string(123) == "unknown status"
    assert gdr.version() >= 100


def _call(shape, ptrs=None, chunk=64, gate=gdr.GATE_SCALAR, inv=gdr.INV_EXACT, ws=None,
          ws_bytes=0):
    # fake but 16-byte-aligned device addresses: validation fails before any use
    p = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)] if ptrs is None else ptrs
    return gdr.load().gdr_chunk_fwd(ctypes.byref(shape), p[0], p[1], p[2], p[3], p[4], p[5],
                                    chunk, gate, inv, p[6], p[7], ws, ws_bytes, None)


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


def test_rejects_sizes_past_the_grid_and_byte_limits(lib):
    # batch and value heads index grid rows (<= 65535); at most 2^40 input elements
    assert _call(gdr.make_shape(70000, 64, 1, 1, 64, 64)) == gdr.ERR_SHAPE
    assert _call(gdr.make_shape(1, 64, 1, 70000, 64, 64)) == gdr.ERR_SHAPE
    assert _call(gdr.make_shape(60000, 1 << 30, 1, 1, 64, 64)) == gdr.ERR_SHAPE
    assert _call(gdr.make_shape(65535, 1, 65535, 65535, 64, 64)) == gdr.ERR_SHAPE   # B Hv >= 2^31
    assert gdr.select_kernel(gdr.make_shape(65536, 64, 1, 1, 64, 64), 64, gdr.GATE_SCALAR) == \
        -gdr.ERR_SHAPE
    # just inside the bound the workspace sizes are exact (no wrap-around)
    big = gdr.make_shape(64, 1 << 20, 16, 16, 128, 128)
    nch = (1 << 20) // 64
    assert gdr.state_segments(big, 64, gdr.GATE_SCALAR) == 1      # many sequences: no segments
    assert gdr.workspace_bytes(big, 64, gdr.GATE_SCALAR) == 64 * 16 * nch * gdr.TC2_SCALAR_RECORD_BYTES
    assert gdr.bwd_workspace_bytes(big, 64, gdr.GATE_SCALAR) == 4 * 64 * 16 * nch * 128 * 128
    simt2 = gdr.make_shape(64, 1 << 20, 16, 16, 128, 128, kernel="simt2")
    assert gdr.workspace_bytes(simt2, 128, gdr.GATE_CHANNEL, "neumann") == \
        64 * 16 * (nch // 2) * 2 * 128 * 128 * 4


def test_rejects_bad_enums_and_dtypes(lib):
    ok = dict(B=1, T=64, Hk=2, Hv=4, dk=64, dv=64)
    assert _call(gdr.make_shape(**ok), gate=7) == gdr.ERR_ARG
    assert _call(gdr.make_shape(**ok), inv=9) == gdr.ERR_ARG
    assert _call(gdr.make_shape(**ok, in_dtype=5)) == gdr.ERR_DTYPE
    assert _call(gdr.make_shape(**ok, out_dtype=5)) == gdr.ERR_DTYPE
    assert _call(gdr.make_shape(**ok, kernel=9)) == gdr.ERR_ARG
    assert gdr.load().gdr_chunk_fwd(None, None, None, None, None, None, None, 64, 0, 0,
                                    None, None, None, 0, None) == gdr.ERR_ARG


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
    assert gdr.select_kernel(bf, 64, gdr.GATE_SCALAR) == gdr.KERNEL_TC2
    assert gdr.select_kernel(gdr.make_shape(4, 4096, 16, 16, 128, 128, kernel="tc"), 64,
                             gdr.GATE_SCALAR) == gdr.KERNEL_TC
    # dk = 256 with grouped gates: the two-pass path (one [Q | W | K] buffer); the
    # scalar gate at dk = 256 has no two-pass record and takes the fused kernel
    sla = gdr.make_shape(2, 8192, 8, 32, 256, 128)
    assert gdr.select_kernel(sla, 64, gdr.GATE_GROUP64) == gdr.KERNEL_TC2
    assert gdr.select_kernel(sla, 128, gdr.GATE_GROUP64, "neumann") == gdr.KERNEL_TC2
    assert gdr.kernel_chunk(sla, 128, gdr.GATE_GROUP64, "neumann") == 128
    assert gdr.state_segments(sla, 64, gdr.GATE_GROUP64) == 1
    assert gdr.select_kernel(sla, 64, gdr.GATE_SCALAR) == gdr.KERNEL_TC
    # records at dk = 256: T, L, then W, Qbar, Khat of four 64-column images and 256 F
    assert gdr.workspace_bytes(sla, 64, gdr.GATE_GROUP64) == 2 * 8 * 128 * (14 * 8192 + 1024)
    assert gdr.select_kernel(gdr.make_shape(2, 8192, 8, 32, 256, 128, kernel="tc"), 64,
                             gdr.GATE_GROUP64) == gdr.KERNEL_TC
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
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL) == gdr.KERNEL_TC2
    assert gdr.kernel_chunk(kda, 128, gdr.GATE_CHANNEL) == 64
    assert gdr.kernel_chunk(kda, 64, gdr.GATE_CHANNEL) == 64
    assert gdr.kernel_chunk(kda, 128, gdr.GATE_CHANNEL, "neumann") == 128
    # ... which the two-pass path runs as pairs of 64-token halves (records with the
    # pair extras: Y, Ntil and, for per-channel gates, Kbar); the one-pass kernels
    # have no pair correction
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL, "neumann") == gdr.KERNEL_TC2
    many = gdr.make_shape(4, 4096, 16, 16, 128, 128)
    for gate, rec in ((gdr.GATE_CHANNEL, gdr.TC2_EXT_RECORD_BYTES + 4 * 8192),
                      (gdr.GATE_SCALAR, gdr.TC2_SCALAR_RECORD_BYTES + 2 * 8192)):
        assert gdr.state_segments(many, 128, gate, "neumann") == 1
        assert gdr.workspace_bytes(many, 128, gate, "neumann") == 4 * 16 * 64 * rec
    assert gdr.select_kernel(gdr.make_shape(1, 4096, 1, 1, 128, 128, kernel="tc"), 128,
                             gdr.GATE_CHANNEL, "neumann") == -gdr.ERR_UNSUPPORTED
    # segments of the segment-parallel state pass start on pair boundaries
    long = gdr.make_shape(1, 65536, 16, 16, 128, 128)
    assert gdr.state_segments(long, 128, gdr.GATE_CHANNEL, "neumann") >= 2
    simt = gdr.make_shape(1, 256, 2, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert gdr.kernel_chunk(simt, 128, gdr.GATE_SCALAR) == 128
    assert gdr.kernel_chunk(simt, 32, gdr.GATE_SCALAR) == 32
    assert gdr.kernel_chunk(gdr.make_shape(1, 256, 2, 3, 64, 64), 64,
                            gdr.GATE_SCALAR) == -gdr.ERR_SHAPE


def test_neumann1_selection(lib):
    # 1-Step Neumann depends on the chunk length (blocks of 16 in a chunk), so it is
    # never re-blocked: chunk 64 runs the two-pass path, chunk 128 the two-pass path
    # as pairs of 64-token halves with the pair correction (the function of the
    # 128-token chunk); the fused one-pass kernels do not implement it.
    kda = gdr.make_shape(2, 8192, 32, 32, 128, 128)
    assert gdr.select_kernel(kda, 64, gdr.GATE_CHANNEL, "neumann1") == gdr.KERNEL_TC2
    assert gdr.kernel_chunk(kda, 64, gdr.GATE_CHANNEL, "neumann1") == 64
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL, "neumann1") == gdr.KERNEL_TC2
    assert gdr.kernel_chunk(kda, 128, gdr.GATE_CHANNEL, "neumann1") == 128
    forced = gdr.make_shape(1, 256, 2, 2, 128, 128, kernel="tc")
    assert gdr.select_kernel(forced, 64, gdr.GATE_SCALAR, "neumann1") == -gdr.ERR_UNSUPPORTED
    sla = gdr.make_shape(2, 8192, 8, 32, 256, 128)      # dk = 256: two-pass path too
    assert gdr.select_kernel(sla, 64, gdr.GATE_GROUP64, "neumann1") == gdr.KERNEL_TC2
    sh = gdr.make_shape(1, 64, 1, 1, 128, 128)
    assert lib.gdr_kernel_chunk(ctypes.byref(sh), 64, 0, 3) == -gdr.ERR_ARG   # no mode 3


def test_output_epilogue_validates(lib):
    # validation happens before any launch (no GPU needed for these)
    f = gdr.load().gdr_output_gate_rmsnorm
    big = gdr.make_shape(1, 4, 1, 1, 1, 300)                 # dv > 256
    assert f(ctypes.byref(big), None, None, None, ctypes.c_float(1e-6), None) == gdr.ERR_SHAPE
    empty = gdr.make_shape(1, 0, 1, 1, 1, 128)               # nothing to do
    assert f(ctypes.byref(empty), None, None, None, ctypes.c_float(1e-6), None) == gdr.OK
    sh = gdr.make_shape(1, 4, 1, 1, 1, 128)
    assert f(ctypes.byref(sh), None, None, None, ctypes.c_float(-1.0), None) == gdr.ERR_ARG
    assert f(ctypes.byref(sh), None, None, None, ctypes.c_float(1e-6), None) == gdr.ERR_ARG
    assert f(None, None, None, None, ctypes.c_float(1e-6), None) == gdr.ERR_ARG


def test_momentum_validates(lib):
    # chunk-boundary momentum: host validation only (nothing launches on these)
    f = gdr.load().gdr_chunk_fwd_momentum
    nul = [None] * 6

    def call(shape, mu=0.5, kappa=None, chunk=64, inverse=gdr.INV_EXACT):
        return f(ctypes.byref(shape), *nul, chunk, gdr.GATE_SCALAR, inverse, ctypes.c_float(mu),
                 kappa, None, None, None, 0, None)

    sh = gdr.make_shape(2, 100, 1, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert call(sh) == gdr.ERR_ARG                                 # tokens but no buffers
    assert call(sh, mu=float("nan")) == gdr.ERR_ARG
    assert call(sh, mu=float("inf")) == gdr.ERR_ARG
    assert call(sh, chunk=0) == gdr.ERR_SHAPE
    empty = gdr.make_shape(0, 100, 1, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert call(empty) == gdr.OK                                   # nothing to do
    assert call(empty, kappa=ctypes.c_void_p(2)) == gdr.ERR_ALIGN  # int32 gates, 4-byte aligned
    tc = gdr.make_shape(0, 100, 1, 2, 64, 64, kernel=gdr.KERNEL_TC2)
    assert call(tc) == gdr.ERR_UNSUPPORTED                         # the two-pass path: dk = 128
    tc128 = gdr.make_shape(0, 100, 1, 2, 128, 64, kernel=gdr.KERNEL_TC2)
    assert call(tc128) == gdr.ERR_WORKSPACE                        # ... given its workspace
    assert call(tc128, chunk=128) == gdr.ERR_UNSUPPORTED           # ... at chunk 64
    assert call(gdr.make_shape(0, 100, 1, 2, 128, 64, kernel=gdr.KERNEL_TC), chunk=64) == \
        gdr.ERR_UNSUPPORTED
    # the velocity tile takes shared memory: dk = 256 with per-channel gates and
    # exact chunks of 118 fits the plain kernel but not the momentum one
    wide = gdr.make_shape(0, 1000, 1, 1, 256, 256, in_dtype=gdr.F32, out_dtype=gdr.F32,
                          kernel="simt")
    assert gdr.select_kernel(wide, 118, gdr.GATE_CHANNEL) == gdr.KERNEL_SIMT
    assert f(ctypes.byref(wide), *nul, 118, gdr.GATE_CHANNEL, gdr.INV_EXACT, ctypes.c_float(0.5),
             None, None, None, None, 0, None) == gdr.ERR_UNSUPPORTED
    assert f(ctypes.byref(wide), *nul, 64, gdr.GATE_CHANNEL, gdr.INV_EXACT, ctypes.c_float(0.5),
             None, None, None, None, 0, None) == gdr.OK


def test_two_pass_simt_selection(lib):
    # the two-pass CUDA-core form runs only when forced; its workspace holds the
    # chunk inverse and L of every chunk (2 C^2 fp32 each)
    sh = gdr.make_shape(2, 1000, 8, 32, 256, 128, kernel="simt2")
    assert gdr.select_kernel(sh, 128, gdr.GATE_GROUP64, "neumann") == gdr.KERNEL_SIMT2
    assert gdr.kernel_chunk(sh, 128, gdr.GATE_GROUP64, "neumann") == 128
    nch = (1000 + 127) // 128
    assert gdr.workspace_bytes(sh, 128, gdr.GATE_GROUP64, "neumann") == 2 * 8 * nch * 2 * 128 * 128 * 4
    auto = gdr.make_shape(2, 1000, 8, 32, 256, 128)
    assert gdr.select_kernel(auto, 128, gdr.GATE_GROUP64, "neumann") == gdr.KERNEL_TC2
    # not enough workspace: nothing launched
    full = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)]
    assert _call(sh, full, chunk=128, gate=gdr.GATE_GROUP64, inv=gdr.INV_NEUMANN,
                 ws=ctypes.c_void_p(0x900000), ws_bytes=1024) == gdr.ERR_WORKSPACE
    # per-channel gates at chunk 128 with two Newton steps: the first pass does not fit
    big = gdr.make_shape(1, 1000, 1, 1, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32,
                         neumann_residual_steps=2, kernel="simt2")
    assert gdr.select_kernel(big, 128, gdr.GATE_CHANNEL, "neumann") == -gdr.ERR_UNSUPPORTED


def test_backward_validates(lib):
    # the backward: workspace size and host validation (nothing launches on these)
    f = gdr.load().gdr_chunk_bwd
    sh = gdr.make_shape(2, 100, 1, 2, 64, 48, in_dtype=gdr.F32, out_dtype=gdr.F32)
    # the fp32 state at every chunk start: B Hv ceil(T / C) dk dv floats
    assert gdr.bwd_workspace_bytes(sh, 32, gdr.GATE_SCALAR) == 4 * 2 * 2 * 4 * 64 * 48
    assert gdr.bwd_workspace_bytes(sh, 100, gdr.GATE_CHANNEL) == 4 * 2 * 2 * 1 * 64 * 48

    def call(shape, chunk=32, gate=gdr.GATE_SCALAR, ptrs=None, ws=None, ws_bytes=0):
        ptrs = ptrs or [None] * 8
        return f(ctypes.byref(shape), *ptrs, chunk, gate, *([None] * 6), ws, ws_bytes, None)

    assert call(sh) == gdr.ERR_ARG                                  # tokens but no buffers
    assert call(sh, chunk=129) == gdr.ERR_SHAPE
    # fake but aligned device addresses: every call below fails validation first (on a
    # machine without a GPU a launch would return GDR_ERR_CUDA and fail the test)
    full = [ctypes.c_void_p(1 << 20)] * 8

    def call_all(shape, chunk=32, gate=gdr.GATE_SCALAR, ws=None, ws_bytes=0, align=0):
        outs = [ctypes.c_void_p((1 << 21) + align)] + [ctypes.c_void_p(1 << 21)] * 5
        return f(ctypes.byref(shape), *full, chunk, gate, *outs, ws, ws_bytes, None)

    need = gdr.bwd_workspace_bytes(sh, 32, gdr.GATE_SCALAR)
    assert call_all(sh, ws=None) == gdr.ERR_WORKSPACE
    assert call_all(sh, ws=ctypes.c_void_p(1 << 22), ws_bytes=need - 1) == gdr.ERR_WORKSPACE
    assert call_all(sh, ws=ctypes.c_void_p(1 << 22), ws_bytes=need, align=4) == gdr.ERR_ALIGN
    tc = gdr.make_shape(2, 100, 1, 2, 64, 48, kernel="tc2")
    assert call_all(tc, ws=ctypes.c_void_p(1 << 22), ws_bytes=need) == gdr.ERR_UNSUPPORTED
    # dk = 256 with per-channel gates at chunk 128 does not fit the backward's shared memory
    wide = gdr.make_shape(1, 100, 1, 1, 256, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert call_all(wide, chunk=128, gate=gdr.GATE_CHANNEL, ws=ctypes.c_void_p(1 << 22),
                    ws_bytes=1 << 30) == gdr.ERR_UNSUPPORTED
    empty = gdr.make_shape(0, 100, 1, 2, 64, 48, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert call(empty) == gdr.OK


def test_wide_state_pass_selection(lib):
    # the 128-column state pass: forced with TC2W (grouped / per-channel gates, dk = 128,
    # dv % 128 == 0, every inverse: the chunk-128 Neumann ones as corrected pairs); AUTO
    # takes it for few long sequences
    kda = gdr.make_shape(1, 4096, 1, 1, 128, 128, kernel="tc2w")
    assert gdr.select_kernel(kda, 64, gdr.GATE_CHANNEL) == gdr.KERNEL_TC2W
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL) == gdr.KERNEL_TC2W
    assert gdr.select_kernel(kda, 64, gdr.GATE_SCALAR) == -gdr.ERR_UNSUPPORTED
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL, "neumann") == gdr.KERNEL_TC2W
    assert gdr.select_kernel(kda, 128, gdr.GATE_CHANNEL, "neumann1") == gdr.KERNEL_TC2W
    # pairs never straddle a segment boundary: segments hold an even number of halves
    pairs = gdr.state_segments(kda, 128, gdr.GATE_CHANNEL, "neumann")
    assert pairs > 1
    assert gdr.select_kernel(gdr.make_shape(1, 4096, 1, 1, 128, 64, kernel="tc2w"), 64,
                             gdr.GATE_CHANNEL) == -gdr.ERR_UNSUPPORTED
    long = gdr.make_shape(1, 65536, 16, 16, 128, 128)
    assert gdr.select_kernel(long, 128, gdr.GATE_CHANNEL) == gdr.KERNEL_TC2
    nseg = gdr.state_segments(long, 128, gdr.GATE_CHANNEL)
    assert nseg >= 2
    # the workspace follows the plan of the pass that runs
    forced = gdr.make_shape(1, 65536, 16, 16, 128, 128, kernel="tc2w")
    assert gdr.state_segments(forced, 128, gdr.GATE_CHANNEL) == nseg
    assert gdr.workspace_bytes(forced, 128, gdr.GATE_CHANNEL) == \
        gdr.workspace_bytes(long, 128, gdr.GATE_CHANNEL)


def test_state_segments(lib):
    # The two-pass state pass stays sequential while the value tiles of all
    # sequences fill the SMs, and cuts few long sequences into segments whose
    # state maps are composed; the segment buffers then follow the records in the
    # workspace.
    many = gdr.make_shape(4, 4096, 16, 16, 128, 128)
    assert gdr.state_segments(many, 64, gdr.GATE_SCALAR) == 1
    assert gdr.workspace_bytes(many, 64, gdr.GATE_SCALAR) == 4 * 16 * 64 * gdr.TC2_SCALAR_RECORD_BYTES
    assert gdr.state_segments(gdr.make_shape(1, 256, 1, 1, 128, 128), 64, gdr.GATE_SCALAR) == 1
    long = gdr.make_shape(1, 65536, 16, 16, 128, 128)
    nseg = gdr.state_segments(long, 128, gdr.GATE_CHANNEL)
    assert 2 <= nseg <= 1024 // 16
    recs = 16 * 1024 * gdr.TC2_EXT_RECORD_BYTES
    # two dk x dv fp32 states per value head and a dk x dk one per key head, per segment
    assert gdr.workspace_bytes(long, 128, gdr.GATE_CHANNEL) == recs + nseg * 16 * 3 * 128 * 128 * 4
    # other kernels: 0; rejected requests: the negative status
    simt = gdr.make_shape(1, 256, 2, 2, 64, 64, in_dtype=gdr.F32, out_dtype=gdr.F32)
    assert gdr.state_segments(simt, 64, gdr.GATE_SCALAR) == 0
    assert gdr.state_segments(gdr.make_shape(1, 256, 2, 3, 64, 64), 64,
                              gdr.GATE_SCALAR) == -gdr.ERR_SHAPE


def test_host_entry_validates(lib):
    shape = gdr.make_shape(1, 64, 2, 4, 64, 64)
    io = gdr.GdrIO()
    assert gdr.load().gdr_chunk_fwd_host(ctypes.byref(shape), None, ctypes.byref(io), 64, 0, 0,
                                         None, 0, None) == gdr.ERR_ARG
    assert gdr.load().gdr_chunk_fwd_host(ctypes.byref(shape), ctypes.byref(io),
                                         ctypes.byref(io), 64, 0, 0, None, 0, None) == gdr.ERR_ARG


def test_workspace_rules(lib):
    # two-pass path: dk = 128 bf16; the workspace is B * Hk * ceil(T/64) chunk records
    sh = gdr.make_shape(2, 200, 3, 6, 128, 128)
    need = gdr.workspace_bytes(sh, 64, gdr.GATE_CHANNEL)
    assert need == 2 * 3 * 4 * gdr.TC2_EXT_RECORD_BYTES
    assert gdr.workspace_bytes(sh, 64, gdr.GATE_SCALAR) == 2 * 3 * 4 * gdr.TC2_SCALAR_RECORD_BYTES
    assert gdr.select_kernel(sh, 64, gdr.GATE_CHANNEL) == gdr.KERNEL_TC2
    # exact C = 128 runs blocked by 64 on the two-pass path too
    assert gdr.workspace_bytes(sh, 128, gdr.GATE_CHANNEL) == need
    forced = gdr.make_shape(2, 200, 3, 6, 128, 128, kernel="tc2")
    assert _call(forced, gate=gdr.GATE_CHANNEL) == gdr.ERR_WORKSPACE
    assert _call(forced, gate=gdr.GATE_CHANNEL, ws=ctypes.c_void_p(0x900000),
                 ws_bytes=need - 16) == gdr.ERR_WORKSPACE
    assert _call(forced, gate=gdr.GATE_CHANNEL, ws=ctypes.c_void_p(0x900004),
                 ws_bytes=need) == gdr.ERR_ALIGN
    # the one-pass kernels need none; forcing the two-pass kernel outside its envelope
    assert gdr.workspace_bytes(gdr.make_shape(1, 64, 1, 1, 256, 128), 64, gdr.GATE_SCALAR) == 0
    assert gdr.workspace_bytes(gdr.make_shape(1, 64, 1, 1, 64, 64, in_dtype=gdr.F32,
                                              out_dtype=gdr.F32), 64, gdr.GATE_SCALAR) == 0
    with pytest.raises(gdr.GdrError):
        gdr.workspace_bytes(gdr.make_shape(1, 64, 1, 1, 256, 128, kernel="tc2"), 64,
                            gdr.GATE_SCALAR)
    n = ctypes.c_size_t(0)
    assert lib.gdr_workspace_bytes(ctypes.byref(sh), 64, 0, 0, None) == gdr.ERR_ARG
    assert lib.gdr_workspace_bytes(ctypes.byref(sh), 64, 0, 7, ctypes.byref(n)) == gdr.ERR_ARG


def test_prepare_validates(lib):
    sh = gdr.make_shape(1, 130, 2, 2, 128, 128)
    need = 1 * 2 * 3 * gdr.PREP_CHUNK_BYTES
    p = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(5)]
    call = lambda shape, ptrs, chunk=64, nbytes=need: lib.gdr_chunk_prepare(
        ctypes.byref(shape), ptrs[0], ptrs[1], ptrs[2], ptrs[3], chunk, gdr.GATE_SCALAR,
        gdr.INV_EXACT, ptrs[4], nbytes, None)
    assert call(sh, p, nbytes=need - 1) == gdr.ERR_WORKSPACE
    assert call(sh, p, chunk=32) == gdr.ERR_UNSUPPORTED
    assert call(gdr.make_shape(1, 130, 2, 2, 64, 64), p) == gdr.ERR_UNSUPPORTED
    for i in range(5):
        q = list(p)
        q[i] = None
        assert call(sh, q) == gdr.ERR_ARG, i
        q[i] = ctypes.c_void_p(0x10000 * (i + 1) + 8)
        assert call(sh, q) == gdr.ERR_ALIGN, i
    assert call(gdr.make_shape(0, 130, 2, 2, 128, 128), [None] * 5) == gdr.OK
