"""The CUDA-core kernels' own source (the forward of gdr_simt.cu, the backward of
gdr_bwd.cu) compiled for the host and compared with the oracle, without a GPU.

The kernel is written as phases separated by __syncthreads(), each phase a loop
`for (idx = tid; idx < n; idx += NT)`.  With NT = 1 and the barriers as no-ops
(stand-in headers in tests/host_emu/) every phase runs to completion before the
next, so the host build computes exactly what the kernel's phases define; it
checks the kernel's algebra, indexing and shared-memory layout (a canary after
the layout's last float and around the outputs), not races between threads or
anything of the device's rounding.  CTAs run one after another over the grid
the library launches (value tiles x value heads x batch).  The parity tests on
the GPU remain the acceptance check."""
import ctypes
import os
import subprocess
import zlib

import numpy as np
import pytest

import oracle
import oracle_pins as P
from gated_delta_rule_141_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "gated_delta_rule_141_b200", "csrc")
SMEM_FLOATS = 227 * 1024 // 4
CANARY = 4096

RUNNER = r'''
}  // namespace host_emu_bwd
}  // namespace gdr
thread_local host_uint3 threadIdx, blockIdx, gridDim;
static float host_smem[%(smem)d + %(canary)d];
static const uint32_t kCanary = 0x7fc0dead;   // a NaN pattern

template <bool I, bool O, int NV, bool M, bool PRE>
static int run_grid(const gdr::Params &p)
{
    const gdr::host_emu::SimtLayout Ly = gdr::host_emu::simt_layout(
        p.C, p.G, p.dk, !PRE && (p.neumann != 0 || p.neumann1 != 0), PRE ? 0 : p.neu_resid, NV,
        p.momentum != 0);
    if (Ly.total > %(smem)d)
        return -1;
    for (unsigned b = 0; b < (unsigned)p.B; ++b)
        for (unsigned h = 0; h < (unsigned)p.Hv; ++h)
            for (unsigned x = 0; x < (unsigned)((p.dv + NV - 1) / NV); ++x) {
                threadIdx = {0, 0, 0};
                blockIdx = {x, h, b};
                std::memset(host_smem, 0xff, sizeof(float) * Ly.total);   // NaN: unset reads show
                for (int c = 0; c < %(canary)d; ++c)
                    std::memcpy(&host_smem[Ly.total + c], &kCanary, 4);
                gdr::host_emu::simt_fwd_kernel<I, O, NV, M, PRE>(p);
                for (int c = 0; c < %(canary)d; ++c)
                    if (std::memcmp(&host_smem[Ly.total + c], &kCanary, 4) != 0)
                        return -2;
            }
    return 0;
}

template <bool I, bool O, int NV>
static int run_m(const gdr::Params &p)
{
    if (p.factors != nullptr)   // second pass of the two-pass form
        return run_grid<I, O, NV, false, true>(p);
    return p.momentum ? run_grid<I, O, NV, true, false>(p) : run_grid<I, O, NV, false, false>(p);
}

template <int NV>
static int run_nv(const gdr::Params &p)
{
    if (p.in_bf16)
        return p.out_bf16 ? run_m<true, true, NV>(p) : run_m<true, false, NV>(p);
    return p.out_bf16 ? run_m<false, true, NV>(p) : run_m<false, false, NV>(p);
}

// the value-tile width the library picks: 32 columns if they fit, else 16
extern "C" int emu_tile(const gdr::Params *p)
{
    const bool pre = p->factors != nullptr;
    for (int NV : {32, 16})
        if (gdr::host_emu::simt_layout(p->C, p->G, p->dk,
                                       !pre && (p->neumann != 0 || p->neumann1 != 0),
                                       pre ? 0 : p->neu_resid, NV, p->momentum != 0).total * 4 <=
            227 * 1024)
            return NV;
    return 0;
}

// first pass of the two-pass form over its grid (chunks x key heads x batch)
extern "C" int emu_factors(const gdr::Params *p, float *rec)
{
    const gdr::host_emu::SimtLayout Ly = gdr::host_emu::simt_layout(
        p->C, p->G, p->dk, p->neumann != 0 || p->neumann1 != 0, p->neu_resid, 8, false);
    if (Ly.total * 4 > 227 * 1024)
        return -1;
    const int nch = (p->T + p->C - 1) / p->C;
    for (unsigned b = 0; b < (unsigned)p->B; ++b)
        for (unsigned h = 0; h < (unsigned)p->Hk; ++h)
            for (unsigned c = 0; c < (unsigned)nch; ++c) {
                threadIdx = {0, 0, 0};
                blockIdx = {c, h, b};
                std::memset(host_smem, 0xff, sizeof(float) * Ly.total);
                for (int k = 0; k < %(canary)d; ++k)
                    std::memcpy(&host_smem[Ly.total + k], &kCanary, 4);
                if (p->in_bf16)
                    gdr::host_emu::simt_factors_kernel<true>(*p, rec);
                else
                    gdr::host_emu::simt_factors_kernel<false>(*p, rec);
                for (int k = 0; k < %(canary)d; ++k)
                    if (std::memcmp(&host_smem[Ly.total + k], &kCanary, 4) != 0)
                        return -2;
            }
    return 0;
}

extern "C" int emu_run(const gdr::Params *p)
{
    const int NV = emu_tile(p);
    return NV == 32 ? run_nv<32>(*p) : NV == 16 ? run_nv<16>(*p) : -3;
}

// the backward kernel over its grid (the caller has run the forward for the
// chunk-start states and zeroed the accumulated gradients)
template <bool I, int NV>
static int run_bwd_grid(const gdr::Params &p)
{
    const int total = gdr::host_emu_bwd::bwd_layout(p.C, p.G, p.dk, NV, I ? 2 : 4).total;
    if (total > %(smem)d)
        return -1;
    for (unsigned b = 0; b < (unsigned)p.B; ++b)
        for (unsigned h = 0; h < (unsigned)p.Hv; ++h)
            for (unsigned x = 0; x < (unsigned)((p.dv + NV - 1) / NV); ++x) {
                threadIdx = {0, 0, 0};
                blockIdx = {x, h, b};
                std::memset(host_smem, 0xff, sizeof(float) * total);
                for (int c = 0; c < %(canary)d; ++c)
                    std::memcpy(&host_smem[total + c], &kCanary, 4);
                gdr::host_emu_bwd::simt_bwd_kernel<I, NV>(p);
                for (int c = 0; c < %(canary)d; ++c)
                    if (std::memcmp(&host_smem[total + c], &kCanary, 4) != 0)
                        return -2;
            }
    return 0;
}

extern "C" int emu_bwd_tile(const gdr::Params *p)
{
    for (int NV : {32, 16})
        if (gdr::host_emu_bwd::bwd_layout(p->C, p->G, p->dk, NV, p->in_bf16 ? 2 : 4).total * 4 <= 227 * 1024)
            return NV;
    return 0;
}

extern "C" int emu_bwd(const gdr::Params *p)
{
    const int NV = emu_bwd_tile(p);
    if (NV == 32)
        return p->in_bf16 ? run_bwd_grid<true, 32>(*p) : run_bwd_grid<false, 32>(*p);
    if (NV == 16)
        return p->in_bf16 ? run_bwd_grid<true, 16>(*p) : run_bwd_grid<false, 16>(*p);
    return -3;
}
'''


class Params(ctypes.Structure):
    # gdr::Params of gdr_internal.h, field for field
    _fields_ = ([(n, ctypes.c_int) for n in
                 "B T Hk Hv dk dv G C R in_bf16 out_bf16 neumann neumann1 pair wide_state neu_order neu_resid "
                 "momentum".split()] +
                [("mu", ctypes.c_float), ("kappa", ctypes.c_void_p)] +
                [(n, ctypes.c_void_p) for n in
                 "q k v g beta S0 o S_final S_chunks factors dO dS_final grad_q grad_k grad_v grad_g "
                 "grad_beta grad_S0".split()])


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    def kernel_part(name, marker, ns):
        src = open(os.path.join(CSRC, name)).read()
        body = src[:src.index(marker)]
        for old, new in (("constexpr int NT = 256;", "constexpr int NT = 1;"),
                         ("namespace {", "namespace %s {" % ns)):
            assert body.count(old) == 1, old
            body = body.replace(old, new)
        assert "extern __shared__ float sm[];" in body     # every kernel's shared memory
        return body.replace("extern __shared__ float sm[];", "float *const sm = host_smem_ptr();")

    fwd = kernel_part("gdr_simt.cu", "template <bool I, bool O, int NV, bool MOM, bool PRE>\nint launch_variant",
                      "host_emu")
    bwd = kernel_part("gdr_bwd.cu", "template <bool I, int NV>\nint launch_bwd_variant", "host_emu_bwd")
    # each part ends inside `namespace gdr { namespace ... {`; close the first
    body = fwd + "}  // namespace host_emu\n}  // namespace gdr\n" + bwd
    head = "float *host_smem_ptr();\n"
    tail = RUNNER % {"smem": SMEM_FLOATS, "canary": CANARY} + "float *host_smem_ptr() { return host_smem; }\n"
    d = tmp_path_factory.mktemp("host_emu")
    cpp = d / "simt_host.cpp"
    cpp.write_text(head + body + tail)
    so = d / "simt_host.so"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-w",
                           "-I" + os.path.join(HERE, "host_emu"), "-I" + CSRC,
                           "-I" + os.path.join(ROOT, "include"), str(cpp), "-o", str(so)])
    lib = ctypes.CDLL(str(so))
    lib.emu_run.argtypes = [ctypes.POINTER(Params)]
    lib.emu_tile.argtypes = [ctypes.POINTER(Params)]
    lib.emu_factors.argtypes = [ctypes.POINTER(Params), ctypes.c_void_p]
    lib.emu_bwd.argtypes = [ctypes.POINTER(Params)]
    lib.emu_bwd_tile.argtypes = [ctypes.POINTER(Params)]
    return lib


def _bf16_bits(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _from_bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def run_host(lib, x, chunk, inverse="exact", order=4, resid=1, bf16=False, mu=None, kappa=None,
             two_pass=False):
    q = x["q"]
    B, Hk, T, dk = q.shape
    Hv, dv, G = x["v"].shape[1], x["v"].shape[3], x["g"].shape[3]
    conv = _bf16_bits if bf16 else (lambda a: np.ascontiguousarray(a, np.float32))
    qq, kk, vv = conv(x["q"]), conv(x["k"]), conv(x["v"])
    g = np.ascontiguousarray(x["g"], np.float32)
    beta = np.ascontiguousarray(x["beta"], np.float32)
    S0 = None if x["S0"] is None else np.ascontiguousarray(x["S0"], np.float32)
    guard = 64
    n_o = B * Hv * T * dv
    o_buf = np.full(n_o + 2 * guard, 0x7FC1, np.uint16) if bf16 else np.full(n_o + 2 * guard, 12345.0, np.float32)
    s_buf = np.full(B * Hv * dk * dv + 2 * guard, 12345.0, np.float32)
    kap = None if kappa is None else np.ascontiguousarray(kappa, np.int32)
    ptr = lambda a, off=0: None if a is None else a.ctypes.data + off * a.itemsize
    p = Params(B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, G=G, C=chunk, R=Hv // Hk,
               in_bf16=int(bf16), out_bf16=int(bf16), neumann=int(inverse == "neumann"),
               neumann1=int(inverse == "neumann1"),
               neu_order=order if inverse == "neumann" else 0,
               neu_resid=resid if inverse == "neumann" else 0,
               momentum=int(mu is not None), mu=0.0 if mu is None else mu, kappa=ptr(kap),
               q=ptr(qq), k=ptr(kk), v=ptr(vv), g=ptr(g), beta=ptr(beta), S0=ptr(S0),
               o=ptr(o_buf, guard), S_final=ptr(s_buf, guard))
    if two_pass:   # the first pass's records; NaN where a record is not written
        nch = (T + chunk - 1) // chunk
        rec = np.full(B * Hk * nch * 2 * chunk * chunk + 2 * guard, np.nan, np.float32)
        assert lib.emu_factors(ctypes.byref(p), ptr(rec, guard)) == 0
        assert np.all(np.isnan(rec[:guard])) and np.all(np.isnan(rec[-guard:]))
        p.factors = ptr(rec, guard)
    assert lib.emu_tile(ctypes.byref(p)) in (16, 32)
    rc = lib.emu_run(ctypes.byref(p))
    assert rc == 0, "host run failed (%d: -2 = shared-memory canary overwritten)" % rc
    for buf in (o_buf, s_buf):   # nothing written outside the outputs
        assert np.all(buf[:guard] == buf[0]) and np.all(buf[-guard:] == buf[0])
    o = o_buf[guard:guard + n_o]
    o = (_from_bf16(o) if bf16 else o).reshape(B, Hv, T, dv).astype(np.float64)
    S = s_buf[guard:-guard].reshape(B, Hv, dk, dv).astype(np.float64)
    return o, S


def rel(x, ref):
    den = np.abs(ref).max() if ref.size else 0.0
    return float(np.abs(x - ref).max() / den) if den > 0 else float(np.abs(x).max() if x.size else 0.0)


# (T, Hk, Hv, dk, dv, G, chunk, inverse, order, resid, with S0)
CASES = [
    (37, 1, 2, 32, 48, 1, 16, "exact", 4, 1, True),
    (70, 1, 1, 64, 32, 64, 32, "exact", 4, 1, False),
    (203, 1, 3, 64, 40, 1, 64, "exact", 4, 1, True),       # ragged last chunk, 3 value heads
    (91, 1, 1, 64, 20, 64, 128, "exact", 4, 1, True),      # one short chunk, dv not a multiple of 8
    (40, 1, 1, 256, 24, 4, 32, "exact", 4, 1, True),       # dk = 256 (16-column tiles)
    (50, 1, 1, 32, 32, 4, 16, "neumann", 4, 1, True),      # chunk below the value tile
    (187, 1, 3, 32, 24, 1, 100, "neumann", 1, 1, False),
    (51, 1, 3, 64, 24, 64, 64, "neumann", 3, 2, True),     # two residual steps (P buffer)
    (45, 1, 1, 32, 40, 32, 24, "neumann1", 4, 1, True),
    (144, 1, 2, 128, 72, 1, 100, "neumann1", 4, 1, False),
    (9, 1, 1, 16, 8, 16, 1, "exact", 4, 1, True),          # chunk of one token
    (0, 1, 1, 32, 32, 1, 64, "exact", 4, 1, True),         # no tokens: S_final = S0
]


@pytest.mark.parametrize("case", CASES, ids=["T%d-R%d-dk%d-dv%d-G%d-C%d-%s" % (c[0], c[2] // c[1], c[3], c[4], c[5], c[6], c[7])
                                             for c in CASES])
def test_host_kernel_matches_oracle(emu, case):
    T, Hk, Hv, dk, dv, G, chunk, inverse, order, resid, with_s0 = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    q, k, v, g, beta, S0 = P.rand_inputs(rng, 1, T, Hk, Hv, dk, dv, G)
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0 if with_s0 else None}
    o, S = run_host(emu, x, chunk, inverse, order, resid)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    if inverse == "exact":
        o_ref, S_ref = oracle.recurrent(*args)
    else:
        o_ref, S_ref = oracle.chunked(*args, chunk=chunk, inverse=inverse, order=order, resid=resid)
    assert rel(o, o_ref) <= 1e-5 and rel(S, S_ref) <= 1e-5


@pytest.mark.parametrize("case", CASES, ids=["T%d-R%d-dk%d-dv%d-G%d-C%d-%s" % (c[0], c[2] // c[1], c[3], c[4], c[5], c[6], c[7])
                                             for c in CASES])
def test_host_two_pass_matches_oracle(emu, case):
    # the two-pass form (chunk factors of all chunks first, then the value tiles'
    # pass reading them): the same results as the one-pass kernel computes
    T, Hk, Hv, dk, dv, G, chunk, inverse, order, resid, with_s0 = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    q, k, v, g, beta, S0 = P.rand_inputs(rng, 1, T, Hk, Hv, dk, dv, G)
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0 if with_s0 else None}
    o, S = run_host(emu, x, chunk, inverse, order, resid, two_pass=True)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    if inverse == "exact":
        o_ref, S_ref = oracle.recurrent(*args)
    else:
        o_ref, S_ref = oracle.chunked(*args, chunk=chunk, inverse=inverse, order=order, resid=resid)
    assert rel(o, o_ref) <= 1e-5 and rel(S, S_ref) <= 1e-5


@pytest.mark.parametrize("chunk,inverse,mu", [(64, "exact", 0.9), (16, "neumann1", -0.3), (32, "neumann", 1.0)])
def test_host_kernel_momentum(emu, chunk, inverse, mu):
    rng = np.random.default_rng(chunk)
    q, k, v, g, beta, S0 = P.rand_inputs(rng, 2, 150, 1, 2, 32, 40, 32)
    kappa = (rng.random((2, (150 + chunk - 1) // chunk)) < 0.7).astype(np.int32)
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0}
    o, S = run_host(emu, x, chunk, inverse, mu=mu, kappa=kappa)
    o_ref, S_ref = oracle.chunked(q, k, v, g, beta, S0, chunk=chunk, inverse=inverse, mu=mu, kappa=kappa)
    assert rel(o, o_ref) <= 1e-5 and rel(S, S_ref) <= 1e-5


def test_host_kernel_bf16_io(emu):
    # bf16 loads and stores: inputs already on the bf16 grid, o rounded once
    w, x = W.workload_inputs(1, B=1, Hk=1, Hv=2, T=150)
    o, S = run_host(emu, x, 64, bf16=True)
    o_ref, S_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    assert rel(S, S_ref) <= 1e-5
    assert rel(o, o_ref) <= 2.0 ** -8


def run_host_bwd(lib, x, chunk, dO, dSf, bf16=False):
    """The library's backward on the host: the forward kernel for the chunk-start
    states (no outputs), then the backward kernel; returns the gradients."""
    q = x["q"]
    B, Hk, T, dk = q.shape
    Hv, dv, G = x["v"].shape[1], x["v"].shape[3], x["g"].shape[3]
    conv = _bf16_bits if bf16 else (lambda a: np.ascontiguousarray(a, np.float32))
    qq, kk, vv = conv(x["q"]), conv(x["k"]), conv(x["v"])
    g = np.ascontiguousarray(x["g"], np.float32)
    beta = np.ascontiguousarray(x["beta"], np.float32)
    S0 = None if x["S0"] is None else np.ascontiguousarray(x["S0"], np.float32)
    nch = (T + chunk - 1) // chunk
    guard = 64
    f32 = lambda n: np.full(n + 2 * guard, 12345.0, np.float32)
    Sc = f32(B * Hv * nch * dk * dv)
    outs = {"q": (B, Hk, T, dk), "k": (B, Hk, T, dk), "v": (B, Hv, T, dv), "g": (B, Hk, T, G),
            "beta": (B, Hk, T), "S0": (B, Hv, dk, dv)}
    bufs = {n: f32(int(np.prod(s))) for n, s in outs.items()}
    for n in ("q", "k", "g", "beta"):       # accumulated: the library zeroes them first
        bufs[n][guard:-guard] = 0.0
    dO32 = np.ascontiguousarray(dO, np.float32)
    dS32 = None if dSf is None else np.ascontiguousarray(dSf, np.float32)
    ptr = lambda a, off=0: None if a is None else a.ctypes.data + off * a.itemsize
    p = Params(B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, G=G, C=chunk, R=Hv // Hk,
               in_bf16=int(bf16), out_bf16=0, neumann=0, neumann1=0, neu_order=0, neu_resid=0,
               momentum=0, mu=0.0, kappa=None, q=ptr(qq), k=ptr(kk), v=ptr(vv), g=ptr(g),
               beta=ptr(beta), S0=ptr(S0), o=None, S_final=None, S_chunks=ptr(Sc, guard))
    assert lib.emu_run(ctypes.byref(p)) == 0
    p.S_chunks = ptr(Sc, guard)
    p.dO, p.dS_final = ptr(dO32), ptr(dS32)
    p.grad_q, p.grad_k, p.grad_v = ptr(bufs["q"], guard), ptr(bufs["k"], guard), ptr(bufs["v"], guard)
    p.grad_g, p.grad_beta, p.grad_S0 = ptr(bufs["g"], guard), ptr(bufs["beta"], guard), ptr(bufs["S0"], guard)
    assert lib.emu_bwd_tile(ctypes.byref(p)) in (16, 32)
    rc = lib.emu_bwd(ctypes.byref(p))
    assert rc == 0, "host backward failed (%d: -2 = shared-memory canary overwritten)" % rc
    for buf in [Sc] + list(bufs.values()):
        assert np.all(buf[:guard] == 12345.0) and np.all(buf[-guard:] == 12345.0)
    return {n: bufs[n][guard:-guard].reshape(s).astype(np.float64) for n, s in outs.items()}


# (T, Hk, Hv, dk, dv, G, chunk, with S0, with dS_final)
BWD_CASES = [
    (37, 1, 2, 32, 48, 1, 16, True, True),      # ragged tail, two value heads, two value tiles
    (70, 1, 1, 64, 32, 64, 32, True, False),    # per-channel decay
    (45, 2, 4, 64, 20, 1, 64, False, True),     # one short chunk, dv not a multiple of 8
    (50, 1, 1, 128, 16, 2, 16, True, True),     # 64-channel groups
    (9, 1, 1, 16, 8, 16, 1, True, True),        # chunks of one token
    (0, 1, 1, 32, 32, 1, 64, True, True),       # no tokens: dS0 = dS_final
]


@pytest.mark.parametrize("case", BWD_CASES, ids=["T%d-R%d-dk%d-dv%d-G%d-C%d" % (c[0], c[2] // c[1], c[3], c[4], c[5], c[6])
                                                 for c in BWD_CASES])
def test_host_backward_matches_oracle(emu, case):
    T, Hk, Hv, dk, dv, G, chunk, with_s0, with_dsf = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    q, k, v, g, beta, S0 = P.rand_inputs(rng, 1, T, Hk, Hv, dk, dv, G)
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0 if with_s0 else None}
    dO = rng.standard_normal((1, Hv, T, dv))
    dSf = rng.standard_normal((1, Hv, dk, dv)) if with_dsf else None
    got = run_host_bwd(emu, x, chunk, dO, dSf)
    ref = oracle.recurrent_grad(q, k, v, g, beta, x["S0"], dO, dSf)
    for n in ("q", "k", "v", "g", "beta", "S0"):
        assert rel(got[n], ref[n]) <= 1e-4, (n, rel(got[n], ref[n]))


def test_host_kernel_momentum_bf16_io(emu):
    # momentum with bf16 q, k, v and bf16 o (the gdn_scalar_bf16 shapes, shortened)
    w, x = W.workload_inputs(1, B=2, Hk=1, Hv=2, T=200)
    kappa = (np.random.default_rng(9).random((2, 4)) < 0.7).astype(np.int32)
    o, S = run_host(emu, x, 64, bf16=True, mu=0.25, kappa=kappa)
    o_ref, S_ref = oracle.chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], chunk=64,
                                  mu=0.25, kappa=kappa)
    assert rel(S, S_ref) <= 1e-5
    assert rel(o, o_ref) <= 2.0 ** -8
