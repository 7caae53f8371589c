// gdr_api.cu -- the C ABI of libgdr.so (declared in include/gdr.h): argument
// validation, kernel selection and the host-buffer convenience entry point.
// Every computation happens in the kernels of gdr_simt.cu / gdr_tc.cu.
#include <cstdint>
#include <cstddef>

#include "gdr.h"
#include "gdr_internal.h"

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(gdr_dtype d) { return d == GDR_BF16 ? 2 : 4; }

gdr_status make_params(const gdr_shape *s, int chunk, gdr_gate_mode gm, gdr_inverse_mode im,
                       gdr::Params *p)
{
    if (s == nullptr)
        return GDR_ERR_ARG;
    if (s->in_dtype != GDR_F32 && s->in_dtype != GDR_BF16)
        return GDR_ERR_DTYPE;
    if (s->out_dtype != GDR_F32 && s->out_dtype != GDR_BF16)
        return GDR_ERR_DTYPE;
    if (s->kernel != GDR_KERNEL_AUTO && s->kernel != GDR_KERNEL_SIMT && s->kernel != GDR_KERNEL_TC &&
        s->kernel != GDR_KERNEL_TC2 && s->kernel != GDR_KERNEL_SIMT2 && s->kernel != GDR_KERNEL_TC2W)
        return GDR_ERR_ARG;
    if (s->B < 0 || s->T < 0 || s->Hk < 1 || s->Hv < 1 || s->Hv % s->Hk != 0)
        return GDR_ERR_SHAPE;
    if (s->dk < 1 || s->dk > 256 || s->dv < 1 || s->dv > 256)
        return GDR_ERR_SHAPE;
    // batch and heads index grid rows (at most 65535), and at most 2^40 input
    // elements keep every byte count here (records, workspaces) far inside 64 bits
    if (s->B > 65535 || s->Hv > 65535 || (long)s->B * s->Hv > 0x7fffffffL)   // and 32-bit sequence indices
        return GDR_ERR_SHAPE;
    if ((double)s->B * s->T * ((double)s->Hk * s->dk + (double)s->Hv * s->dv) > 1099511627776.0)
        return GDR_ERR_SHAPE;
    if (chunk < 1 || chunk > 128)
        return GDR_ERR_SHAPE;
    int G;
    switch (gm) {
    case GDR_GATE_SCALAR: G = 1; break;
    case GDR_GATE_GROUP64:
        if (s->dk % 64 != 0)
            return GDR_ERR_SHAPE;
        G = s->dk / 64;
        break;
    case GDR_GATE_CHANNEL: G = s->dk; break;
    default: return GDR_ERR_ARG;
    }
    if (im != GDR_INV_EXACT && im != GDR_INV_NEUMANN && im != GDR_INV_NEUMANN1)
        return GDR_ERR_ARG;
    if (im == GDR_INV_NEUMANN &&
        (s->neumann_order < 0 || s->neumann_order > 256 || s->neumann_residual_steps < 0 ||
         s->neumann_residual_steps > 16))
        return GDR_ERR_SHAPE;
    *p = gdr::Params{};
    p->B = s->B; p->T = s->T; p->Hk = s->Hk; p->Hv = s->Hv; p->dk = s->dk; p->dv = s->dv;
    p->G = G; p->C = chunk; p->R = s->Hv / s->Hk;
    p->in_bf16 = s->in_dtype == GDR_BF16;
    p->out_bf16 = s->out_dtype == GDR_BF16;
    p->neumann = im == GDR_INV_NEUMANN;
    p->neumann1 = im == GDR_INV_NEUMANN1;
    p->neu_order = p->neumann ? s->neumann_order : 0;
    p->neu_resid = p->neumann ? s->neumann_residual_steps : 0;
    p->wide_state = s->kernel == GDR_KERNEL_TC2W;
    return GDR_OK;
}

// GDR_KERNEL_SIMT / GDR_KERNEL_TC / GDR_KERNEL_TC2 / GDR_KERNEL_SIMT2 (forced
// only), or -status, for a call that brings `ws_bytes` of workspace (SIZE_MAX:
// as much as the kernel asks for).
int choose(const gdr::Params &p, gdr_kernel want, size_t ws_bytes)
{
    const bool tc2 = gdr::tc2_supports(p);
    const bool tc2_fits = tc2 && ws_bytes >= gdr::tc2_workspace_bytes(p);
    const bool tc = gdr::tc_supports(p);
    const bool simt = gdr::simt_smem_bytes(p) <= 227 * 1024;
    switch (want) {
    case GDR_KERNEL_TC2:
        if (!tc2)
            return -GDR_ERR_UNSUPPORTED;
        return tc2_fits ? GDR_KERNEL_TC2 : -GDR_ERR_WORKSPACE;
    case GDR_KERNEL_TC2W:
        if (!gdr::tc2w_supports(p))
            return -GDR_ERR_UNSUPPORTED;
        return tc2_fits ? GDR_KERNEL_TC2W : -GDR_ERR_WORKSPACE;
    case GDR_KERNEL_TC: return tc ? GDR_KERNEL_TC : -GDR_ERR_UNSUPPORTED;
    case GDR_KERNEL_SIMT: return simt ? GDR_KERNEL_SIMT : -GDR_ERR_UNSUPPORTED;
    case GDR_KERNEL_SIMT2:
        if (!gdr::simt2_supports(p))
            return -GDR_ERR_UNSUPPORTED;
        return ws_bytes >= gdr::simt2_workspace_bytes(p) ? GDR_KERNEL_SIMT2 : -GDR_ERR_WORKSPACE;
    default: break;
    }
    if (tc2_fits)
        return GDR_KERNEL_TC2;
    if (tc)
        return GDR_KERNEL_TC;
    return simt ? GDR_KERNEL_SIMT : -GDR_ERR_UNSUPPORTED;
}

// Every check gdr_chunk_fwd makes before it launches anything: the request, the
// device pointers, their alignment and the kernel choice given the workspace.
// On GDR_OK *p holds the request with its pointers and *which the kernel.
gdr_status validate_fwd(const gdr_shape *shape, const void *q, const void *k, const void *v,
                        const float *g, const float *beta, const float *S0, int chunk,
                        gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode, void *o,
                        float *S_final, void *workspace, size_t workspace_bytes, gdr::Params *p,
                        int *which)
{
    gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, p);
    if (st != GDR_OK)
        return st;
    const bool has_tokens = (long)p->B * p->T > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !o))
        return GDR_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, o, S_final, workspace};
    for (const void *ptr : ptrs)
        if (ptr != nullptr && !aligned16(ptr))
            return GDR_ERR_ALIGN;
    const int w = choose(*p, shape->kernel, workspace != nullptr ? workspace_bytes : 0);
    if (w < 0)
        return static_cast<gdr_status>(-w);
    p->q = q; p->k = k; p->v = v; p->g = g; p->beta = beta; p->S0 = S0; p->o = o; p->S_final = S_final;
    *which = w;
    return GDR_OK;
}

gdr_status launch_fwd(const gdr::Params &p, int which, void *workspace, cudaStream_t s)
{
    if (p.B == 0)
        return GDR_OK;
    int rc;
    if (which == GDR_KERNEL_TC2 || which == GDR_KERNEL_TC2W)
        rc = gdr::launch_tc2(p, workspace, s);
    else if (which == GDR_KERNEL_SIMT2)
        rc = gdr::launch_simt2(p, workspace, s);
    else if (which == GDR_KERNEL_TC)
        rc = gdr::launch_tc(p, s);
    else
        rc = gdr::launch_simt(p, s);
    return static_cast<gdr_status>(rc);
}

}  // namespace

extern "C" {

gdr_status gdr_chunk_fwd(const gdr_shape *shape, const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0, int chunk,
                         gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode, void *o,
                         float *S_final, void *workspace, size_t workspace_bytes, void *stream)
{
    gdr::Params p;
    int which = 0;
    const gdr_status st = validate_fwd(shape, q, k, v, g, beta, S0, chunk, gate_mode, inverse_mode,
                                       o, S_final, workspace, workspace_bytes, &p, &which);
    if (st != GDR_OK)
        return st;
    return launch_fwd(p, which, workspace, static_cast<cudaStream_t>(stream));
}

gdr_status gdr_bwd_workspace_bytes(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                                   size_t *bytes)
{
    if (bytes == nullptr)
        return GDR_ERR_ARG;
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, GDR_INV_EXACT, &p);
    if (st != GDR_OK)
        return st;
    *bytes = gdr::bwd_workspace_bytes(p);
    return GDR_OK;
}

gdr_status gdr_chunk_bwd(const gdr_shape *shape, const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0, const float *dO,
                         const float *dS_final, int chunk, gdr_gate_mode gate_mode, float *dq,
                         float *dk, float *dv, float *dg, float *dbeta, float *dS0,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    gdr::Params p;
    gdr_status st = make_params(shape, chunk, gate_mode, GDR_INV_EXACT, &p);
    if (st != GDR_OK)
        return st;
    const bool has_tokens = (long)p.B * p.T > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta))
        return GDR_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, dO, dS_final, dq, dk, dv, dg, dbeta, dS0, workspace};
    for (const void *ptr : ptrs)
        if (ptr != nullptr && !aligned16(ptr))
            return GDR_ERR_ALIGN;
    if (shape->kernel != GDR_KERNEL_AUTO && shape->kernel != GDR_KERNEL_SIMT)
        return GDR_ERR_UNSUPPORTED;
    if (gdr::bwd_smem_bytes(p) > 227 * 1024 || gdr::simt_smem_bytes(p) > 227 * 1024)
        return GDR_ERR_UNSUPPORTED;
    const size_t need = gdr::bwd_workspace_bytes(p);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return GDR_ERR_WORKSPACE;
    if (p.B == 0)
        return GDR_OK;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.S0 = S0;
    p.dO = dO; p.dS_final = dS_final;
    p.grad_q = dq; p.grad_k = dk; p.grad_v = dv; p.grad_g = dg; p.grad_beta = dbeta; p.grad_S0 = dS0;
    return static_cast<gdr_status>(gdr::launch_bwd(p, workspace, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_chunk_fwd_momentum(const gdr_shape *shape, const void *q, const void *k,
                                  const void *v, const float *g, const float *beta,
                                  const float *S0, int chunk, gdr_gate_mode gate_mode,
                                  gdr_inverse_mode inverse_mode, float mu, const int32_t *kappa,
                                  void *o, float *S_final, void *workspace, size_t workspace_bytes,
                                  void *stream)
{
    gdr::Params p;
    gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return st;
    if (!(mu > -1e30f && mu < 1e30f))   // finite (NaN fails both)
        return GDR_ERR_ARG;
    const bool has_tokens = (long)p.B * p.T > 0;
    if (has_tokens && (!q || !k || !v || !g || !beta || !o))
        return GDR_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, o, S_final, workspace};
    for (const void *ptr : ptrs)
        if (ptr != nullptr && !aligned16(ptr))
            return GDR_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(kappa) & 3u) != 0)
        return GDR_ERR_ALIGN;
    const gdr_kernel want = shape->kernel;
    if (want != GDR_KERNEL_AUTO && want != GDR_KERNEL_SIMT && want != GDR_KERNEL_TC2)
        return GDR_ERR_UNSUPPORTED;
    p.momentum = 1;
    p.mu = mu;
    p.kappa = kappa;
    // the two-pass tensor-core path when it applies and the workspace suffices
    const bool tc2 = want != GDR_KERNEL_SIMT && gdr::tc2_supports(p) && workspace != nullptr &&
                     workspace_bytes >= gdr::tc2_workspace_bytes(p);
    if (want == GDR_KERNEL_TC2 && !tc2)
        return gdr::tc2_supports(p) ? GDR_ERR_WORKSPACE : GDR_ERR_UNSUPPORTED;
    if (!tc2 && gdr::simt_smem_bytes(p) > 227 * 1024)
        return GDR_ERR_UNSUPPORTED;
    if (p.B == 0)
        return GDR_OK;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.S0 = S0; p.o = o; p.S_final = S_final;
    auto s = static_cast<cudaStream_t>(stream);
    return static_cast<gdr_status>(tc2 ? gdr::launch_tc2(p, workspace, s) : gdr::launch_simt(p, s));
}

gdr_status gdr_workspace_bytes(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                               gdr_inverse_mode inverse_mode, size_t *bytes)
{
    if (bytes == nullptr)
        return GDR_ERR_ARG;
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return st;
    const int which = choose(p, shape->kernel, SIZE_MAX);
    if (which < 0)
        return static_cast<gdr_status>(-which);
    *bytes = which == GDR_KERNEL_TC2 || which == GDR_KERNEL_TC2W ? gdr::tc2_workspace_bytes(p)
             : which == GDR_KERNEL_SIMT2 ? gdr::simt2_workspace_bytes(p)
                                         : 0;
    return GDR_OK;
}

gdr_status gdr_chunk_prepare(const gdr_shape *shape, const void *q, const void *k,
                             const float *g, const float *beta, int chunk,
                             gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode,
                             void *factors, size_t factors_bytes, void *stream)
{
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return st;
    const bool has_tokens = (long)p.B * p.T > 0;
    if (has_tokens && (!q || !k || !g || !beta || !factors))
        return GDR_ERR_ARG;
    const void *ptrs[] = {q, k, g, beta, factors};
    for (const void *ptr : ptrs)
        if (ptr != nullptr && !aligned16(ptr))
            return GDR_ERR_ALIGN;
    if (!gdr::prepare_supports(p))
        return GDR_ERR_UNSUPPORTED;
    if (factors_bytes < gdr::prepare_bytes(p))
        return GDR_ERR_WORKSPACE;
    if (!has_tokens)
        return GDR_OK;
    p.q = q; p.k = k; p.g = g; p.beta = beta;
    return static_cast<gdr_status>(gdr::launch_prepare(p, factors, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_chunk_fwd_host(const gdr_shape *shape, const gdr_io *host, const gdr_io *dev,
                              int chunk, gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    if (host == nullptr || dev == nullptr)
        return GDR_ERR_ARG;
    // the whole device-side request is validated before any copy is queued, so
    // that a refused call leaves nothing on the stream
    gdr::Params p;
    int which = 0;
    gdr_status st = validate_fwd(shape, dev->q, dev->k, dev->v, dev->g, dev->beta, dev->S0, chunk,
                                 gate_mode, inverse_mode, dev->o, dev->S_final, workspace,
                                 workspace_bytes, &p, &which);
    if (st != GDR_OK)
        return st;
    const bool has_tokens = (long)p.B * p.T > 0;
    if (has_tokens && (!host->q || !host->k || !host->v || !host->g || !host->beta || !host->o))
        return GDR_ERR_ARG;
    if ((host->S0 == nullptr) != (dev->S0 == nullptr) ||
        (host->S_final == nullptr) != (dev->S_final == nullptr))
        return GDR_ERR_ARG;
    const size_t si = elem_size(shape->in_dtype), so = elem_size(shape->out_dtype);
    const size_t nk = (size_t)p.B * p.Hk * p.T, nv = (size_t)p.B * p.Hv * p.T;
    const size_t nstate = (size_t)p.B * p.Hv * p.dk * p.dv;
    auto s = static_cast<cudaStream_t>(stream);
    struct Copy { void *dst; const void *src; size_t bytes; };
    const Copy in[] = {
        {const_cast<void *>(dev->q), host->q, nk * p.dk * si},
        {const_cast<void *>(dev->k), host->k, nk * p.dk * si},
        {const_cast<void *>(dev->v), host->v, nv * p.dv * si},
        {const_cast<float *>(dev->g), host->g, nk * p.G * sizeof(float)},
        {const_cast<float *>(dev->beta), host->beta, nk * sizeof(float)},
        {const_cast<float *>(dev->S0), host->S0, nstate * sizeof(float)},
    };
    for (const Copy &c : in) {
        if (c.bytes == 0 || c.src == nullptr)
            continue;
        if (cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return GDR_ERR_CUDA;
    }
    st = launch_fwd(p, which, workspace, s);
    if (st != GDR_OK)
        return st;
    if (has_tokens &&
        cudaMemcpyAsync(host->o, dev->o, nv * p.dv * so, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (host->S_final && nstate &&
        cudaMemcpyAsync(host->S_final, dev->S_final, nstate * sizeof(float),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDR_ERR_CUDA;
    return GDR_OK;
}

int gdr_select_kernel(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                      gdr_inverse_mode inverse_mode)
{
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return -static_cast<int>(st);
    return choose(p, shape->kernel, SIZE_MAX);
}

int gdr_kernel_chunk(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                     gdr_inverse_mode inverse_mode)
{
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return -static_cast<int>(st);
    const int which = choose(p, shape->kernel, SIZE_MAX);
    if (which < 0)
        return which;
    return (which == GDR_KERNEL_SIMT || which == GDR_KERNEL_SIMT2) ? p.C : gdr::tc_kernel_chunk(p);
}

int gdr_state_segments(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                       gdr_inverse_mode inverse_mode)
{
    gdr::Params p;
    const gdr_status st = make_params(shape, chunk, gate_mode, inverse_mode, &p);
    if (st != GDR_OK)
        return -static_cast<int>(st);
    const int which = choose(p, shape->kernel, SIZE_MAX);
    if (which < 0)
        return which;
    return (which == GDR_KERNEL_TC2 || which == GDR_KERNEL_TC2W) ? gdr::tc2_state_segments(p) : 0;
}

gdr_status gdr_device_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDR_ERR_CUDA;
    const int v = gdr::read_and_clear_device_status();
    if (v < 0)
        return GDR_ERR_CUDA;
    return v == 0 ? GDR_OK : GDR_ERR_TIMEOUT;
}

gdr_status gdr_selftest_bounded_wait(uint64_t limit_ns, void *stream)
{
    if (limit_ns < 1000u || limit_ns > 1000000000u)
        return GDR_ERR_ARG;
    return static_cast<gdr_status>(gdr::launch_wait_probe(limit_ns, static_cast<cudaStream_t>(stream)));
}

const char *gdr_status_string(gdr_status status)
{
    switch (status) {
    case GDR_OK: return "ok";
    case GDR_ERR_ARG: return "invalid argument (null pointer or bad enum)";
    case GDR_ERR_SHAPE: return "sizes outside the supported envelope";
    case GDR_ERR_DTYPE: return "unsupported dtype";
    case GDR_ERR_ALIGN: return "pointer not 16-byte aligned";
    case GDR_ERR_UNSUPPORTED: return "no kernel implements this request";
    case GDR_ERR_CUDA: return "CUDA runtime error";
    case GDR_ERR_TIMEOUT: return "a bounded device wait gave up";
    case GDR_ERR_NONFINITE: return "non-finite input";
    case GDR_ERR_WORKSPACE: return "workspace smaller than the selected kernel needs";
    case GDR_ERR_SCRATCH_LIMIT:
        return "request needs more than the GDR_STATIC_SCRATCH_BYTES scratch of gdr_chunk_fwd_static";
    }
    return "unknown status";
}

int gdr_version(void) { return kVersion; }

}  // extern "C"
