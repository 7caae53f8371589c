// gdr_static.cu -- gdr_chunk_fwd_static: the two-pass tensor-core forward with
// its workspace in a fixed device array that belongs to this library, for
// callers that may not allocate device memory themselves.
//
// The array is GDR_STATIC_SCRATCH_BYTES long and 256-byte aligned.  Every GPU
// on which the library's device code is loaded keeps it until the process
// exits.  In host code its name only stands in for the symbol (it is not a
// device address), so the address the kernels receive comes from
// cudaGetSymbolAddress, asked again on every call with the caller's device
// current: the answer belongs to the device context current at that moment,
// and a remembered one could outlive its context (after cudaDeviceReset, or
// when the caller switches contexts).  The lookup allocates nothing.
#include <cstddef>

#include "gdr.h"
#include "gdr_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[GDR_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch in the current device context, or nullptr.
void *scratch_on_current_device()
{
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_static_scratch) != cudaSuccess)
        return nullptr;
    return addr;
}

}  // namespace

extern "C" gdr_status gdr_chunk_fwd_static(const gdr_shape *shape, const void *q, const void *k,
                                           const void *v, const float *g, const float *beta,
                                           const float *S0, int chunk, gdr_gate_mode gate_mode,
                                           gdr_inverse_mode inverse_mode, void *o, float *S_final,
                                           void *stream)
{
    if (shape == nullptr)
        return GDR_ERR_ARG;
    if (shape->kernel != GDR_KERNEL_AUTO && shape->kernel != GDR_KERNEL_TC2)
        return GDR_ERR_UNSUPPORTED;
    gdr_shape sh = *shape;
    sh.kernel = GDR_KERNEL_TC2;
    size_t need = 0;
    const gdr_status st = gdr_workspace_bytes(&sh, chunk, gate_mode, inverse_mode, &need);
    if (st != GDR_OK)
        return st;
    if (need > GDR_STATIC_SCRATCH_BYTES)
        return GDR_ERR_SCRATCH_LIMIT;
    void *scratch = scratch_on_current_device();
    if (scratch == nullptr)
        return GDR_ERR_CUDA;
    // The first pass writes every record the second pass reads, so whatever an
    // earlier call left in the array needs no clearing.
    return gdr_chunk_fwd(&sh, q, k, v, g, beta, S0, chunk, gate_mode, inverse_mode, o, S_final,
                         scratch, GDR_STATIC_SCRATCH_BYTES, stream);
}
