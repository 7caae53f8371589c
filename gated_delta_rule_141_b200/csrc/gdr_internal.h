// gdr_internal.h -- launch parameters shared by the C-ABI layer and the kernels
// of libgdr.so (not part of the public ABI).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace gdr {

// One validated gdr_chunk_fwd request, flattened for the kernels.
struct Params {
    int B, T, Hk, Hv, dk, dv;
    int G;          // decay groups: 1, dk/64 or dk
    int C;          // chunk length
    int R;          // value heads per key head
    int in_bf16;    // q, k, v are bf16 (else fp32)
    int out_bf16;   // o is bf16 (else fp32)
    int neumann;    // 0 exact inverse, 1 truncated Neumann
    int neumann1;   // 1-Step Neumann in blocks of 16 (neumann is 0 then)
    int pair;       // two-pass path: the request's chunk of 2C runs as pairs of C-token
                    // halves, the second half corrected by the pair's Y (internal)
    int wide_state; // two-pass path: 1 forces the 128-column state pass, 0 leaves it
                    // to the segment cost model
    int neu_order;  // Neumann order m
    int neu_resid;  // Newton residual corrections
    int momentum;   // chunk-boundary momentum (CUDA-core kernel only)
    float mu;       // momentum coefficient
    const int *kappa;  // [B][ceil(T / C)] momentum gates, or nullptr for ones
    const void *q, *k, *v;
    const float *g, *beta, *S0;
    void *o;          // may be nullptr for the CUDA-core kernel (states only)
    float *S_final;
    float *S_chunks;  // CUDA-core kernel: [B][Hv][ceil(T/C)][dk][dv] state at each chunk's start, or nullptr
    const float *factors;  // two-pass CUDA-core form: [B][Hk][ceil(T/C)][2][C][C] (inverse, L) records
    // backward (gdr_chunk_bwd): upstream gradients in, gradients out (fp32)
    const float *dO, *dS_final;
    float *grad_q, *grad_k, *grad_v, *grad_g, *grad_beta, *grad_S0;
};

// Status word that kernels set when a bounded wait gives up (0 = fine).  It
// lives in gdr_tc.cu, the translation unit whose kernels wait; this reads it
// (after the caller synchronised) and clears it.  Returns -1 on a CUDA error.
int read_and_clear_device_status();

// One warp that waits on an mbarrier nothing arrives on, for limit_ns, then sets
// the status word to the timeout code and releases its tensor memory.
int launch_wait_probe(uint64_t limit_ns, cudaStream_t stream);

// CUDA-core kernel (fp32 arithmetic).  Returns 0 on launch, or a gdr_status
// code if the request does not fit the kernel's shared-memory budget.
int simt_smem_bytes(const Params &p);
int launch_simt(const Params &p, cudaStream_t stream);
// Two-pass CUDA-core form: the chunk inverse and L of every chunk in parallel
// (into a workspace), then the value tiles' pass over the chunks.
bool simt2_supports(const Params &p);
size_t simt2_workspace_bytes(const Params &p);
int launch_simt2(const Params &p, void *workspace, cudaStream_t stream);

// Backward of the chunked forward (exact inverse), CUDA cores, fp32: the states
// at the chunk starts are recomputed by the forward kernel into the workspace,
// then one reverse sweep over the chunks per value tile.
size_t bwd_workspace_bytes(const Params &p);
int bwd_smem_bytes(const Params &p);
int launch_bwd(const Params &p, void *workspace, cudaStream_t stream);

// Tensor-core kernel (tcgen05 + TMEM + TMA, bf16 operands, fp32 accumulate).
bool tc_supports(const Params &p);
// Chunk length the tensor-core kernel actually blocks by (an exact-mode request
// for C = 128 runs on the C = 64 kernels).
int tc_kernel_chunk(const Params &p);
int launch_tc(const Params &p, cudaStream_t stream);

// Two-pass tensor-core path: the chunk-local factors of all chunks in parallel
// (written to a caller-owned workspace), then the state pass that reads them.
bool tc2_supports(const Params &p);
// ... with the 128-column state pass (GDR_KERNEL_TC2W)
bool tc2w_supports(const Params &p);
size_t tc2_workspace_bytes(const Params &p);
int launch_tc2(const Params &p, void *workspace, cudaStream_t stream);
// Segments per sequence of its state pass (1: sequential; more: segment-parallel).
int tc2_state_segments(const Params &p);

// The first pass alone, at the requested chunk length (public gdr_chunk_prepare).
bool prepare_supports(const Params &p);
size_t prepare_bytes(const Params &p);
int launch_prepare(const Params &p, void *out, cudaStream_t stream);

}  // namespace gdr
