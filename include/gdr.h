/*
 * gdr.h -- C ABI of libgdr.so: the chunkwise-parallel forward pass of gated
 * delta-rule linear attention on an NVIDIA B200 (sm_100a).
 *
 * The operation ("Systolic Linear Attention: Co-Designing Tile-Grouped Gated
 * Delta Attention for TPUs", §2.1 Eq. (2); §2.3 Table 2):
 *
 *     S_t = (I - beta_t k_t k_t^T) F_t S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,              F_t = diag(exp(g_t)) expanded to dk channels,
 *
 * computed chunk by chunk (chunk length C): inside a chunk the strictly
 * lower-triangular system (I + M_c)^{-1} is solved with block matrix products,
 * exactly (block doubling, §2.4.3) or by a truncated Neumann series with
 * structural masking and residual correction ("When Good Enough Is Optimal:
 * Multiplication-Only Matrix Inversion Approximation for Quantized Gated
 * DeltaNet", Lemma 3.1); the state S stays on chip across chunks.  There is
 * no 1/sqrt(dk) query scale.  Beside the forward: its gradients
 * (gdr_chunk_bwd, the custom-VJP backward of §2.5), the forward with
 * chunk-boundary momentum (gdr_chunk_fwd_momentum, §2.3) and the readout
 * epilogue (gdr_output_gate_rmsnorm, §2.3 Eq. (5)).
 *
 * Conventions shared by every entry point
 *  - Tensors are dense, row-major, contiguous, in the layouts given below.
 *    "Device pointer" means memory of the current CUDA device; the caller owns
 *    every buffer.  The library allocates no device memory on any call
 *    (tensor memory on chip is allocated and released inside each kernel).
 *  - Every device pointer must be 16-byte aligned (tensor-memory-access tile
 *    loads); otherwise GDR_ERR_ALIGN.  (The int32 kappa of
 *    gdr_chunk_fwd_momentum needs 4 bytes.)
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Arguments are validated on the host
 *    before anything is launched; on any error nothing is launched and the
 *    status says why.  No exception, abort or exit crosses the ABI.
 *  - Thread safety: calls may be issued from several host threads; the
 *    library-global state is the device status word read by
 *    gdr_device_status() and the fixed scratch array of gdr_chunk_fwd_static
 *    (calls of that entry point that overlap on the GPU race on it).
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_ARG = 1,         /* NULL pointer where data is required, bad enum  */
    GDR_ERR_SHAPE = 2,       /* sizes outside the supported envelope           */
    GDR_ERR_DTYPE = 3,       /* unsupported dtype combination                  */
    GDR_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned               */
    GDR_ERR_UNSUPPORTED = 5, /* valid request no kernel here implements        */
    GDR_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed           */
    GDR_ERR_TIMEOUT = 7,     /* a bounded on-device wait gave up               */
    GDR_ERR_NONFINITE = 8,   /* reserved: non-finite input detected            */
    GDR_ERR_WORKSPACE = 9,   /* workspace smaller than the selected kernel needs */
    GDR_ERR_SCRATCH_LIMIT = 10 /* request needs more scratch than
                                  gdr_chunk_fwd_static's fixed array holds      */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/* Decay groups G of the forget gate F_t (SLA §2.1 and §2.3):
 *  SCALAR  G = 1      one decay per head and token (GDN)
 *  GROUP64 G = dk/64  one decay per 64-channel tile (SLA); needs dk % 64 == 0
 *  CHANNEL G = dk     one decay per key channel (KDA)                       */
typedef enum { GDR_GATE_SCALAR = 0, GDR_GATE_GROUP64 = 1, GDR_GATE_CHANNEL = 2 } gdr_gate_mode;

/* Chunk inverse A_c = (I + M_c)^{-1}:
 *  EXACT    block-doubling inverse, exact up to rounding (SLA §2.4.3)
 *  NEUMANN  sum_{p<=order} (-M)^p with masking, then `neumann_residual_steps`
 *           Newton residual corrections X <- X + X (I - (I + M) X)
 *           (Multiplication-Only Matrix Inversion ..., Lemma 3.1, §4.1)
 *  NEUMANN1 1-Step Neumann (SLA §2.4.3): with D the block-diagonal part of
 *           I + M in blocks of 16 rows and N = D^{-1} M_off, A = (I - N) D^{-1}
 *           (exact on the diagonal blocks and the first block below them);
 *           depends on the chunk length, which is never re-blocked          */
typedef enum { GDR_INV_EXACT = 0, GDR_INV_NEUMANN = 1, GDR_INV_NEUMANN1 = 2 } gdr_inverse_mode;

/* Kernel selection.
 *  TC    one fused tensor-core kernel per (batch, value head, 64 value
 *        columns) that walks the chunks in order (bf16 inputs, dk in
 *        {64,128,256}, dv % 64 == 0, chunk 64, or 128 in exact mode).
 *  TC2   two tensor-core passes: the chunk-local factors of every chunk in
 *        parallel (gdr_chunk_prepare), written to the caller's workspace, then
 *        the state pass that reads them (bf16 inputs, dk = 128 with any gate
 *        grouping or dk = 256 with grouped / per-channel gates, dv % 64 == 0,
 *        chunk 64 or 128, every inverse mode).  Needs gdr_workspace_bytes() of
 *        device workspace.  For few long sequences its state pass runs
 *        segment-parallel, with 128 value columns per CTA when that is the
 *        cheaper.
 *  TC2W  TC2 with the 128-column state pass forced (grouped / per-channel
 *        gates, dk = 128, dv % 128 == 0, every inverse mode: the chunk-128
 *        Neumann inverses as corrected pairs of 64-token halves; no momentum):
 *        a test and benchmark switch; gdr_select_kernel reports TC2 for what
 *        AUTO picks.
 *  SIMT  the fp32 CUDA-core kernel (any dtype, chunk 1..128).
 *  SIMT2 the same arithmetic in two passes: the chunk inverse and score matrix
 *        L of every chunk in parallel, written to the caller's workspace
 *        (2 C^2 fp32 per (batch, key head, chunk); gdr_workspace_bytes), then
 *        the value tiles' pass over the chunks that reads them.  Only when
 *        forced; any dtype, chunk 1..128, every inverse mode.
 *  AUTO  TC2 when it applies and the call's workspace is large enough, else
 *        TC when it applies, else SIMT.  Forcing a kernel outside its
 *        envelope fails with GDR_ERR_UNSUPPORTED.                           */
typedef enum { GDR_KERNEL_AUTO = 0, GDR_KERNEL_SIMT = 1, GDR_KERNEL_TC = 2,
               GDR_KERNEL_TC2 = 3, GDR_KERNEL_SIMT2 = 4, GDR_KERNEL_TC2W = 5 } gdr_kernel;

/* Shape of a request.  Besides the per-field ranges, B * Hv must be below 2^31
 * and B * T * (Hk dk + Hv dv) must not exceed 2^40 elements (GDR_ERR_SHAPE
 * otherwise). */
typedef struct {
    int B;      /* batch, 0..65535                                           */
    int T;      /* tokens per sequence, >= 0; any T (a ragged last chunk is
                   handled as a shorter chunk)                               */
    int Hk;     /* key heads, >= 1                                           */
    int Hv;     /* value heads, multiple of Hk, at most 65535; value head hv
                   reads key head hv / (Hv / Hk) (grouped value heads,
                   SLA §2.4.1)                                               */
    int dk;     /* key width, 1..256                                         */
    int dv;     /* value width per value head, 1..256                        */
    gdr_dtype in_dtype;   /* dtype of q, k, v                                */
    gdr_dtype out_dtype;  /* dtype of o                                      */
    int neumann_order;            /* NEUMANN only, >= 0 (4 in the workloads) */
    int neumann_residual_steps;   /* NEUMANN only, >= 0 (1 in the workloads) */
    gdr_kernel kernel;            /* normally GDR_KERNEL_AUTO                */
} gdr_shape;

/*
 * gdr_chunk_fwd -- one chunkwise forward pass over all (batch, head) pairs.
 *
 * Device inputs (read only):
 *   q, k   [B, Hk, T, dk]  in_dtype
 *   v      [B, Hv, T, dv]  in_dtype
 *   g      [B, Hk, T, G]   fp32 log forget gate (alpha = exp(g), normally g <= 0;
 *                          G per gate_mode)
 *   beta   [B, Hk, T]      fp32 write gate, shared by the value heads of a key head
 *   S0     [B, Hv, dk, dv] fp32 initial state, or NULL for a zero state
 * Device outputs (written):
 *   o      [B, Hv, T, dv]  out_dtype
 *   S_final[B, Hv, dk, dv] fp32 state after token T, or NULL to skip
 * chunk: chunk length C, 1..128 (see gdr_kernel_chunk for the blocking used).
 * workspace, workspace_bytes: device scratch for the TC2 kernel (see
 *   gdr_workspace_bytes), or NULL, 0; the one-pass kernels use none.
 * Returns GDR_OK once the work is queued on `stream`.  Kernel-side wait
 * timeouts are reported through gdr_device_status().
 */
gdr_status gdr_chunk_fwd(const gdr_shape *shape,
                         const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0,
                         int chunk, gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode,
                         void *o, float *S_final,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr_chunk_bwd -- gradients of the chunkwise forward (exact chunk inverse):
 * given the upstream gradients dO of o and dS_final of S_final, the gradients
 * of sum(dO * o) + sum(dS_final * S_final) with respect to every input
 * ("Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta Attention
 * for TPUs", §2.5: only the state at each chunk's start is kept, and a reverse
 * scan over the chunks recomputes the chunk's factors from it).
 * Device inputs (read only): q, k, v, g, beta, S0 as gdr_chunk_fwd (S0 may be
 *   NULL: zero initial state);
 *   dO       [B, Hv, T, dv]  fp32
 *   dS_final [B, Hv, dk, dv] fp32, or NULL for zero
 * Device outputs (written, fp32): dq, dk [B, Hk, T, dk]; dv [B, Hv, T, dv];
 *   dg [B, Hk, T, G]; dbeta [B, Hk, T]; dS0 [B, Hv, dk, dv] or NULL to skip.
 *   The key-side gradients (dq, dk, dg, dbeta) sum the contributions of all
 *   value heads of a key head, added with fp32 atomics: their last bits may
 *   differ from run to run.
 * workspace: at least gdr_bwd_workspace_bytes (the fp32 state at the start of
 *   every chunk, [B, Hv, ceil(T / chunk), dk, dv]); GDR_ERR_WORKSPACE if
 *   smaller.  shape->in_dtype gives the dtype of q, k, v; out_dtype is unused.
 * Runs on the CUDA cores (fp32): shape->kernel AUTO or SIMT (otherwise
 * GDR_ERR_UNSUPPORTED, as for a request whose shared memory does not fit,
 * e.g. dk = 256 with per-channel gates at chunk 128).  Asynchronous on
 * `stream`.
 */
gdr_status gdr_chunk_bwd(const gdr_shape *shape,
                         const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0,
                         const float *dO, const float *dS_final,
                         int chunk, gdr_gate_mode gate_mode,
                         float *dq, float *dk, float *dv, float *dg, float *dbeta,
                         float *dS0, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes gdr_chunk_bwd needs for this request (into *bytes). */
gdr_status gdr_bwd_workspace_bytes(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                                   size_t *bytes);

/*
 * gdr_chunk_fwd_momentum -- gdr_chunk_fwd with chunk-boundary momentum
 * ("Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta Attention
 * for TPUs", §2.3, the momentum update after Eq. (5)).  Each chunk's state
 * update is blended with a velocity buffer Z that starts at zero:
 *   Z_c = mu kappa_c Z_{c-1} + (S~_c - F_c S_{c-1}),  S_c = F_c S_{c-1} + Z_c,
 * with S~_c the plain chunk update from S_{c-1} and F_c the chunk's total decay;
 * the outputs of chunk c are those of the plain chunk computation from S_{c-1}.
 * Inputs, outputs and chunk / gate / inverse arguments as gdr_chunk_fwd, plus:
 *   mu     momentum coefficient (finite; mu = 0 gives gdr_chunk_fwd's result)
 *   kappa  [B, ceil(T / chunk)] int32 device array of per-chunk gates on the
 *          carried velocity (0 where a document reset falls in the chunk), or
 *          NULL for ones; 4-byte aligned (GDR_ERR_ALIGN otherwise)
 * Chunks are taken at exactly `chunk` tokens (no re-blocking).  Kernels:
 * TC2 (bf16 inputs, dk = 128, dv % 64 == 0, chunk 64, any gate grouping and
 * inverse; the velocity is one more fp32 tensor-memory tile of the state pass,
 * which then walks every sequence whole) when shape->kernel is AUTO or TC2 and
 * the call brings gdr_workspace_bytes() of workspace for the same request;
 * otherwise the CUDA-core kernel (fp32 arithmetic; SIMT forces it), whose
 * velocity takes one more dk x 32 fp32 tile of shared memory (a request that
 * then does not fit returns GDR_ERR_UNSUPPORTED).  Other kernels:
 * GDR_ERR_UNSUPPORTED.  The velocity is not returned.  Asynchronous on `stream`.
 */
gdr_status gdr_chunk_fwd_momentum(const gdr_shape *shape,
                                  const void *q, const void *k, const void *v,
                                  const float *g, const float *beta, const float *S0,
                                  int chunk, gdr_gate_mode gate_mode,
                                  gdr_inverse_mode inverse_mode, float mu,
                                  const int32_t *kappa, void *o, float *S_final,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace (bytes) that gdr_chunk_fwd needs for this request with the
 * kernel AUTO or shape->kernel selects when given enough: 0 for the one-pass
 * kernels; for TC2, B * Hk * ceil(T / 64) records of 33296 bytes (scalar gate)
 * or 66048 bytes (grouped / per-channel gates): the chunk factors T and L plus
 * the decayed operands and decay factors the second pass reads.  The truncated
 * Neumann inverse at chunk 128 runs as pairs of 64-token halves, and its records
 * carry the pair correction and its inputs: 16384 more bytes (scalar gate) or
 * 32768 more (grouped / per-channel gates).  When the
 * sequences are few and long enough that the state pass runs segment-parallel
 * (each sequence cut into segments whose state maps are composed), three
 * fp32 states per segment and head (end state, start state: dk x dv per value
 * head; transition: dk x dk per key head) follow the records, 256-byte
 * aligned.  The caller allocates it (16-byte aligned) and passes it with its
 * size; its contents on entry do not matter.  A call
 * whose workspace is smaller falls back (AUTO) or fails with
 * GDR_ERR_WORKSPACE (TC2 forced).  Calls that share a workspace must not
 * overlap on the GPU. */
gdr_status gdr_workspace_bytes(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                               gdr_inverse_mode inverse_mode, size_t *bytes);

/*
 * gdr_chunk_prepare -- the chunk-local factors of every chunk, all chunks in
 * parallel (the first pass of TC2).  Per (b, hk, chunk n) of C = 64 tokens,
 * with Lambda = cumsum of g inside the chunk and decays exp(Lambda_t - Lambda_j):
 *   L_tj = (t >= j) sum_i q_ti k_ji exp(Lambda_ti - Lambda_ji)
 *   M_tj = (t >  j) beta_j sum_i k_ti k_ji exp(Lambda_ti - Lambda_ji)
 *   T    = diag(beta) (I + M)^{-1}  (exact or Neumann, as inverse_mode)
 * (SLA §2.1, §2.3 Table 2; rows past T are zero).
 * Output `factors` (device, written): [B][Hk][ceil(T/64)] records of 16384
 * bytes: T then L, each a 64 x 64 bf16 matrix stored as 64 rows of 128 bytes
 * in which the 16-byte piece holding columns 8c..8c+7 of row r sits at
 * position (c XOR (r mod 8)) -- the 128-byte-swizzled tile layout.
 * factors_bytes must be at least B * Hk * ceil(T/64) * 16384.  Needs bf16
 * q, k, dk in {128, 256} and chunk 64; q, k, g, beta as for gdr_chunk_fwd.
 */
gdr_status gdr_chunk_prepare(const gdr_shape *shape, const void *q, const void *k,
                             const float *g, const float *beta, int chunk,
                             gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode,
                             void *factors, size_t factors_bytes, void *stream);

/* Buffers of one call, either all on the host or all on the device. */
typedef struct {
    const void *q, *k, *v;
    const float *g, *beta, *S0;   /* S0 may be NULL                          */
    void *o;
    float *S_final;               /* may be NULL                             */
} gdr_io;

/*
 * gdr_chunk_fwd_host -- the same pass for inputs and outputs in host memory.
 * Copies `host`'s inputs into the caller-owned device buffers `dev`
 * (cudaMemcpyAsync, one copy per tensor; pinned host memory makes them
 * asynchronous), runs gdr_chunk_fwd on them and copies o and S_final back to
 * `host`, all on `stream`.  The host outputs are valid after the stream
 * synchronises.  `dev` and the device `workspace` must satisfy
 * gdr_chunk_fwd's rules; host pointers need no alignment.
 */
gdr_status gdr_chunk_fwd_host(const gdr_shape *shape, const gdr_io *host, const gdr_io *dev,
                              int chunk, gdr_gate_mode gate_mode,
                              gdr_inverse_mode inverse_mode,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Size of the device array gdr_chunk_fwd_static uses as its workspace. */
#define GDR_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * gdr_chunk_fwd_static -- gdr_chunk_fwd on the TC2 kernel, with no workspace
 * argument: for callers that may not allocate device memory on their call
 * path, such as a serving engine whose memory planner owns all device memory
 * once it has started, or a latency-critical loop that cannot afford the
 * device-wide synchronisation an allocation can cause.  (The paper has no
 * counterpart; this is a deployment convenience of this library.)
 *
 * Arguments, layouts, alignment and errors are those of gdr_chunk_fwd, with
 * shape->kernel AUTO or TC2 (anything else: GDR_ERR_UNSUPPORTED; requests
 * outside TC2's envelope fail as a forced TC2 call does).  The workspace is a
 * fixed array of GDR_STATIC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library's device code holds until the process exits; a
 * request whose TC2 workspace (gdr_workspace_bytes) is larger fails with
 * GDR_ERR_SCRATCH_LIMIT before anything is launched.  Nothing is allocated:
 * no cudaMalloc, no cudaFree, no allocating library call.
 *  - Set-up: every call looks up the array's device address in the device
 *    context current at that moment (cudaGetSymbolAddress, which allocates
 *    nothing), so the address is never stale after a cudaDeviceReset or a
 *    context switch.  The first call on a device can load the library's
 *    device code there; make that first call before any stream capture.
 *  - Sharing: every call on a device uses the same array, which keeps what the
 *    last call left there.  Nothing in it needs clearing between calls (each
 *    call rewrites all it reads), but two calls that overlap on the GPU (other
 *    streams, other host threads) race on it: order them on one stream or
 *    synchronise between them.
 */
gdr_status gdr_chunk_fwd_static(const gdr_shape *shape,
                                const void *q, const void *k, const void *v,
                                const float *g, const float *beta, const float *S0,
                                int chunk, gdr_gate_mode gate_mode,
                                gdr_inverse_mode inverse_mode,
                                void *o, float *S_final, void *stream);

/* Which kernel gdr_chunk_fwd would launch for this request when given the
 * workspace gdr_workspace_bytes asks for: GDR_KERNEL_SIMT, GDR_KERNEL_TC,
 * GDR_KERNEL_TC2 or GDR_KERNEL_SIMT2, or a negative gdr_status value if it
 * would be rejected. */
int gdr_select_kernel(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                      gdr_inverse_mode inverse_mode);

/* Chunk length the kernel selected for this request actually blocks by, or a
 * negative gdr_status value if the request would be rejected.  It equals
 * `chunk` except on the tensor-core kernel in exact mode, where chunk 128 runs
 * as chunk 64: the exact chunkwise form equals the token recurrence for any
 * chunk length (WY representation of the SLA paper, §2.4.2), so the result is
 * the same function up to rounding.  The truncated Neumann inverse depends on
 * the chunk length and is never re-blocked. */
int gdr_kernel_chunk(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                     gdr_inverse_mode inverse_mode);

/* Segments per sequence of the TC2 state pass for this request, when TC2 is
 * the kernel selected given the workspace gdr_workspace_bytes asks for: 1 when
 * the pass walks every sequence whole (one launch after the first pass); n > 1
 * when few long sequences are each cut into n segments whose state maps
 * S -> A S + B are formed in parallel, composed in order and applied (three
 * launches after the first pass; an affine two-level scan of the chunk
 * recurrence); 0 when another kernel is selected; a negative gdr_status value
 * if the request would be rejected.  Host only, no GPU work. */
int gdr_state_segments(const gdr_shape *shape, int chunk, gdr_gate_mode gate_mode,
                       gdr_inverse_mode inverse_mode);

/*
 * gdr_output_gate_rmsnorm -- the readout epilogue of the SLA recurrence (SLA
 * §2.3 Eq. (5)), in place on the output of gdr_chunk_fwd:
 *   o_{t,m} <- sigmoid(z_{t,m}) * o_{t,m} / sqrt(mean_i o_{t,m,i}^2 + eps) * weight
 * for every (batch, value head m, token t) row of dv channels.
 *   o      [B, Hv, T, dv] out_dtype, device, read and written
 *   z      [B, Hv, T, dv] out_dtype output-gate logits, device, read only
 *   weight [dv] fp32 per-channel RMSNorm weight shared by the value heads, or
 *          NULL for ones; device, read only
 *   eps    >= 0 (1e-6 is usual)
 * Uses B, T, Hv, dv and out_dtype of `shape` (dv <= 256).  Statistics in fp32.
 * Asynchronous on `stream`; validation happens before any launch (GDR_ERR_ARG
 * for NULL o or z or a bad eps, GDR_ERR_SHAPE, GDR_ERR_DTYPE).
 */
gdr_status gdr_output_gate_rmsnorm(const gdr_shape *shape, void *o, const void *z,
                                   const float *weight, float eps, void *stream);

/* Synchronises `stream`, then returns and clears the device status word that
 * kernels set when a bounded wait gives up (GDR_OK or GDR_ERR_TIMEOUT), or
 * GDR_ERR_CUDA if the stream reported an error. */
gdr_status gdr_device_status(void *stream);

/*
 * gdr_selftest_bounded_wait -- test of the failure path of the kernels'
 * bounded waits (no counterpart in the pages; a diagnostic of this library).
 * Launches one warp on `stream` that takes tensor memory, waits on an
 * mbarrier nothing arrives on, gives up after limit_ns nanoseconds of wall
 * time (1e3 .. 1e9, else GDR_ERR_ARG), sets the status word that
 * gdr_device_status() reports as GDR_ERR_TIMEOUT, releases the tensor memory
 * and returns: the CUDA context stays usable.  No forward entry point
 * reaches it.
 */
gdr_status gdr_selftest_bounded_wait(uint64_t limit_ns, void *stream);

/* Static, NUL-terminated description of a status code. */
const char *gdr_status_string(gdr_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
