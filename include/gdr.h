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
 * no 1/sqrt(dk) query scale.
 *
 * Conventions shared by every entry point
 *  - Tensors are dense, row-major, contiguous, in the layouts given below.
 *    "Device pointer" means memory of the current CUDA device; the caller owns
 *    every buffer.  The library allocates no device memory on any call
 *    (tensor memory on chip is allocated and released inside each kernel).
 *  - Every device pointer must be 16-byte aligned (tensor-memory-access tile
 *    loads); otherwise GDR_ERR_ALIGN.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Arguments are validated on the host
 *    before anything is launched; on any error nothing is launched and the
 *    status says why.  No exception, abort or exit crosses the ABI.
 *  - Thread safety: calls may be issued from several host threads; the only
 *    library-global state is the device status word read by
 *    gdr_device_status().
 */
#ifndef GDR_H_
#define GDR_H_

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
    GDR_ERR_NONFINITE = 8    /* reserved: non-finite input detected            */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/* Decay groups G of the forget gate F_t (SLA §2.1 and §2.3):
 *  SCALAR  G = 1      one decay per head and token (GDN)
 *  GROUP64 G = dk/64  one decay per 64-channel tile (SLA); needs dk % 64 == 0
 *  CHANNEL G = dk     one decay per key channel (KDA)                       */
typedef enum { GDR_GATE_SCALAR = 0, GDR_GATE_GROUP64 = 1, GDR_GATE_CHANNEL = 2 } gdr_gate_mode;

/* Chunk inverse A_c = (I + M_c)^{-1}:
 *  EXACT   block-doubling inverse, exact up to rounding (SLA §2.4.3)
 *  NEUMANN sum_{p<=order} (-M)^p with masking, then `neumann_residual_steps`
 *          Newton residual corrections X <- X + X (I - (I + M) X)
 *          (Multiplication-Only Matrix Inversion ..., Lemma 3.1, §4.1)      */
typedef enum { GDR_INV_EXACT = 0, GDR_INV_NEUMANN = 1 } gdr_inverse_mode;

/* Kernel selection.  AUTO picks the tensor-core kernel whenever the request
 * is inside its envelope (bf16 inputs, dk in {64,128,256}, dv % 16 == 0,
 * chunk in {64,128}) and the CUDA-core kernel otherwise.  SIMT forces the
 * fp32 CUDA-core kernel; TC forces the tensor-core kernel and fails with
 * GDR_ERR_UNSUPPORTED outside its envelope.                                 */
typedef enum { GDR_KERNEL_AUTO = 0, GDR_KERNEL_SIMT = 1, GDR_KERNEL_TC = 2 } gdr_kernel;

typedef struct {
    int B;      /* batch, >= 0                                               */
    int T;      /* tokens per sequence, >= 0; any T (a ragged last chunk is
                   handled as a shorter chunk)                               */
    int Hk;     /* key heads, >= 1                                           */
    int Hv;     /* value heads, multiple of Hk; value head hv reads key head
                   hv / (Hv / Hk) (grouped value heads, SLA §2.4.1)          */
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
 * Returns GDR_OK once the work is queued on `stream`.  Kernel-side wait
 * timeouts are reported through gdr_device_status().
 */
gdr_status gdr_chunk_fwd(const gdr_shape *shape,
                         const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0,
                         int chunk, gdr_gate_mode gate_mode, gdr_inverse_mode inverse_mode,
                         void *o, float *S_final, void *stream);

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
 * synchronises.  `dev` must satisfy gdr_chunk_fwd's rules; host pointers
 * need no alignment.
 */
gdr_status gdr_chunk_fwd_host(const gdr_shape *shape, const gdr_io *host, const gdr_io *dev,
                              int chunk, gdr_gate_mode gate_mode,
                              gdr_inverse_mode inverse_mode, void *stream);

/* Which kernel gdr_chunk_fwd would launch for this request: GDR_KERNEL_SIMT or
 * GDR_KERNEL_TC, or a negative gdr_status value if it would be rejected. */
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

/* Synchronises `stream`, then returns and clears the device status word that
 * kernels set when a bounded wait gives up (GDR_OK or GDR_ERR_TIMEOUT), or
 * GDR_ERR_CUDA if the stream reported an error. */
gdr_status gdr_device_status(void *stream);

/* Static, NUL-terminated description of a status code. */
const char *gdr_status_string(gdr_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
