// gdr_simt.cu -- chunkwise gated delta-rule forward on the CUDA cores, in fp32.
//
// The general kernel of the library: any gate mode, any chunk length up to 128,
// fp32 or bf16 inputs, fp32 arithmetic throughout.  It is the fp32 path
// (spec tolerance 1e-4) and serves every request the tensor-core kernel
// does not take.  It follows the chunkwise WY algebra of "Systolic Linear
// Attention: Co-Designing Tile-Grouped Gated Delta Attention for TPUs"
// (§2.1 "Chunkwise WY parallelization", §2.3 Table 2, §2.4.2):
//   Lambda_t = cumsum g,  M_tj = 1[t>j] beta_j sum_i k_ti k_ji e^{Lambda_ti - Lambda_ji},
//   A = (I + M)^{-1},  E = diag(beta) A (V - Kbar S),  O = Qbar S + L E,
//   S <- F S + Khat^T E,
// with every decay factor formed as the exponential of a non-positive
// difference of cumulative log-decays (no division by decay prefixes).  The
// exact inverse is forward substitution in shared memory; the Neumann inverse
// follows "When Good Enough Is Optimal: Multiplication-Only Matrix Inversion
// Approximation for Quantized Gated DeltaNet" (masked powers, Lemma 3.1, then
// Newton residual corrections).
//
// With chunk-boundary momentum ("Systolic Linear Attention ...", §2.3) the state
// update of each chunk is blended with a velocity Z (zero at the start), kept
// beside S:
//   Z <- mu kappa_c Z + Khat^T E,  S <- F S + Z,
// where Khat^T E is exactly the plain update minus F S; the chunk's outputs are
// those of the plain chunk computation from the entry state.
//
// One CTA owns one value head and NV value columns; chunks run in order.  In the
// two-pass form (PRE) a first kernel computes every chunk's inverse and L at
// once, and this kernel reads them instead of recomputing them per value tile.
// With o == nullptr it only walks the states (writing the state at each chunk's
// start to S_chunks when given: the backward's recomputation).
#include <cuda_bf16.h>

#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int NT = 256;  // threads per CTA
constexpr int LB = 16;   // rows per row block (L readout, Neumann products)

struct SimtLayout {      // offsets in floats into dynamic shared memory
    int lam, A, P, X, S, rhs, qs, E, blk, beta, row, Z, total;
};

// Neumann mode keeps N (in A) and the series X; a third C x C buffer P is only
// needed for more than one residual step (the single-step correction writes
// its residual over N).  Q S (C x NV) is staged in X once X has been applied,
// when X is large enough to hold it (C >= NV).
__host__ __device__ inline SimtLayout simt_layout(int C, int G, int dk, bool neumann, int resid,
                                                  int NV, bool momentum)
{
    SimtLayout s;
    int off = 0;
    s.lam = off;  off += C * G;
    s.A = off;    off += C * C;
    s.X = off;    off += neumann ? C * C : 0;
    s.P = off;    off += (neumann && resid > 1) ? C * C : 0;
    s.S = off;    off += dk * NV;
    s.rhs = off;  off += C * NV;
    const bool qs_in_x = neumann && C >= NV;
    s.qs = qs_in_x ? s.X : off;
    off += qs_in_x ? 0 : C * NV;
    s.E = off;    off += C * NV;
    s.blk = off;  off += LB * C;
    s.beta = off; off += C;
    s.row = off;  off += C;
    s.Z = off;    off += momentum ? dk * NV : 0;   // momentum velocity, last
    s.total = off;
    return s;
}

template <bool BF>
__device__ __forceinline__ float ld_in(const void *p, long i)
{
    if constexpr (BF)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else
        return static_cast<const float *>(p)[i];
}

template <bool BF>
__device__ __forceinline__ void st_out(void *p, long i, float x)
{
    if constexpr (BF)
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else
        static_cast<float *>(p)[i] = x;
}

// The chunk's Gram M (strictly lower, beta on the column) into A and its inverse
// (I + M)^{-1}: forward substitution (exact), the truncated Neumann series with
// Newton residual steps, or the 1-Step Neumann in blocks of 16.  lam and sbeta
// hold the chunk's Lambda and beta.  Returns the array that holds the inverse (A,
// or X in Neumann mode); every thread of the CTA calls it, and it ends on a
// barrier.
template <bool IN_BF16>
__device__ const float *chunk_inverse(const Params &p, long kh, int c0, int Cl, const float *lam,
                                      const float *sbeta, float *A, float *X, float *P,
                                      float *blk, float *row)
{
    const int C = p.C, G = p.G, dk = p.dk, T = p.T;
    const int width = dk / G;
    const bool neu = p.neumann != 0;
    const bool blk1 = p.neumann1 != 0;
    const int tid = threadIdx.x;
    // --- Gram M (strictly lower, beta on the column) into A
    for (int idx = tid; idx < Cl * Cl; idx += NT) {
        const int t = idx / Cl, j = idx % Cl;
        float m = 0.f;
        if (j < t) {
            const long kt = (kh * T + c0 + t) * dk, kj = (kh * T + c0 + j) * dk;
            for (int gi = 0; gi < G; ++gi) {
                float s = 0.f;
                for (int i = gi * width; i < (gi + 1) * width; ++i)
                    s += ld_in<IN_BF16>(p.k, kt + i) * ld_in<IN_BF16>(p.k, kj + i);
                m += expf(lam[t * G + gi] - lam[j * G + gi]) * s;
            }
            m *= sbeta[j];
        }
        A[t * C + j] = m;
    }
    __syncthreads();
    // --- chunk inverse
    if (!neu) {
        // forward substitution in place: row t of M becomes row t of A.  For the
        // 1-Step Neumann inverse only within each 16-row diagonal block (the
        // exact D^{-1}); the blocks below keep M until the step after.
        for (int t = tid; t < Cl; t += NT)
            A[t * C + t] = 1.f;
        __syncthreads();
        for (int t = 1; t < Cl; ++t) {
            const int b0 = blk1 ? (t / 16) * 16 : 0;
            for (int j = b0 + tid; j < t; j += NT)
                row[j] = A[t * C + j];
            __syncthreads();
            for (int c = b0 + tid; c < t; c += NT) {
                float acc = -row[c];
                for (int j = c + 1; j < t; ++j)
                    acc -= row[j] * A[j * C + c];
                A[t * C + c] = acc;
            }
            __syncthreads();
        }
        if (blk1) {
            // ("Systolic Linear Attention ...", §2.4.3) A = (I - D^{-1} M_off) D^{-1}:
            // below the diagonal blocks A_ij = -D_ii^{-1} M_ij D_jj^{-1}; first
            // X = M_off D^{-1}, then A_off = -D^{-1} X (row i reads its own diagonal
            // block, which this step does not write)
            for (int idx = tid; idx < Cl * Cl; idx += NT) {
                const int i = idx / Cl, c = idx % Cl;
                if (c >= (i / 16) * 16)
                    continue;
                const int ce = min((c / 16) * 16 + 16, Cl);
                float acc = 0.f;
                for (int l = c; l < ce; ++l)
                    acc += A[i * C + l] * A[l * C + c];
                X[i * C + c] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < Cl * Cl; idx += NT) {
                const int i = idx / Cl, c = idx % Cl, b0 = (i / 16) * 16;
                if (c >= b0)
                    continue;
                float acc = 0.f;
                for (int l = b0; l <= i; ++l)
                    acc += A[i * C + l] * X[l * C + c];
                A[i * C + c] = -acc;
            }
            __syncthreads();
        }
    } else {
        // X0 = sum_{p<=m} (-N)^p, N = M (in A), by Horner's rule X <- I - N X
        // (m times from X = I).  N is strictly lower triangular, so row i of
        // N X reads only rows above i: the update runs in place, one row block
        // at a time from the bottom up.  This equals the sum of the masked
        // powers of N (the masks only drop entries that are exactly zero).
        for (int idx = tid; idx < Cl * Cl; idx += NT) {
            const int i = idx / Cl, j = idx % Cl;
            X[i * C + j] = (i == j) ? 1.f : 0.f;
        }
        __syncthreads();
        for (int pw = 1; pw <= p.neu_order; ++pw) {
            for (int r0 = ((Cl - 1) / LB) * LB; r0 >= 0; r0 -= LB) {
                const int nr = min(LB, Cl - r0);
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl, i = r0 + r;
                    float acc = (i == c) ? 1.f : 0.f;
                    for (int l = c; l < i; ++l)
                        acc -= A[i * C + l] * X[l * C + c];
                    blk[r * C + c] = acc;
                }
                __syncthreads();
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl;
                    X[(r0 + r) * C + c] = blk[r * C + c];
                }
                __syncthreads();
            }
        }
        for (int s = 0; s < p.neu_resid; ++s) {
            // residual Rm = I - (I + N) X; the last step may overwrite N
            float *Rm = (s + 1 < p.neu_resid) ? P : A;
            for (int r0 = 0; r0 < Cl; r0 += LB) {
                const int nr = min(LB, Cl - r0);
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl, i = r0 + r;
                    float acc = (i == c ? 1.f : 0.f) - X[i * C + c];
                    for (int l = c; l < i; ++l)
                        acc -= A[i * C + l] * X[l * C + c];
                    blk[r * C + c] = acc;
                }
                __syncthreads();
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl;
                    Rm[(r0 + r) * C + c] = blk[r * C + c];
                }
                __syncthreads();
            }
            // Newton correction X <- X + X Rm, one row block at a time
            for (int r0 = 0; r0 < Cl; r0 += LB) {
                const int nr = min(LB, Cl - r0);
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl, i = r0 + r;
                    float acc = X[i * C + c];
                    for (int l = c; l <= i; ++l)
                        acc += X[i * C + l] * Rm[l * C + c];
                    blk[r * C + c] = acc;
                }
                __syncthreads();
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, c = idx % Cl;
                    X[(r0 + r) * C + c] = blk[r * C + c];
                }
                __syncthreads();
            }
        }
    }
    return neu ? X : A;
}

template <bool IN_BF16, bool OUT_BF16, int NV, bool MOM, bool PRE>
__global__ void __launch_bounds__(NT) simt_fwd_kernel(const Params p)
{
    extern __shared__ float sm[];
    const int C = p.C, G = p.G, dk = p.dk, dv = p.dv, T = p.T;
    const bool neu = p.neumann != 0;
    const bool blk1 = p.neumann1 != 0;   // 1-Step Neumann: X is its scratch
    // (the two-pass form reads the inverse: no Neumann buffers)
    const SimtLayout Ly = simt_layout(C, G, dk, !PRE && (neu || blk1), PRE ? 0 : p.neu_resid, NV, MOM);
    float *lam = sm + Ly.lam, *A = sm + Ly.A, *P = sm + Ly.P, *X = sm + Ly.X;
    float *S = sm + Ly.S, *rhs = sm + Ly.rhs, *qs = sm + Ly.qs, *E = sm + Ly.E;
    float *blk = sm + Ly.blk, *sbeta = sm + Ly.beta, *row = sm + Ly.row;
    float *Z = sm + Ly.Z;   // momentum only

    const int tid = threadIdx.x;
    const int n0 = blockIdx.x * NV;           // first value column of this CTA
    const int hv = blockIdx.y, b = blockIdx.z;
    const int hk = hv / p.R;                  // key head read by this value head
    const int nv = min(NV, dv - n0);          // live columns of this CTA
    const long kh = (long)b * p.Hk + hk;      // key-head sequence
    const long vh = (long)b * p.Hv + hv;      // value-head sequence
    const int width = dk / G;                 // channels per decay group

    for (int idx = tid; idx < dk * NV; idx += NT) {
        const int i = idx / NV, n = idx % NV;
        S[idx] = (p.S0 != nullptr && n < nv) ? p.S0[(vh * dk + i) * dv + n0 + n] : 0.f;
        if constexpr (MOM)
            Z[idx] = 0.f;
    }

    for (int c0 = 0; c0 < T; c0 += C) {
        const int Cl = min(C, T - c0);        // a ragged last chunk is shorter
        __syncthreads();
        if (p.S_chunks != nullptr) {          // the chunk's entry state, for the backward
            float *dst = p.S_chunks + ((vh * ((T + C - 1) / C) + c0 / C) * dk) * (long)dv + n0;
            for (int idx = tid; idx < dk * NV; idx += NT) {
                const int i = idx / NV, n = idx % NV;
                if (n < nv)
                    dst[(long)i * dv + n] = S[idx];
            }
        }
        // --- write gates and cumulative log-decay Lambda (summed, per group)
        for (int t = tid; t < Cl; t += NT)
            sbeta[t] = p.beta[kh * T + c0 + t];
        for (int gi = tid; gi < G; gi += NT) {
            float acc = 0.f;
            for (int t = 0; t < Cl; ++t) {
                acc += p.g[(kh * T + c0 + t) * G + gi];
                lam[t * G + gi] = acc;
            }
        }
        __syncthreads();
        const float *Ai;
        if constexpr (PRE) {
            // two-pass form: the inverse comes from the first pass's record
            const float *src = p.factors + (kh * ((T + C - 1) / C) + c0 / C) * (2L * C * C);
            for (int idx = tid; idx < Cl * Cl; idx += NT) {
                const int t = idx / Cl, j = idx % Cl;
                A[t * C + j] = src[t * C + j];
            }
            __syncthreads();
            Ai = A;
        } else {
            Ai = chunk_inverse<IN_BF16>(p, kh, c0, Cl, lam, sbeta, A, X, P, blk, row);
        }
        // --- RHS = V - Kbar S, Kbar_t = k_t e^{Lambda_t}
        for (int idx = tid; idx < Cl * (NV / 8); idx += NT) {
            const int t = idx / (NV / 8), nb = (idx % (NV / 8)) * 8;
            float ar[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                ar[u] = 0.f;
            const long kt = (kh * T + c0 + t) * dk;
            for (int i = 0; i < dk; ++i) {
                const float kb = ld_in<IN_BF16>(p.k, kt + i) * expf(lam[t * G + i / width]);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    ar[u] += kb * S[i * NV + nb + u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int n = nb + u;
                const float vv = (n < nv) ? ld_in<IN_BF16>(p.v, (vh * T + c0 + t) * dv + n0 + n) : 0.f;
                rhs[t * NV + n] = vv - ar[u];
            }
        }
        __syncthreads();
        // --- E = diag(beta) A RHS
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int t = idx / NV, n = idx % NV;
            float acc = 0.f;
            for (int j = 0; j <= t; ++j)
                acc += Ai[t * C + j] * rhs[j * NV + n];
            E[t * NV + n] = sbeta[t] * acc;
        }
        __syncthreads();
        // --- outputs (skipped when only the chunk-start states are wanted: a uniform
        //     condition, so every thread takes the same barriers)
        if (p.o != nullptr) {
            // --- Qbar S, Qbar_t = q_t e^{Lambda_t} (staged in X in Neumann mode when it fits: X is spent)
            for (int idx = tid; idx < Cl * (NV / 8); idx += NT) {
                const int t = idx / (NV / 8), nb = (idx % (NV / 8)) * 8;
                float aq[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    aq[u] = 0.f;
                const long qt = (kh * T + c0 + t) * dk;
                for (int i = 0; i < dk; ++i) {
                    const float qb = ld_in<IN_BF16>(p.q, qt + i) * expf(lam[t * G + i / width]);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        aq[u] += qb * S[i * NV + nb + u];
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    qs[t * NV + nb + u] = aq[u];
            }
            __syncthreads();
            // --- O = Qbar S + L E, L formed one row block at a time
            for (int r0 = 0; r0 < Cl; r0 += LB) {
                const int nr = min(LB, Cl - r0);
                for (int idx = tid; idx < nr * Cl; idx += NT) {
                    const int r = idx / Cl, j = idx % Cl, t = r0 + r;
                    float l = 0.f;
                    if constexpr (PRE) {
                        if (j <= t)
                            l = p.factors[(kh * ((T + C - 1) / C) + c0 / C) * (2L * C * C) +
                                          (long)C * C + (long)t * C + j];
                    } else if (j <= t) {
                        const long qt = (kh * T + c0 + t) * dk, kj = (kh * T + c0 + j) * dk;
                        for (int gi = 0; gi < G; ++gi) {
                            float s = 0.f;
                            for (int i = gi * width; i < (gi + 1) * width; ++i)
                                s += ld_in<IN_BF16>(p.q, qt + i) * ld_in<IN_BF16>(p.k, kj + i);
                            l += expf(lam[t * G + gi] - lam[j * G + gi]) * s;
                        }
                    }
                    blk[r * C + j] = l;
                }
                __syncthreads();
                for (int idx = tid; idx < nr * NV; idx += NT) {
                    const int r = idx / NV, n = idx % NV, t = r0 + r;
                    if (n < nv) {
                        float acc = qs[t * NV + n];
                        for (int j = 0; j <= t; ++j)
                            acc += blk[r * C + j] * E[j * NV + n];
                        st_out<OUT_BF16>(p.o, (vh * T + c0 + t) * dv + n0 + n, acc);
                    }
                }
                __syncthreads();
            }
        }
        // --- S <- F S + Khat^T E,  F = e^{Lambda_C}, Khat_t = k_t e^{Lambda_C - Lambda_t}
        //     (momentum: Z <- mu kappa_c Z + Khat^T E, S <- F S + Z)
        float mk = 0.f;
        if constexpr (MOM) {
            const long nch = (T + C - 1) / C;
            mk = p.mu * (p.kappa != nullptr ? (float)p.kappa[(long)b * nch + c0 / C] : 1.f);
        }
        for (int idx = tid; idx < dk * (NV / 8); idx += NT) {
            const int i = idx / (NV / 8), nb = (idx % (NV / 8)) * 8;
            const float lc = lam[(Cl - 1) * G + i / width];
            const float f = expf(lc);
            float acc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                acc[u] = MOM ? 0.f : f * S[i * NV + nb + u];
            for (int t = 0; t < Cl; ++t) {
                const float w = ld_in<IN_BF16>(p.k, (kh * T + c0 + t) * dk + i) *
                                expf(lc - lam[t * G + i / width]);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    acc[u] += w * E[t * NV + nb + u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if constexpr (MOM) {
                    const float z = mk * Z[i * NV + nb + u] + acc[u];
                    Z[i * NV + nb + u] = z;
                    S[i * NV + nb + u] = f * S[i * NV + nb + u] + z;
                } else {
                    S[i * NV + nb + u] = acc[u];
                }
            }
        }
    }
    __syncthreads();
    if (p.S_final != nullptr)
        for (int idx = tid; idx < dk * NV; idx += NT) {
            const int i = idx / NV, n = idx % NV;
            if (n < nv)
                p.S_final[(vh * dk + i) * dv + n0 + n] = S[idx];
        }
}

// First pass of the two-pass form: one CTA per (batch, key head, chunk), all chunks
// at once, computes the chunk's inverse and its score matrix L (lower, with the
// diagonal) once for all value tiles and heads, into the record
// [A (C x C) | L (C x C)] fp32 of that chunk (rows and columns past a ragged
// chunk's length are left unwritten and never read).
template <bool IN_BF16>
__global__ void __launch_bounds__(NT) simt_factors_kernel(const Params p, float *rec)
{
    extern __shared__ float sm[];
    const int C = p.C, G = p.G, dk = p.dk, T = p.T;
    const SimtLayout Ly = simt_layout(C, G, dk, p.neumann != 0 || p.neumann1 != 0, p.neu_resid, 8,
                                      false);
    float *lam = sm + Ly.lam, *A = sm + Ly.A, *P = sm + Ly.P, *X = sm + Ly.X;
    float *blk = sm + Ly.blk, *sbeta = sm + Ly.beta, *row = sm + Ly.row;
    const int tid = threadIdx.x;
    const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const long kh = (long)b * p.Hk + hk;
    const int nch = (T + C - 1) / C;
    const int c0 = c * C, Cl = min(C, T - c0);
    const int width = dk / G;

    for (int t = tid; t < Cl; t += NT)
        sbeta[t] = p.beta[kh * T + c0 + t];
    for (int gi = tid; gi < G; gi += NT) {
        float acc = 0.f;
        for (int t = 0; t < Cl; ++t) {
            acc += p.g[(kh * T + c0 + t) * G + gi];
            lam[t * G + gi] = acc;
        }
    }
    __syncthreads();
    const float *Ai = chunk_inverse<IN_BF16>(p, kh, c0, Cl, lam, sbeta, A, X, P, blk, row);
    float *dst = rec + (kh * nch + c) * (2L * C * C);
    for (int idx = tid; idx < Cl * Cl; idx += NT) {
        const int t = idx / Cl, j = idx % Cl;
        dst[t * C + j] = Ai[t * C + j];
        float l = 0.f;
        if (j <= t) {
            const long qt = (kh * T + c0 + t) * dk, kj = (kh * T + c0 + j) * dk;
            for (int gi = 0; gi < G; ++gi) {
                float sum = 0.f;
                for (int i = gi * width; i < (gi + 1) * width; ++i)
                    sum += ld_in<IN_BF16>(p.q, qt + i) * ld_in<IN_BF16>(p.k, kj + i);
                l += expf(lam[t * G + gi] - lam[j * G + gi]) * sum;
            }
        }
        dst[(long)C * C + t * C + j] = l;
    }
}

template <bool I, bool O, int NV, bool MOM, bool PRE>
int launch_variant(const Params &p, int smem, cudaStream_t stream)
{
    auto kern = simt_fwd_kernel<I, O, NV, MOM, PRE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 6;  // GDR_ERR_CUDA
    dim3 grid((p.dv + NV - 1) / NV, p.Hv, p.B);
    kern<<<grid, NT, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

constexpr int kMaxSmem = 227 * 1024;

int smem_for(const Params &p, int NV, bool pre = false)
{
    return simt_layout(p.C, p.G, p.dk, !pre && (p.neumann != 0 || p.neumann1 != 0),
                       pre ? 0 : p.neu_resid, NV, p.momentum != 0).total *
           (int)sizeof(float);
}

// first pass of the two-pass form: the Neumann buffers, no value tile
int factors_smem(const Params &p)
{
    return simt_layout(p.C, p.G, p.dk, p.neumann != 0 || p.neumann1 != 0, p.neu_resid, 8, false)
               .total * (int)sizeof(float);
}

template <int NV, bool MOM, bool PRE>
int launch_io(const Params &p, int smem, cudaStream_t stream)
{
    if (p.in_bf16)
        return p.out_bf16 ? launch_variant<true, true, NV, MOM, PRE>(p, smem, stream)
                          : launch_variant<true, false, NV, MOM, PRE>(p, smem, stream);
    return p.out_bf16 ? launch_variant<false, true, NV, MOM, PRE>(p, smem, stream)
                      : launch_variant<false, false, NV, MOM, PRE>(p, smem, stream);
}

template <int NV>
int launch_nv(const Params &p, int smem, cudaStream_t stream)
{
    return p.momentum ? launch_io<NV, true, false>(p, smem, stream)
                      : launch_io<NV, false, false>(p, smem, stream);
}

template <int NV>
int launch_nv_pre(const Params &p, int smem, cudaStream_t stream)
{
    return launch_io<NV, false, true>(p, smem, stream);
}

int launch_factors(const Params &p, float *rec, cudaStream_t stream)
{
    const int smem = factors_smem(p);
    auto kern = p.in_bf16 ? simt_factors_kernel<true> : simt_factors_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 6;  // GDR_ERR_CUDA
    dim3 grid((p.T + p.C - 1) / p.C, p.Hk, p.B);
    kern<<<grid, NT, smem, stream>>>(p, rec);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace

// Shared memory of the widest value tile (32, else 16 columns) that fits.
int simt_smem_bytes(const Params &p)
{
    const int s32 = smem_for(p, 32);
    return s32 <= kMaxSmem ? s32 : smem_for(p, 16);
}

int launch_simt(const Params &p, cudaStream_t stream)
{
    const int s32 = smem_for(p, 32);
    if (s32 <= kMaxSmem)
        return launch_nv<32>(p, s32, stream);
    const int s16 = smem_for(p, 16);
    if (s16 <= kMaxSmem)
        return launch_nv<16>(p, s16, stream);
    return 5;  // GDR_ERR_UNSUPPORTED
}

// Two-pass form (no momentum): the chunk factors of every chunk in parallel, then
// the value tiles' pass over the chunks reading them.
bool simt2_supports(const Params &p)
{
    return p.momentum == 0 && factors_smem(p) <= kMaxSmem && smem_for(p, 16, true) <= kMaxSmem;
}

size_t simt2_workspace_bytes(const Params &p)
{
    return sizeof(float) * 2 * (size_t)p.C * p.C * (size_t)p.B * p.Hk * ((p.T + p.C - 1) / p.C);
}

int launch_simt2(const Params &p, void *workspace, cudaStream_t stream)
{
    if (p.T > 0) {   // no chunks, no first pass: the second copies S0 to S_final
        const int rc = launch_factors(p, static_cast<float *>(workspace), stream);
        if (rc != 0)
            return rc;
    }
    Params pre = p;
    pre.factors = static_cast<const float *>(workspace);
    const int s32 = smem_for(pre, 32, true);
    if (s32 <= kMaxSmem)
        return launch_nv_pre<32>(pre, s32, stream);
    const int s16 = smem_for(pre, 16, true);
    if (s16 <= kMaxSmem)
        return launch_nv_pre<16>(pre, s16, stream);
    return 5;  // GDR_ERR_UNSUPPORTED
}

}  // namespace gdr
