// gdr_bwd.cu -- backward of the chunkwise gated delta-rule forward (exact chunk
// inverse), on the CUDA cores in fp32.
//
// "Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta Attention for
// TPUs" (§2.5, custom VJP) keeps only the state at each chunk's start and, in a
// reverse scan over the chunks, recomputes the chunk's factors and back-propagates
// through them.  Here the forward kernel (gdr_simt.cu) writes those states into
// the workspace, then one CTA per (batch, value head, NV value columns) runs the
// chunks backwards with its tile of dS (the gradient of the state) in shared
// memory.  With the chunk's forward in the notation of gdr_simt.cu
//   P_tj = 1[t>j] sum_i k_ti k_ji e^{Lambda_ti - Lambda_ji},  M_tj = beta_j P_tj,
//   A = (I + M)^{-1},  R = V - Kbar S,  Y = A R,  E = diag(beta) Y,
//   L_tj = 1[t>=j] sum_i q_ti k_ji e^{Lambda_ti - Lambda_ji},
//   O = Qbar S + L E,  S' = F S + Khat^T E,
// and upstream gradients dO, dS', the chunk's gradients are
//   dE = L^T dO + Khat dS',  dY = diag(beta) dE,  dR = A^T dY,  dV = dR,
//   dM = -(dR Y^T) on t > j       (A^T dY Y^T, since dA^{-1} = -A dM A),
//   dL = dO E^T on t >= j,  dQbar = dO S^T,  dKbar = -dR S^T,  dKhat = E dS'^T,
//   dbeta_t = sum_n dE_tn Y_tn + sum_{t'>t} dM_t't P_t't,
//   dS = F dS' + Qbar^T dO - Kbar^T dR,
// and the pair sums of P and L give dq, dk and dLambda per channel with every
// decay factor an exponential of a non-positive difference.  dg is the reverse
// cumulative sum of dLambda inside the chunk (Lambda restarts at every chunk)
// plus, at every token, the gradient of the chunk-end decay Lambda_C, which is
// sum_n dS'_in S'_in per channel i.
//
// Key-side gradients (dq, dk, dg, dbeta) are sums over the value tiles and the
// value heads of a key head; each CTA adds its part with fp32 atomics (the
// order of those additions is not fixed).  dv and dS0 are written directly.
#include <cuda_bf16.h>

#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int NT = 256;  // threads per CTA

struct BwdLayout {       // offsets in floats into dynamic shared memory
    int lam, beta, row, P, A, L, S, dS, Y, dO, dE, dR, DL, DLg, F, X, E1, qk, ldq, total;
    bool tab;            // scalar gate: e^{Lambda_t - Lambda_j} (C x C) and e^{Lambda_t} (C)
                         // tabulated in E1
    bool stage;          // the chunk's q and k rows staged at qk (row stride ldq elements)
};

constexpr int kBwdSmemFloats = 227 * 1024 / 4;

// in_bytes: the size of an input element (2 for bf16 q, k, v; 4 for fp32)
__host__ __device__ inline BwdLayout bwd_layout(int C, int G, int dk, int NV, int in_bytes)
{
    BwdLayout s;
    int off = 0;
    s.lam = off;  off += C * G;
    s.beta = off; off += C;
    s.row = off;  off += C;
    s.P = off;    off += C * C;     // P (no beta)
    s.A = off;    off += C * C;     // M, then A = (I + M)^{-1}, then dM
    s.L = off;    off += C * C;     // L, then dL
    s.S = off;    off += dk * NV;   // state at the chunk's start
    s.dS = off;   off += dk * NV;   // gradient of the state after the chunk, then before it
    s.Y = off;    off += C * NV;    // Y = A R
    s.dO = off;   off += C * NV;
    s.dE = off;   off += C * NV;    // dE, then dY = beta dE
    s.dR = off;   off += C * NV;    // R, then dR
    s.DL = off;   off += C * dk;    // dLambda per (token, channel)
    s.DLg = off;  off += (G < dk) ? C * G : 0;   // dLambda per (token, group)
    s.F = off;    off += dk;        // e^{Lambda_C} per channel
    s.X = off;    off += dk;        // gradient of Lambda_C per channel
    // scalar gate: the pair factors depend on (t, j) only; tabulate them when
    // they fit beside the rest (last, so the other offsets do not move)
    s.tab = G == 1 && off + C * C + C <= kBwdSmemFloats;
    s.E1 = off;   off += s.tab ? C * C + C : 0;
    // the chunk's q and k rows in the input type, when they fit: every product of the chunk
    // reads them 2 C to dk times, from here instead of global memory (rows padded by one
    // word, so that a warp reading one column of many rows meets every bank once)
    s.ldq = dk + 4 / in_bytes;
    const int qk_floats = (2 * C * s.ldq * in_bytes + 3) / 4;
    s.qk = off;
    s.stage = off + qk_floats <= kBwdSmemFloats;
    off += s.stage ? qk_floats : 0;
    s.total = off;
    return s;
}

template <bool BF> struct InElem { using type = float; };
template <> struct InElem<true> { using type = __nv_bfloat16; };
__device__ __forceinline__ float in_f(float x) { return x; }
__device__ __forceinline__ float in_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <bool BF>
__device__ __forceinline__ float ld_in(const void *p, long i)
{
    if constexpr (BF)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else
        return static_cast<const float *>(p)[i];
}

__global__ void __launch_bounds__(NT) zero_kernel(float *a, long n)
{
    for (long i = (long)blockIdx.x * NT + threadIdx.x; i < n; i += (long)gridDim.x * NT)
        a[i] = 0.f;
}

template <bool IN_BF16, int NV>
__global__ void __launch_bounds__(NT) simt_bwd_kernel(const Params p)
{
    extern __shared__ float sm[];
    const int C = p.C, G = p.G, dk = p.dk, dv = p.dv, T = p.T;
    const BwdLayout Ly = bwd_layout(C, G, dk, NV, IN_BF16 ? 2 : 4);
    float *lam = sm + Ly.lam, *sbeta = sm + Ly.beta, *row = sm + Ly.row, *P = sm + Ly.P;
    float *A = sm + Ly.A, *L = sm + Ly.L, *S = sm + Ly.S, *dS = sm + Ly.dS, *Y = sm + Ly.Y;
    float *dO = sm + Ly.dO, *dE = sm + Ly.dE, *dR = sm + Ly.dR, *DL = sm + Ly.DL;
    float *Fv = sm + Ly.F, *X = sm + Ly.X, *E1 = sm + Ly.E1;
    const bool tab = Ly.tab;
    float *Et = E1 + C * C;                   // tab: e^{Lambda_t}
    const int width = dk / G;                 // channels per decay group
    float *DLg = width > 1 ? sm + Ly.DLg : DL;   // per group (the same array when G = dk)
    using In = typename InElem<IN_BF16>::type;
    In *qs = reinterpret_cast<In *>(sm + Ly.qk);
    In *ks = qs + C * Ly.ldq;
    const bool st = Ly.stage;
    const int ldq = Ly.ldq;

    const int tid = threadIdx.x;
    const int n0 = blockIdx.x * NV;
    const int hv = blockIdx.y, b = blockIdx.z;
    const int hk = hv / p.R;
    const int nv = min(NV, dv - n0);
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int nch = (T + C - 1) / C;

    for (int idx = tid; idx < dk * NV; idx += NT) {
        const int i = idx / NV, n = idx % NV;
        dS[idx] = (p.dS_final != nullptr && n < nv) ? p.dS_final[(vh * dk + i) * dv + n0 + n] : 0.f;
    }

    for (int c = nch - 1; c >= 0; --c) {
        const int c0 = c * C;
        const int Cl = min(C, T - c0);
        // q and k of token t (of the chunk) at channel i
        auto qq = [&](int t, int i) {
            return st ? in_f(qs[t * ldq + i]) : ld_in<IN_BF16>(p.q, (kh * T + c0 + t) * dk + i);
        };
        auto kk = [&](int t, int i) {
            return st ? in_f(ks[t * ldq + i]) : ld_in<IN_BF16>(p.k, (kh * T + c0 + t) * dk + i);
        };
        __syncthreads();
        // --- the chunk's start state, gates, Lambda, the dO tile
        {
            const float *src = p.S_chunks + ((vh * nch + c) * dk) * (long)dv + n0;
            for (int idx = tid; idx < dk * NV; idx += NT) {
                const int i = idx / NV, n = idx % NV;
                S[idx] = n < nv ? src[(long)i * dv + n] : 0.f;
            }
        }
        for (int t = tid; t < Cl; t += NT)
            sbeta[t] = p.beta[kh * T + c0 + t];
        for (int gi = tid; gi < G; gi += NT) {
            float acc = 0.f;
            for (int t = 0; t < Cl; ++t) {
                acc += p.g[(kh * T + c0 + t) * G + gi];
                lam[t * G + gi] = acc;
            }
        }
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int t = idx / NV, n = idx % NV;
            dO[idx] = n < nv ? p.dO[(vh * T + c0 + t) * dv + n0 + n] : 0.f;
        }
        if (st)
            for (int idx = tid; idx < Cl * dk; idx += NT) {
                const int t = idx / dk, i = idx % dk;
                const long g = (kh * T + c0 + t) * dk + i;
                qs[t * ldq + i] = static_cast<const In *>(p.q)[g];
                ks[t * ldq + i] = static_cast<const In *>(p.k)[g];
            }
        __syncthreads();
        // --- P, M = P diag(beta) (into A), L
        for (int idx = tid; idx < Cl * Cl; idx += NT) {
            const int t = idx / Cl, j = idx % Cl;
            float pm = 0.f, lm = 0.f;
            if (j <= t) {
                for (int gi = 0; gi < G; ++gi) {
                    float skk = 0.f, sqk = 0.f;
                    for (int i = gi * width; i < (gi + 1) * width; ++i) {
                        const float kji = kk(j, i);
                        skk += kk(t, i) * kji;
                        sqk += qq(t, i) * kji;
                    }
                    const float e = expf(lam[t * G + gi] - lam[j * G + gi]);
                    pm += e * skk;
                    lm += e * sqk;
                    if (tab)
                        E1[t * C + j] = e;
                }
                if (j == t)
                    pm = 0.f;
            }
            P[t * C + j] = pm;
            A[t * C + j] = (j == t) ? 1.f : pm * sbeta[j];
            L[t * C + j] = lm;
        }
        if (tab)
            for (int t = tid; t < Cl; t += NT)
                Et[t] = expf(lam[t]);
        __syncthreads();
        // --- A = (I + M)^{-1} by forward substitution in place (row t from the rows above)
        for (int t = 1; t < Cl; ++t) {
            for (int j = tid; j < t; j += NT)
                row[j] = A[t * C + j];
            __syncthreads();
            for (int cc = tid; cc < t; cc += NT) {
                float acc = -row[cc];
                for (int j = cc + 1; j < t; ++j)
                    acc -= row[j] * A[j * C + cc];
                A[t * C + cc] = acc;
            }
            __syncthreads();
        }
        // --- R = V - Kbar S (into dR), Kbar_t = k_t e^{Lambda_t}
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int t = idx / NV, n = idx % NV;
            float acc = 0.f;
            for (int i = 0; i < dk; ++i)
                acc += kk(t, i) * (tab ? Et[t] : expf(lam[t * G + i / width])) * S[i * NV + n];
            const float vv = n < nv ? ld_in<IN_BF16>(p.v, (vh * T + c0 + t) * dv + n0 + n) : 0.f;
            dR[idx] = vv - acc;
        }
        __syncthreads();
        // --- Y = A R;  dE = L^T dO + Khat dS', Khat_j = k_j e^{Lambda_C - Lambda_j}
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int t = idx / NV, n = idx % NV;
            float acc = 0.f;
            for (int j = 0; j <= t; ++j)
                acc += A[t * C + j] * dR[j * NV + n];
            Y[idx] = acc;
        }
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int j = idx / NV, n = idx % NV;
            float acc = 0.f;
            for (int t = j; t < Cl; ++t)
                acc += L[t * C + j] * dO[t * NV + n];
            for (int i = 0; i < dk; ++i) {
                const int gi = i / width;
                acc += kk(j, i) *
                       (tab ? E1[(Cl - 1) * C + j] : expf(lam[(Cl - 1) * G + gi] - lam[j * G + gi])) *
                       dS[i * NV + n];
            }
            dE[idx] = acc;
        }
        __syncthreads();
        // --- dbeta_t += sum_n dE_tn Y_tn (this tile's part); dY = beta dE in place (one row a thread)
        for (int t = tid; t < Cl; t += NT) {
            float db = 0.f;
            for (int n = 0; n < NV; ++n) {
                db += dE[t * NV + n] * Y[t * NV + n];
                dE[t * NV + n] *= sbeta[t];
            }
            atomicAdd(&p.grad_beta[kh * T + c0 + t], db);
        }
        __syncthreads();
        // --- dR = A^T dY (R is spent)
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int j = idx / NV, n = idx % NV;
            float acc = 0.f;
            for (int t = j; t < Cl; ++t)
                acc += A[t * C + j] * dE[t * NV + n];
            dR[idx] = acc;
        }
        __syncthreads();
        // --- dV = dR;  dM = -dR Y^T (t > j) into A;  dL = dO E^T (t >= j) into L;
        //     per channel F_i = e^{Lambda_C} and X_i = sum_n dS'_in S'_in, S' = F S + Khat^T E
        for (int idx = tid; idx < Cl * NV; idx += NT) {
            const int t = idx / NV, n = idx % NV;
            if (n < nv)
                p.grad_v[(vh * T + c0 + t) * dv + n0 + n] = dR[idx];
        }
        for (int idx = tid; idx < Cl * Cl; idx += NT) {
            const int t = idx / Cl, j = idx % Cl;
            float dm = 0.f, dl = 0.f;
            if (j < t)
                for (int n = 0; n < NV; ++n)
                    dm -= dR[t * NV + n] * Y[j * NV + n];
            if (j <= t) {
                for (int n = 0; n < NV; ++n)
                    dl += dO[t * NV + n] * Y[j * NV + n];
                dl *= sbeta[j];
            }
            A[t * C + j] = dm;
            L[t * C + j] = dl;
        }
        for (int i = tid; i < dk; i += NT) {
            const int gi = i / width;
            const float lc = lam[(Cl - 1) * G + gi];
            const float f = expf(lc);
            float x = 0.f;
            for (int n = 0; n < NV; ++n) {
                float sn = f * S[i * NV + n];
                for (int t = 0; t < Cl; ++t)
                    sn += kk(t, i) *
                          (tab ? E1[(Cl - 1) * C + t] : expf(lc - lam[t * G + gi])) *
                          sbeta[t] * Y[t * NV + n];
                x += dS[i * NV + n] * sn;
            }
            Fv[i] = f;
            X[i] = x;
        }
        __syncthreads();
        // --- dbeta_j += sum_{t > j} dM_tj P_tj
        for (int j = tid; j < Cl; j += NT) {
            float acc = 0.f;
            for (int t = j + 1; t < Cl; ++t)
                acc += A[t * C + j] * P[t * C + j];
            atomicAdd(&p.grad_beta[kh * T + c0 + j], acc);
        }
        // --- per (token t, channel i): dq, dk (this tile's part) and dLambda.  With
        //     dP_tj = beta_j dM_tj and e_tj = e^{Lambda_ti - Lambda_ji} (t >= j):
        //     a = sum_{j<t} dP_tj k_ji e_tj,   b = sum_{t'>t} dP_t't k_t'i e_t't,
        //     c = sum_{j<=t} dL_tj k_ji e_tj,  d = sum_{t'>=t} dL_t't q_t'i e_t't
        for (int idx = tid; idx < Cl * dk; idx += NT) {
            const int t = idx / dk, i = idx % dk, gi = i / width;
            const float lt = lam[t * G + gi], lc = lam[(Cl - 1) * G + gi];
            const long base = (kh * T + c0) * dk + i;
            const float kti = kk(t, i);
            const float qti = qq(t, i);
            float a = 0.f, bb = 0.f, cc = 0.f, d = 0.f;
            for (int j = 0; j <= t; ++j) {
                const float e = tab ? E1[t * C + j] : expf(lt - lam[j * G + gi]);
                const float kji = kk(j, i);
                if (j < t)
                    a += sbeta[j] * A[t * C + j] * kji * e;
                cc += L[t * C + j] * kji * e;
            }
            for (int t2 = t; t2 < Cl; ++t2) {
                const float e = tab ? E1[t2 * C + t] : expf(lam[t2 * G + gi] - lt);
                if (t2 > t)
                    bb += sbeta[t] * A[t2 * C + t] * kk(t2, i) * e;
                d += L[t2 * C + t] * qq(t2, i) * e;
            }
            float dqb = 0.f, dkb = 0.f, dkh = 0.f;
            for (int n = 0; n < NV; ++n) {
                dqb += dO[t * NV + n] * S[i * NV + n];
                dkb -= dR[t * NV + n] * S[i * NV + n];
                dkh += Y[t * NV + n] * dS[i * NV + n];
            }
            dkh *= sbeta[t];
            const float et = tab ? Et[t] : expf(lt);
            const float eh = tab ? E1[(Cl - 1) * C + t] : expf(lc - lt);
            atomicAdd(&p.grad_q[base + (long)t * dk], cc + dqb * et);
            atomicAdd(&p.grad_k[base + (long)t * dk], a + bb + d + dkb * et + dkh * eh);
            DL[t * dk + i] = kti * (a - bb - d) + qti * cc + (dqb * qti + dkb * kti) * et - dkh * kti * eh;
        }
        __syncthreads();
        if (width > 1) {
            for (int idx = tid; idx < Cl * G; idx += NT) {
                const int t = idx / G, gi = idx % G;
                float acc = 0.f;
                for (int i = gi * width; i < (gi + 1) * width; ++i)
                    acc += DL[t * dk + i];
                DLg[idx] = acc;
            }
            __syncthreads();
        }
        // --- dg: reverse cumulative sum of dLambda in the chunk, plus the gradient of
        //     Lambda_C at every token;  dS <- F dS' + Qbar^T dO - Kbar^T dR
        for (int gi = tid; gi < G; gi += NT) {
            float xg = 0.f;
            for (int i = gi * width; i < (gi + 1) * width; ++i)
                xg += X[i];
            float run = 0.f;
            for (int t = Cl - 1; t >= 0; --t) {
                run += DLg[t * G + gi];
                atomicAdd(&p.grad_g[(kh * T + c0 + t) * G + gi], run + xg);
            }
        }
        for (int idx = tid; idx < dk * NV; idx += NT) {
            const int i = idx / NV, n = idx % NV, gi = i / width;
            float acc = Fv[i] * dS[idx];
            for (int t = 0; t < Cl; ++t) {
                const float e = tab ? Et[t] : expf(lam[t * G + gi]);
                acc += e * (qq(t, i) * dO[t * NV + n] - kk(t, i) * dR[t * NV + n]);
            }
            dS[idx] = acc;
        }
    }
    __syncthreads();
    if (p.grad_S0 != nullptr)
        for (int idx = tid; idx < dk * NV; idx += NT) {
            const int i = idx / NV, n = idx % NV;
            if (n < nv)
                p.grad_S0[(vh * dk + i) * dv + n0 + n] = dS[idx];
        }
}

template <bool I, int NV>
int launch_bwd_variant(const Params &p, int smem, cudaStream_t stream)
{
    auto kern = simt_bwd_kernel<I, NV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 6;  // GDR_ERR_CUDA
    dim3 grid((p.dv + NV - 1) / NV, p.Hv, p.B);
    kern<<<grid, NT, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

constexpr int kMaxSmem = kBwdSmemFloats * 4;

int bwd_smem_for(const Params &p, int NV)
{
    return bwd_layout(p.C, p.G, p.dk, NV, p.in_bf16 ? 2 : 4).total * (int)sizeof(float);
}

int zero(float *a, long n, cudaStream_t stream)
{
    if (n <= 0)
        return 0;
    long blocks = (n + NT - 1) / NT;
    if (blocks > 4096)
        blocks = 4096;
    zero_kernel<<<(unsigned)blocks, NT, 0, stream>>>(a, n);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace

size_t bwd_workspace_bytes(const Params &p)
{
    const long nch = (p.T + p.C - 1) / p.C;
    return sizeof(float) * (size_t)p.B * p.Hv * nch * p.dk * p.dv;
}

int bwd_smem_bytes(const Params &p)
{
    const int s32 = bwd_smem_for(p, 32);
    return s32 <= kMaxSmem ? s32 : bwd_smem_for(p, 16);
}

int launch_bwd(const Params &p, void *workspace, cudaStream_t stream)
{
    const int s32 = bwd_smem_for(p, 32), s16 = bwd_smem_for(p, 16);
    if (s16 > kMaxSmem)
        return 5;  // GDR_ERR_UNSUPPORTED
    // the forward, for the states at the chunk starts only
    Params f = p;
    f.o = nullptr;
    f.S_final = nullptr;
    f.S_chunks = static_cast<float *>(workspace);
    f.momentum = 0;
    int rc = launch_simt(f, stream);
    if (rc != 0)
        return rc;
    // key-side gradients are accumulated
    const long nk = (long)p.B * p.Hk * p.T;
    if ((rc = zero(p.grad_q, nk * p.dk, stream)) || (rc = zero(p.grad_k, nk * p.dk, stream)) ||
        (rc = zero(p.grad_g, nk * p.G, stream)) || (rc = zero(p.grad_beta, nk, stream)))
        return rc;
    Params bp = p;
    bp.S_chunks = static_cast<float *>(workspace);
    if (s32 <= kMaxSmem)
        return p.in_bf16 ? launch_bwd_variant<true, 32>(bp, s32, stream)
                         : launch_bwd_variant<false, 32>(bp, s32, stream);
    return p.in_bf16 ? launch_bwd_variant<true, 16>(bp, s16, stream)
                     : launch_bwd_variant<false, 16>(bp, s16, stream);
}

}  // namespace gdr
