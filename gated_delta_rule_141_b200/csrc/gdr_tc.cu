// gdr_tc.cu -- chunkwise gated delta-rule forward on the B200 tensor cores.
//
// One CTA (256 threads) owns one (batch, value head, 64-column value tile) and
// walks the chunks of its sequence in order, keeping the fp32 state tile S
// (dk x 64) in registers and a bf16 copy in shared memory as an MMA operand.
// Per chunk of C tokens ("Systolic Linear Attention: Co-Designing Tile-Grouped
// Gated Delta Attention for TPUs", §2.1 "Chunkwise WY parallelization", §2.3
// Table 2, §2.4.2):
//   1. TMA brings the chunk's q, k (C x dk) and v (C x 64) tiles (next chunk
//      prefetched into a second stage).
//   2. Gate: Lambda_t = cumsum g (warp scans); decay factors are exponentials of
//      non-positive differences: e^{Lambda_t}, e^{Lambda_C - Lambda_t},
//      e^{Lambda_t - Lambda_j} (t >= j) -- no division by decay prefixes.
//   3. tcgen05: Q K^T and K K^T into TMEM; decay masks and beta applied on the
//      way out: M (strictly lower, beta_j on column j) and L (lower).
//   4. A = (I + M)^{-1} by block doubling in fp32 (§2.4.3): exact 16 x 16
//      diagonal blocks, then merges X21 = -X22 M21 X11.
//   5. tcgen05: W = diag(beta) A diag(e^Lambda) K,  U = diag(beta) A V.
//   6. tcgen05: P = W S and Q S;  E = U - P;  E_hat = diag(e^{Lambda_C - Lambda}) E.
//   7. tcgen05: dS = K^T E_hat and L E;  S <- e^{Lambda_C} S + dS;
//      O = diag(e^Lambda) Q S + L E.
// With a scalar gate the decays are row/column scalings of the C x C matrices,
// so q, k, v are used exactly as loaded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "gdr_internal.h"
#include "gdr_ptx.cuh"

namespace gdr {

__device__ int g_device_status = 0;

int read_and_clear_device_status()
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return -1;
    return v;
}

namespace {

using namespace ptx;

constexpr int NT = 256;            // threads per CTA
constexpr int NV = 64;             // value columns per CTA
constexpr int CH = 64;             // chunk length of this kernel
constexpr uint32_t TMEM_COLS = 512;
constexpr int kTimeoutStatus = 7;  // GDR_ERR_TIMEOUT

// TMEM column map (fp32 accumulators)
constexpr uint32_t TM_GQ = 0;      // Q K^T        C cols
constexpr uint32_t TM_GK = 64;     // K K^T        C cols
constexpr uint32_t TM_W = 0;       // W            dk cols (after the Grams are read)
constexpr uint32_t TM_U = 256;     // U            64 cols
constexpr uint32_t TM_P = 320;     // W S          64 cols
constexpr uint32_t TM_OS = 384;    // Q S          64 cols
constexpr uint32_t TM_OI = 448;    // L E          64 cols
constexpr uint32_t TM_DS = 256;    // K^T E_hat    64 cols (after U is read)

constexpr int MF_LD = CH + 4;      // row stride of the fp32 C x C scratch matrices

struct Smem {                      // byte offsets from the 1024-aligned base
    uint32_t q[2], k[2], v[2];     // TMA stages (SW128 tiles)
    uint32_t S, L, Ab, Abe, W, E, Eh;
    uint32_t Mf, Af, Tf;           // fp32 scratch
    uint32_t lam, ea, eb, beta;    // fp32 per-token
    uint32_t bar;                  // mbarriers: tma[2], mma
    uint32_t misc;                 // tmem slot, abort flag
    uint32_t total;
};

__host__ __device__ inline Smem smem_plan(int dk)
{
    Smem s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    for (int i = 0; i < 2; ++i) {
        s.q[i] = take(CH * dk * 2);
        s.k[i] = take(CH * dk * 2);
        s.v[i] = take(CH * NV * 2);
    }
    s.S = take(dk * NV * 2);
    s.L = take(CH * CH * 2);
    s.Ab = take(CH * CH * 2);
    s.Abe = take(CH * CH * 2);
    s.W = take(CH * dk * 2);
    s.E = take(CH * NV * 2);
    s.Eh = take(CH * NV * 2);
    s.Mf = take(CH * MF_LD * 4);
    s.Af = take(CH * MF_LD * 4);
    s.Tf = take(CH * MF_LD * 4);
    s.lam = take(CH * 4 * 4);       // lam, ea, eb, beta packed in one 1 KB block
    s.ea = s.lam + CH * 4;
    s.eb = s.lam + 2 * CH * 4;
    s.beta = s.lam + 3 * CH * 4;
    s.bar = take(64);
    s.misc = s.bar + 32;
    s.total = o + 1024;             // slack for aligning the dynamic base
    return s;
}

struct TcArgs {
    Params p;
    int nvt;                        // value tiles per value head (dv / NV)
};

// Row of an M = 64 (C = 64) accumulator held by this thread, or -1.
__device__ __forceinline__ int row64(int warp, int lane) { return lane < 16 ? 16 * (warp & 3) + lane : -1; }

// Issue D = A * B over K (one elected thread).
__device__ __forceinline__ void issue_kmajor_x_mnmajor(uint32_t d, uint32_t a_tile, int a_rows,
                                                       uint32_t b_tile, int b_rows, int K,
                                                       uint32_t idesc, bool acc)
{
    for (int k0 = 0; k0 < K; k0 += 16)
        mma_bf16(d, desc_kmajor(a_tile, a_rows, 0, k0), desc_mnmajor(b_tile, b_rows, k0, 0),
                 idesc, (acc || k0 > 0) ? 1u : 0u);
}

template <int DK, bool OUT_BF16>
__global__ void __launch_bounds__(NT, 1)
tc_scalar_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const TcArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const Smem Ly = smem_plan(DK);
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));
    auto f32at = [&](uint32_t off) { return reinterpret_cast<float *>(base + off); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = blockIdx.x % args.nvt;        // value tile inside the head
    const int hv = blockIdx.x / args.nvt;
    const int b = blockIdx.y;
    const int hk = hv / p.R;
    const int n0 = nt * NV;
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int T = p.T;
    const int nchunks = (T + CH - 1) / CH;

    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint64_t *mma_bar = tma_bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);
    float *lam = f32at(Ly.lam), *ea = f32at(Ly.ea), *eb = f32at(Ly.eb), *sbeta = f32at(Ly.beta);
    float *Mf = f32at(Ly.Mf), *Af = f32at(Ly.Af), *Tf = f32at(Ly.Tf);

    if (tid == 0) {
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(mma_bar, 1);
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);  // this warp's lanes
    const int half = warp >> 2;                  // column half of a 64-wide accumulator

    // ---- state: row i of S (= TMEM lane of dS), columns [32*half, 32*half+32)
    const int srow = (DK == 128) ? 32 * (warp & 3) + lane : row64(warp, lane);
    float sreg[32];
#pragma unroll
    for (int n = 0; n < 32; ++n)
        sreg[n] = 0.f;
    if (srow >= 0 && p.S0 != nullptr) {
        const float *src = p.S0 + (vh * DK + srow) * p.dv + n0 + 32 * half;
#pragma unroll
        for (int n = 0; n < 32; n += 4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(src + n);
            sreg[n] = t4.x; sreg[n + 1] = t4.y; sreg[n + 2] = t4.z; sreg[n + 3] = t4.w;
        }
    }
    if (srow >= 0)
#pragma unroll
        for (int n = 0; n < 32; n += 8)
            st_tile8(base_u32 + Ly.S, DK, srow, 32 * half + n, &sreg[n]);

    uint32_t mma_phase = 0;
    bool tma_pending[2] = {false, false};
    uint32_t tma_parity[2] = {0, 0};   // phase parity a pending TMA stage completes
    bool mma_pending = false;
    const uint32_t tx_bytes = 2u * CH * DK * 2u + CH * NV * 2u;

    auto issue_tma = [&](int c, int s) {
        mbar_arrive_expect_tx(&tma_bar[s], tx_bytes);
#pragma unroll
        for (int kb = 0; kb < DK / 64; ++kb) {
            tma_load_3d(base + Ly.q[s] + kb * CH * 128, &tm_q, &tma_bar[s], 64 * kb, c * CH, (int)kh);
            tma_load_3d(base + Ly.k[s] + kb * CH * 128, &tm_k, &tma_bar[s], 64 * kb, c * CH, (int)kh);
        }
        tma_load_3d(base + Ly.v[s], &tm_v, &tma_bar[s], n0, c * CH, (int)vh);
    };
    // every thread waits (bounded); returns true, for the whole CTA, if any
    // thread gave up -- the caller then leaves for the cleanup path
    auto wait_sync = [&](uint64_t *bar, uint32_t parity) -> bool {
        const bool gave_up = !mbar_wait(bar, parity);
        if (gave_up)
            atomicExch(&g_device_status, kTimeoutStatus);
        return __syncthreads_or(gave_up ? 1 : 0) != 0;
    };

    if (tid == 0 && nchunks > 0) {
        issue_tma(0, 0);
    }
    tma_pending[0] = nchunks > 0;
    tma_parity[0] = 0;
    fence_proxy_async_smem();      // S tile written by all threads
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const long c0 = (long)c * CH;
        const int Cl = (int)min((long)CH, T - c0);
        if (c + 1 < nchunks) {
            if (tid == 0)
                issue_tma(c + 1, st ^ 1);
            tma_pending[st ^ 1] = true;
            tma_parity[st ^ 1] = ((c + 1) >> 1) & 1;
        }
        // ---- gate: Lambda (inclusive cumsum), decay factors, beta
        if (warp < 2) {
            const int t = 32 * warp + lane;
            float gv = (t < Cl) ? p.g[kh * T + c0 + t] : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, gv, off);
                if (lane >= off)
                    gv += y;
            }
            lam[t] = gv;
            sbeta[t] = (t < Cl) ? p.beta[kh * T + c0 + t] : 0.f;
        }
        __syncthreads();
        if (tid < CH) {
            const float l = lam[tid] + (tid >= 32 ? lam[31] : 0.f);
            Tf[tid] = l;   // staged: lam[31] is still read by other threads
        }
        __syncthreads();
        if (tid < CH) {
            lam[tid] = Tf[tid];
        }
        __syncthreads();
        if (tid < CH) {
            ea[tid] = __expf(lam[tid]);
            eb[tid] = __expf(lam[CH - 1] - lam[tid]);
        }
        if (wait_sync(&tma_bar[st], (c >> 1) & 1))
            goto cleanup;
        tma_pending[st] = false;

        // ---- Grams: Q K^T, K K^T  (M = N = C, K = dk)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(CH, CH, false, false);
            for (int k0 = 0; k0 < DK; k0 += 16) {
                mma_bf16(tmem + TM_GQ, desc_kmajor(base_u32 + Ly.q[st], CH, 0, k0),
                         desc_kmajor(base_u32 + Ly.k[st], CH, 0, k0), id, k0 > 0);
                mma_bf16(tmem + TM_GK, desc_kmajor(base_u32 + Ly.k[st], CH, 0, k0),
                         desc_kmajor(base_u32 + Ly.k[st], CH, 0, k0), id, k0 > 0);
            }
            mma_commit(mma_bar);
        }
        mma_pending = true;
        if (wait_sync(mma_bar, mma_phase))
            goto cleanup;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();
        // ---- decay masks: M (strict lower, beta_j), L (lower) ; thread = row t, 32 cols
        {
            const int t = row64(warp, lane);
            const int j0 = 32 * half;
            float gq[32], gk[32];
            tmem_ld16(tq + TM_GQ + j0, *reinterpret_cast<float(*)[16]>(&gq[0]));
            tmem_ld16(tq + TM_GQ + j0 + 16, *reinterpret_cast<float(*)[16]>(&gq[16]));
            tmem_ld16(tq + TM_GK + j0, *reinterpret_cast<float(*)[16]>(&gk[0]));
            tmem_ld16(tq + TM_GK + j0 + 16, *reinterpret_cast<float(*)[16]>(&gk[16]));
            tmem_ld_wait();
            if (t >= 0) {
                const float lt = lam[t];
                float lrow[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int j = j0 + u;
                    const float d = (j <= t) ? __expf(lt - lam[j]) : 0.f;
                    Mf[t * MF_LD + j] = (j < t) ? sbeta[j] * d * gk[u] : 0.f;
                    lrow[u] = d * gq[u];
                }
#pragma unroll
                for (int u = 0; u < 32; u += 8)
                    st_tile8(base_u32 + Ly.L, CH, t, j0 + u, &lrow[u]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- A = (I + M)^{-1}: exact 16 x 16 diagonal blocks, then doublings
        for (int idx = tid; idx < CH * CH; idx += NT)
            Af[(idx / CH) * MF_LD + (idx % CH)] = 0.f;
        __syncthreads();
        if (tid < CH) {
            const int blk = tid >> 4, cc = tid & 15, o = 16 * blk;
            float x[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                float acc = (t == cc) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < t; ++j)
                    acc -= (j >= cc) ? Mf[(o + t) * MF_LD + o + j] * x[j] : 0.f;
                x[t] = (t >= cc) ? acc : 0.f;
            }
#pragma unroll
            for (int t = 0; t < 16; ++t)
                Af[(o + t) * MF_LD + o + cc] = x[t];
        }
        __syncthreads();
        for (int bs = 16; bs < CH; bs *= 2) {
            const int npairs = CH / (2 * bs);
            // T = M21 X11
            for (int idx = tid; idx < npairs * bs * bs; idx += NT) {
                const int pr = idx / (bs * bs), r = (idx / bs) % bs, cc = idx % bs;
                const int o = 2 * bs * pr;
                float acc = 0.f;
                for (int l = cc; l < bs; ++l)
                    acc += Mf[(o + bs + r) * MF_LD + o + l] * Af[(o + l) * MF_LD + o + cc];
                Tf[(pr * bs + r) * MF_LD + cc] = acc;
            }
            __syncthreads();
            // X21 = -X22 T
            for (int idx = tid; idx < npairs * bs * bs; idx += NT) {
                const int pr = idx / (bs * bs), r = (idx / bs) % bs, cc = idx % bs;
                const int o = 2 * bs * pr;
                float acc = 0.f;
                for (int l = 0; l <= r; ++l)
                    acc += Af[(o + bs + r) * MF_LD + o + bs + l] * Tf[(pr * bs + l) * MF_LD + cc];
                Af[(o + bs + r) * MF_LD + o + cc] = -acc;
            }
            __syncthreads();
        }
        // ---- Ab = diag(beta) A,  Abe = diag(beta) A diag(e^Lambda)   (bf16 operands)
        for (int idx = tid; idx < CH * (CH / 8); idx += NT) {
            const int t = idx / (CH / 8), j = (idx % (CH / 8)) * 8;
            float a[8], ae[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a[u] = sbeta[t] * Af[t * MF_LD + j + u];
                ae[u] = a[u] * ea[j + u];
            }
            st_tile8(base_u32 + Ly.Ab, CH, t, j, a);
            st_tile8(base_u32 + Ly.Abe, CH, t, j, ae);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- W = Abe K  (N = dk), U = Ab V (N = 64)
        if (tid == 0) {
            tc_fence_after();
            issue_kmajor_x_mnmajor(tmem + TM_W, base_u32 + Ly.Abe, CH, base_u32 + Ly.k[st], CH, CH,
                                   idesc_bf16(CH, DK, false, true), false);
            issue_kmajor_x_mnmajor(tmem + TM_U, base_u32 + Ly.Ab, CH, base_u32 + Ly.v[st], CH, CH,
                                   idesc_bf16(CH, NV, false, true), false);
            mma_commit(mma_bar);
        }
        mma_pending = true;
        if (wait_sync(mma_bar, mma_phase))
            goto cleanup;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();
        {
            const int t = row64(warp, lane);
            const int c0w = (DK / 2) * half;
#pragma unroll
            for (int cb = 0; cb < DK / 2; cb += 16) {
                float w16[16];
                tmem_ld16(tq + TM_W + c0w + cb, w16);
                tmem_ld_wait();
                if (t >= 0) {
                    st_tile8(base_u32 + Ly.W, CH, t, c0w + cb, &w16[0]);
                    st_tile8(base_u32 + Ly.W, CH, t, c0w + cb + 8, &w16[8]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- P = W S,  Q S
        if (tid == 0) {
            tc_fence_after();
            issue_kmajor_x_mnmajor(tmem + TM_P, base_u32 + Ly.W, CH, base_u32 + Ly.S, DK, DK,
                                   idesc_bf16(CH, NV, false, true), false);
            issue_kmajor_x_mnmajor(tmem + TM_OS, base_u32 + Ly.q[st], CH, base_u32 + Ly.S, DK, DK,
                                   idesc_bf16(CH, NV, false, true), false);
            mma_commit(mma_bar);
        }
        mma_pending = true;
        if (wait_sync(mma_bar, mma_phase))
            goto cleanup;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();
        // ---- E = U - P,  E_hat = e^{Lambda_C - Lambda_t} E
        {
            const int t = row64(warp, lane);
            const int j0 = 32 * half;
            float u[32], pv[32];
            tmem_ld16(tq + TM_U + j0, *reinterpret_cast<float(*)[16]>(&u[0]));
            tmem_ld16(tq + TM_U + j0 + 16, *reinterpret_cast<float(*)[16]>(&u[16]));
            tmem_ld16(tq + TM_P + j0, *reinterpret_cast<float(*)[16]>(&pv[0]));
            tmem_ld16(tq + TM_P + j0 + 16, *reinterpret_cast<float(*)[16]>(&pv[16]));
            tmem_ld_wait();
            if (t >= 0) {
                const float f = eb[t];
                float e[32], eh[32];
#pragma unroll
                for (int n = 0; n < 32; ++n) {
                    e[n] = u[n] - pv[n];
                    eh[n] = f * e[n];
                }
#pragma unroll
                for (int n = 0; n < 32; n += 8) {
                    st_tile8(base_u32 + Ly.E, CH, t, j0 + n, &e[n]);
                    st_tile8(base_u32 + Ly.Eh, CH, t, j0 + n, &eh[n]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- dS = K^T E_hat (M = dk),  O_intra = L E
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_ds = idesc_bf16(DK, NV, true, true);
            for (int k0 = 0; k0 < CH; k0 += 16)
                mma_bf16(tmem + TM_DS, desc_mnmajor(base_u32 + Ly.k[st], CH, k0, 0),
                         desc_mnmajor(base_u32 + Ly.Eh, CH, k0, 0), id_ds, k0 > 0);
            issue_kmajor_x_mnmajor(tmem + TM_OI, base_u32 + Ly.L, CH, base_u32 + Ly.E, CH, CH,
                                   idesc_bf16(CH, NV, false, true), false);
            mma_commit(mma_bar);
        }
        mma_pending = true;
        if (wait_sync(mma_bar, mma_phase))
            goto cleanup;
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();
        // ---- S <- e^{Lambda_C} S + dS ; O = e^{Lambda_t} (Q S) + L E
        {
            const float F = ea[CH - 1];
            float ds[32];
            tmem_ld16(tq + TM_DS + 32 * half, *reinterpret_cast<float(*)[16]>(&ds[0]));
            tmem_ld16(tq + TM_DS + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&ds[16]));
            float os[32], oi[32];
            tmem_ld16(tq + TM_OS + 32 * half, *reinterpret_cast<float(*)[16]>(&os[0]));
            tmem_ld16(tq + TM_OS + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&os[16]));
            tmem_ld16(tq + TM_OI + 32 * half, *reinterpret_cast<float(*)[16]>(&oi[0]));
            tmem_ld16(tq + TM_OI + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&oi[16]));
            tmem_ld_wait();
            if (srow >= 0) {
#pragma unroll
                for (int n = 0; n < 32; ++n)
                    sreg[n] = F * sreg[n] + ds[n];
#pragma unroll
                for (int n = 0; n < 32; n += 8)
                    st_tile8(base_u32 + Ly.S, DK, srow, 32 * half + n, &sreg[n]);
            }
            const int t = row64(warp, lane);
            if (t >= 0 && t < Cl) {
                const float a = ea[t];
                const long orow = (vh * T + c0 + t) * p.dv + n0 + 32 * half;
                if constexpr (OUT_BF16) {
                    uint32_t pk[16];
#pragma unroll
                    for (int n = 0; n < 32; n += 2)
                        pk[n / 2] = pack_bf16(a * os[n] + oi[n], a * os[n + 1] + oi[n + 1]);
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow);
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        dst[n] = make_uint4(pk[4 * n], pk[4 * n + 1], pk[4 * n + 2], pk[4 * n + 3]);
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow);
#pragma unroll
                    for (int n = 0; n < 32; n += 4)
                        dst[n / 4] = make_float4(a * os[n] + oi[n], a * os[n + 1] + oi[n + 1],
                                                 a * os[n + 2] + oi[n + 2], a * os[n + 3] + oi[n + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    if (srow >= 0 && p.S_final != nullptr) {
        float *dst = p.S_final + (vh * DK + srow) * p.dv + n0 + 32 * half;
#pragma unroll
        for (int n = 0; n < 32; n += 4)
            *reinterpret_cast<float4 *>(dst + n) = make_float4(sreg[n], sreg[n + 1], sreg[n + 2], sreg[n + 3]);
    }

cleanup:
    // drain anything still in flight (bounded), then release tensor memory
    if (tid == 0) {
        for (int s = 0; s < 2; ++s)
            if (tma_pending[s])
                mbar_wait(&tma_bar[s], tma_parity[s], 100000000ull);
        if (mma_pending)
            mbar_wait(mma_bar, mma_phase, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D map over [seqs][T][width] bf16 with a box of 64 columns x `rows` rows.
bool make_map(CUtensorMap *m, const void *ptr, int width, int T, long seqs, int rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)T, (cuuint64_t)seqs};
    const cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)width * 2 * T};
    const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, bool OB>
int launch_scalar(const Params &p, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, DK, p.T, (long)p.B * p.Hk, CH) ||
        !make_map(&mk, p.k, DK, p.T, (long)p.B * p.Hk, CH) ||
        !make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CH))
        return 6;
    const Smem Ly = smem_plan(DK);
    auto kern = tc_scalar_kernel<DK, OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    TcArgs a;
    a.p = p;
    a.nvt = p.dv / NV;
    dim3 grid(a.nvt * p.Hv, p.B);
    kern<<<grid, NT, Ly.total, stream>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

// Self-test of the bounded-wait path every tensor-core kernel relies on: one
// warp takes tensor memory, waits on an mbarrier that nothing ever arrives on,
// gives up after limit_ns of wall time exactly as the production waits do (the
// status word becomes the timeout code), releases the tensor memory and returns.
__global__ void __launch_bounds__(32, 1) wait_probe_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t slot;
    tmem_alloc(&slot, 32);
    tmem_relinquish();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns))
        atomicExch(&g_device_status, kTimeoutStatus);
    __syncwarp();
    tmem_dealloc(slot, 32);
}

#include "gdr_tc_ws.cuh"
#include "gdr_tc_gen.cuh"
#include "gdr_tc_prep.cuh"
#include "gdr_tc_pair.cuh"
#include "gdr_tc_split.cuh"
#include "gdr_tc_ab128.cuh"
#include "gdr_tc_split128.cuh"

}  // namespace

// In exact mode the chunkwise form reaches the token recurrence exactly for any
// chunk length (the WY equivalence of the SLA paper, §2.4.2), so a request for
// C = 128 runs on the C = 64 kernels: the same function, blocked more finely.
// The truncated and 1-Step Neumann inverses depend on C: at C = 128 the two-pass
// path runs them as pairs of 64-token halves with the pair correction
// (gdr_tc_pair.cuh), which the one-pass kernels do not have.
static Params as_kernel_chunk(const Params &p)
{
    Params q = p;
    if (p.C == 128 && !p.momentum) {   // momentum acts at the request's chunk boundaries
        q.C = CH;
        q.pair = p.neumann || p.neumann1;
    }
    return q;
}

int tc_kernel_chunk(const Params &p)
{
    const Params q = as_kernel_chunk(p);
    return q.pair ? 2 * q.C : q.C;
}

bool tc_supports(const Params &p0)
{
    const Params p = as_kernel_chunk(p0);
    if (p.pair)
        return false;
    const bool scalar64 = p.in_bf16 && p.G == 1 && p.C == CH && p.dk == 64 && p.dv % NV == 0 &&
                          !p.neumann && p.T >= 1 && p.B <= 65535;
    // the one-pass kernels have no 1-Step Neumann inverse
    return !p.neumann1 && (ws::supports(p) || scalar64 || gen::supports(p));
}

int launch_tc(const Params &p0, cudaStream_t stream)
{
    const Params p = as_kernel_chunk(p0);
    if (p.pair)
        return 5;
    if (ws::supports(p))
        return p.out_bf16 ? ws::launch<true>(p, stream) : ws::launch<false>(p, stream);
    if (gen::supports(p)) {
        if (p.dk == 128)
            return p.out_bf16 ? gen::launch<128, true>(p, stream) : gen::launch<128, false>(p, stream);
        return p.out_bf16 ? gen::launch<256, true>(p, stream) : gen::launch<256, false>(p, stream);
    }
    if (p.dk == 64)
        return p.out_bf16 ? launch_scalar<64, true>(p, stream) : launch_scalar<64, false>(p, stream);
    return 5;
}

bool tc2_supports(const Params &p0) { return split::supports(as_kernel_chunk(p0)); }

bool tc2w_supports(const Params &p0) { return split::supports128(as_kernel_chunk(p0)); }

size_t tc2_workspace_bytes(const Params &p0)
{
    // the records, then (for few long sequences) the segmented state pass's buffers
    const Params p = as_kernel_chunk(p0);
    const size_t rec = prep::ws_bytes(p), seg = split::state_seg_bytes(p);
    return seg == 0 ? rec : ((rec + 255) & ~size_t(255)) + seg;
}

int tc2_state_segments(const Params &p0) { return split::state_seg_plan(as_kernel_chunk(p0)).nseg; }

int launch_tc2(const Params &p0, void *workspace, cudaStream_t stream)
{
    const Params p = as_kernel_chunk(p0);
    if (!split::supports(p))
        return 5;
    const int kind = prep::record_kind(p);
    int rc;
    if (p.dk == 256) {
        rc = prep::launch<256>(p, workspace, kind, stream, p.pair);
        if (rc == 0 && p.pair)
            rc = pair::launch<256>(p, workspace, stream);
        if (rc != 0)
            return rc;
        return p.out_bf16 ? split::launch<256, true>(p, workspace, stream)
                          : split::launch<256, false>(p, workspace, stream);
    }
    const bool wide = split::use128(p);   // the 128-column state pass (stores -W)
    rc = prep::launch<128>(p, workspace, kind, stream, p.pair, wide ? 1 : 0);
    if (rc == 0 && p.pair)
        rc = pair::launch<128>(p, workspace, stream, wide ? 1 : 0);
    if (rc != 0)
        return rc;
    if (wide)
        return p.out_bf16 ? split::launch128<true>(p, workspace, stream)
                          : split::launch128<false>(p, workspace, stream);
    return p.out_bf16 ? split::launch<128, true>(p, workspace, stream)
                      : split::launch<128, false>(p, workspace, stream);
}

int launch_wait_probe(uint64_t limit_ns, cudaStream_t stream)
{
    wait_probe_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

bool prepare_supports(const Params &p) { return prep::supports(p); }

size_t prepare_bytes(const Params &p) { return prep::bytes(p); }

int launch_prepare(const Params &p, void *out, cudaStream_t stream)
{
    if (!prep::supports(p))
        return 5;
    return p.dk == 128 ? prep::launch<128>(p, out, prep::REC_PLAIN, stream)
                       : prep::launch<256>(p, out, prep::REC_PLAIN, stream);
}

}  // namespace gdr
