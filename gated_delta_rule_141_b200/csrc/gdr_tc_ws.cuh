// gdr_tc_ws.cuh -- warp-specialised tensor-core kernel for the scalar gate,
// chunk C = 64, key width dk = 128, 64 value columns per CTA.  Included by
// gdr_tc.cu (it shares that file's device status word).
//
// The chunk recurrence has two dependency chains ("Systolic Linear Attention:
// Co-Designing Tile-Grouped Gated Delta Attention for TPUs", §2.1, §2.3
// Table 2, §2.4.2-2.4.3):
//   intra chunk c+1 (no state): Lambda, Q K^T and K K^T with decay masks,
//       A = (I + M)^{-1}, U = diag(beta) A V, W = diag(beta) A diag(e^Lambda) K;
//   state chunk c: P = W S, E = U - P, S <- e^{Lambda_C} S + K^T E_hat,
//       O = Qbar S + L E.
// Four roles run them concurrently, handing tiles over through mbarriers:
//   warp 0       TMA producer (q, k, v tiles; gates) for a 2-stage ring
//   warp 1       MMA issuer (one thread issues every tcgen05.mma)
//   warps 2-5    state group: E, S update, O epilogue (fp32 S kept in TMEM)
//   warps 6-13   intra team: gates, Gram read-back, chunk inverse, W read-back
// MMA operands are stacked so that every MMA has M = 128:
//   [Q; K] K^T,  [Ab; Abe] V -> U,  [Ab; Abe] K -> W,  [W; Qbar] S -> P, Qbar S,
//   K^T E_hat,  [V; L] E accumulated onto Qbar S (its top half lands on the
//   already-consumed P rows).
// Stage s shared memory: blocks of 64 columns x 192 rows holding W | Q | K
// (rows 0-63 | 64-127 | 128-191) and a 128-row block holding V | L.

namespace ws {

constexpr int NWARP = 14;
constexpr int NTHR = NWARP * 32;     // 448
constexpr int CC = 64;               // chunk length
constexpr int KD = 128;              // key width
constexpr int NVC = 64;              // value columns per CTA
constexpr int W_PROD = 0, W_MMA = 1, W_STATE0 = 2, W_INTRA0 = 6;
constexpr int N_STATE = 128, N_INTRA = 256;
constexpr int NB_INTRA = 1, NB_STATE = 2;   // named barrier ids
constexpr int LDM = 68;              // fp32 scratch row stride
constexpr int LDT = 36;              // merge scratch row stride

constexpr uint32_t T_GRAM = 0;       // [Q;K] K^T         64 cols
constexpr uint32_t T_U = 64;         // [Ab;Abe] V        64 cols (rows 0-63 = U)
constexpr uint32_t T_W = 128;        // [Ab;Abe] K        128 cols (rows 64-127 = W)
constexpr uint32_t T_PO = 256;       // [W;Qbar] S (+[V;L] E)  rows 0-63 P, 64-127 O
constexpr uint32_t T_DS = 320;       // K^T E_hat         64 cols
constexpr uint32_t T_S = 384;        // fp32 state master 64 cols
constexpr uint32_t TMEM_COLS = 512;

enum Bar { FULL0, FULL1, FREE0, FREE1, GRAM_FULL, GRAM_FREE, AB_READY, WU_FULL, W_READY,
           P_FULL, E_READY, DS_FULL, S_READY, DRAIN, NBARS };

struct Gates { float graw[CC], lam[CC], ea[CC], eb[CC], beta[CC]; };

struct Plan {
    uint32_t wqk[2], vl[2], gates[2];
    uint32_t S, E, Eh, AB, Mf, Af, Tf, bar, misc, total;
};

__host__ __device__ inline Plan plan()
{
    Plan s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    for (int i = 0; i < 2; ++i) {
        s.wqk[i] = take((KD / 64) * 192 * 128);
        s.vl[i] = take(128 * 128);
        s.gates[i] = take(sizeof(Gates));
    }
    s.S = take(KD * NVC * 2);
    s.E = take(CC * NVC * 2);
    s.Eh = take(CC * NVC * 2);
    s.AB = take(128 * CC * 2);
    s.Mf = take(CC * LDM * 4);
    s.Af = take(CC * LDM * 4);
    s.Tf = take(32 * LDT * 4);
    s.bar = take(NBARS * 8 + 16);
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

__device__ __forceinline__ void named_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named-barrier OR vote: every participating thread gets the same answer.
__device__ __forceinline__ bool named_vote_or(int id, int n, bool pred)
{
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
        " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
        : "memory");
    return out != 0;
}

// Bounded wait that also gives up when another role raised the abort flag.
// Waiting warps back off with short sleeps so that their probes do not crowd
// the shared-memory pipe that the working roles need.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag)
{
    if (ptx::mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    uint32_t nap = 32;
    for (uint32_t it = 1;; ++it) {
        __nanosleep(nap);
        if (nap < 256)
            nap <<= 1;
        if (ptx::mbar_try_wait(bar, parity))
            return true;
        if ((it & 63) == 0) {
            if (*abort_flag)
                return false;
            if (ptx::globaltimer_ns() - t0 > 2000000000ull) {
                *abort_flag = 1;
                atomicExch(&g_device_status, kTimeoutStatus);
                return false;
            }
        }
    }
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(NTHR, 1)
ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const TcArgs args)
{
    using namespace ptx;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const Plan Ly = plan();
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = blockIdx.x % args.nvt;
    const int hv = blockIdx.x / args.nvt;
    const int b = blockIdx.y;
    const int hk = hv / p.R;
    const int n0 = nt * NVC;
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int T = p.T;
    const int N = (T + CC - 1) / CC;

    const uint32_t pad = base_u32 - smem_u32(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + pad + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + pad + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + pad + Ly.misc + 4);
    float *Mf = reinterpret_cast<float *>(smem_raw + pad + Ly.Mf);
    float *Af = reinterpret_cast<float *>(smem_raw + pad + Ly.Af);
    float *Tf = reinterpret_cast<float *>(smem_raw + pad + Ly.Tf);
    Gates *gates0 = reinterpret_cast<Gates *>(smem_raw + pad + Ly.gates[0]);
    Gates *gates1 = reinterpret_cast<Gates *>(smem_raw + pad + Ly.gates[1]);

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)
            mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = tid; i < CC * LDM; i += NTHR)   // the upper triangle of A stays zero
        Af[i] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        // outstanding loads per stage: bit s of pend, completion parity in par_s
        uint32_t pend = 0, par0 = 0, par1 = 0;
        for (int c = 0; c < N; ++c) {
            const int s = c & 1;
            if (c >= 2) {
                const bool ok = wait_or_abort(&bars[FREE0 + s], ((c >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            const long c0 = (long)c * CC;
            const int Cl = (int)min((long)CC, T - c0);
            Gates *gt = s ? gates1 : gates0;
            for (int t = lane; t < CC; t += 32) {
                gt->graw[t] = (t < Cl) ? p.g[kh * T + c0 + t] : 0.f;
                gt->beta[t] = (t < Cl) ? p.beta[kh * T + c0 + t] : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[FULL0 + s], 4u * CC * 64 * 2 + CC * NVC * 2);
                for (int kb = 0; kb < KD / 64; ++kb) {
                    uint8_t *blk = base + (s ? Ly.wqk[1] : Ly.wqk[0]) + kb * 192 * 128;
                    tma_load_3d(blk + 64 * 128, &tm_q, &bars[FULL0 + s], 64 * kb, (int)c0, (int)kh);
                    tma_load_3d(blk + 128 * 128, &tm_k, &bars[FULL0 + s], 64 * kb, (int)c0, (int)kh);
                }
                tma_load_3d(base + (s ? Ly.vl[1] : Ly.vl[0]), &tm_v, &bars[FULL0 + s], n0, (int)c0, (int)vh);
            }
            pend |= 1u << s;
            if (s)
                par1 = (c >> 1) & 1;
            else
                par0 = (c >> 1) & 1;
        }
        // drain loads that may still be landing (bounded)
        if (lane == 0) {
            if (pend & 1u)
                mbar_wait(&bars[FULL0], par0, 200000000ull);
            if (pend & 2u)
                mbar_wait(&bars[FULL1], par1, 200000000ull);
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_gram = idesc_bf16(128, CC, false, false);
            const uint32_t id_u = idesc_bf16(128, NVC, false, true);
            const uint32_t id_w = idesc_bf16(128, KD, false, true);
            const uint32_t id_po = idesc_bf16(128, NVC, false, true);
            const uint32_t id_ds = idesc_bf16(KD, NVC, true, true);
            const uint32_t ab = base_u32 + Ly.AB;
            auto gram = [&](int s) {
                const uint32_t t = base_u32 + (s ? Ly.wqk[1] : Ly.wqk[0]);
                for (int k0 = 0; k0 < KD; k0 += 16)
                    mma_bf16(tmem + T_GRAM, desc_kmajor(t, 192, 64, k0), desc_kmajor(t, 192, 128, k0),
                             id_gram, k0 > 0);
                mma_commit(&bars[GRAM_FULL]);
            };
            bool ok = true;
            if (N > 0) {
                ok = wait_or_abort(&bars[FULL0], 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    gram(0);
                }
            }
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                const uint32_t par = c & 1;
                const uint32_t wqk = base_u32 + (s ? Ly.wqk[1] : Ly.wqk[0]), vl = base_u32 + (s ? Ly.vl[1] : Ly.vl[0]);
                if (!(ok = wait_or_abort(&bars[AB_READY], par, abort_flag)))
                    break;
                tc_fence_after();
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    mma_bf16(tmem + T_U, desc_kmajor(ab, 128, 0, k0), desc_mnmajor(vl, 128, k0, 0),
                             id_u, k0 > 0);
                    mma_bf16(tmem + T_W, desc_kmajor(ab, 128, 0, k0),
                             desc_mnmajor(wqk, 192, 128 + k0, 0), id_w, k0 > 0);
                }
                mma_commit(&bars[WU_FULL]);
                if (!(ok = wait_or_abort(&bars[W_READY], par, abort_flag)))
                    break;
                if (!(ok = wait_or_abort(&bars[S_READY], par, abort_flag)))
                    break;
                tc_fence_after();
                for (int k0 = 0; k0 < KD; k0 += 16)
                    mma_bf16(tmem + T_PO, desc_kmajor(wqk, 192, 0, k0),
                             desc_mnmajor(base_u32 + Ly.S, KD, k0, 0), id_po, k0 > 0);
                mma_commit(&bars[P_FULL]);
                if (c + 1 < N) {
                    if (!(ok = wait_or_abort(&bars[FULL0 + (s ^ 1)], ((c + 1) >> 1) & 1, abort_flag)))
                        break;
                    if (!(ok = wait_or_abort(&bars[GRAM_FREE], par, abort_flag)))
                        break;
                    tc_fence_after();
                    gram(s ^ 1);
                }
                if (!(ok = wait_or_abort(&bars[E_READY], par, abort_flag)))
                    break;
                tc_fence_after();
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    mma_bf16(tmem + T_DS, desc_mnmajor(wqk, 192, 128 + k0, 0),
                             desc_mnmajor(base_u32 + Ly.Eh, CC, k0, 0), id_ds, k0 > 0);
                    mma_bf16(tmem + T_PO, desc_kmajor(vl, 128, 0, k0),
                             desc_mnmajor(base_u32 + Ly.E, CC, k0, 0), id_po, 1u);
                }
                mma_commit(&bars[DS_FULL]);
                mma_commit(&bars[FREE0 + s]);
            }
            // whatever was issued must finish before tensor memory is released
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, 200000000ull);
        }
    } else if (warp < W_INTRA0) {
        // ------------------------------------------------------------ state group
        const int stid = tid - W_STATE0 * 32;
        const int R = 32 * (warp & 3) + lane;    // state row / TMEM lane
#pragma unroll
        for (int cb = 0; cb < NVC; cb += 16) {
            float sv[16];
#pragma unroll
            for (int n = 0; n < 16; ++n)
                sv[n] = 0.f;
            if (p.S0 != nullptr) {
                const float *src = p.S0 + (vh * KD + R) * p.dv + n0 + cb;
#pragma unroll
                for (int n = 0; n < 16; n += 4) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(src + n);
                    sv[n] = v4.x; sv[n + 1] = v4.y; sv[n + 2] = v4.z; sv[n + 3] = v4.w;
                }
            }
            tmem_st16(tq + T_S + cb, sv);
            st_tile8(base_u32 + Ly.S, KD, R, cb, &sv[0]);
            st_tile8(base_u32 + Ly.S, KD, R, cb + 8, &sv[8]);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        named_sync(NB_STATE, N_STATE);
        if (stid == 0)
            mbar_arrive(&bars[S_READY]);
        for (int c = 0; c < N; ++c) {
            const int s = c & 1;
            const uint32_t par = c & 1;
            const long c0 = (long)c * CC;
            const int Cl = (int)min((long)CC, T - c0);
            if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[P_FULL], par, abort_flag)))
                break;
            tc_fence_after();
            const Gates *gt = s ? gates1 : gates0;
            const float F = gt->ea[CC - 1];
            if (R < CC) {
                const float f = gt->eb[R];
#pragma unroll
                for (int cb = 0; cb < NVC; cb += 16) {
                    float pv[16], uv[16], e[16], eh[16];
                    tmem_ld16(tq + T_PO + cb, pv);
                    tmem_ld16(tq + T_U + cb, uv);
                    tmem_ld_wait();
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        e[n] = uv[n] - pv[n];
                        eh[n] = f * e[n];
                    }
                    st_tile8(base_u32 + Ly.E, CC, R, cb, &e[0]);
                    st_tile8(base_u32 + Ly.E, CC, R, cb + 8, &e[8]);
                    st_tile8(base_u32 + Ly.Eh, CC, R, cb, &eh[0]);
                    st_tile8(base_u32 + Ly.Eh, CC, R, cb + 8, &eh[8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[E_READY]);
            if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[DS_FULL], par, abort_flag)))
                break;
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < NVC; cb += 16) {
                float ds[16], sv[16];
                tmem_ld16(tq + T_DS + cb, ds);
                tmem_ld16(tq + T_S + cb, sv);
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 16; ++n)
                    sv[n] = F * sv[n] + ds[n];
                tmem_st16(tq + T_S + cb, sv);
                st_tile8(base_u32 + Ly.S, KD, R, cb, &sv[0]);
                st_tile8(base_u32 + Ly.S, KD, R, cb + 8, &sv[8]);
            }
            tmem_st_wait();
            if (R >= CC) {
                const int t = R - CC;
                const bool live = t < Cl;
                const long orow = (vh * T + c0 + t) * p.dv + n0;
#pragma unroll
                for (int cb = 0; cb < NVC; cb += 16) {
                    float ov[16];
                    tmem_ld16(tq + T_PO + cb, ov);
                    tmem_ld_wait();
                    if (live) {
                        if constexpr (OUT_BF16) {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow + cb);
                            dst[0] = make_uint4(pack_bf16(ov[0], ov[1]), pack_bf16(ov[2], ov[3]),
                                                pack_bf16(ov[4], ov[5]), pack_bf16(ov[6], ov[7]));
                            dst[1] = make_uint4(pack_bf16(ov[8], ov[9]), pack_bf16(ov[10], ov[11]),
                                                pack_bf16(ov[12], ov[13]), pack_bf16(ov[14], ov[15]));
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow + cb);
#pragma unroll
                            for (int n = 0; n < 4; ++n)
                                dst[n] = make_float4(ov[4 * n], ov[4 * n + 1], ov[4 * n + 2], ov[4 * n + 3]);
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[S_READY]);
        }
        if (p.S_final != nullptr && !*abort_flag) {
            float *dst = p.S_final + (vh * KD + R) * p.dv + n0;
#pragma unroll
            for (int cb = 0; cb < NVC; cb += 16) {
                float sv[16];
                tmem_ld16(tq + T_S + cb, sv);
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 16; n += 4)
                    *reinterpret_cast<float4 *>(dst + cb + n) = make_float4(sv[n], sv[n + 1], sv[n + 2], sv[n + 3]);
            }
        }
    } else {
        // ------------------------------------------------------------ intra team
        const int itid = tid - W_INTRA0 * 32;
        const int q4 = warp & 3;                   // TMEM lane quarter
        const int h = (warp - W_INTRA0) >> 2;      // column half
        const int R = 32 * q4 + lane;
        for (int c = 0; c < N; ++c) {
            const int s = c & 1;
            const uint32_t par = c & 1;
            const uint32_t wqk = base_u32 + (s ? Ly.wqk[1] : Ly.wqk[0]), vl = base_u32 + (s ? Ly.vl[1] : Ly.vl[0]);
            Gates *gt = s ? gates1 : gates0;
            if (named_vote_or(NB_INTRA, N_INTRA,
                              !wait_or_abort(&bars[FULL0 + s], (c >> 1) & 1, abort_flag)))
                break;
            // cumulative log-decay and decay factors (one warp)
            if (warp == W_INTRA0) {
                float a0 = gt->graw[lane], a1 = gt->graw[32 + lane];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, a0, off);
                    const float y1 = __shfl_up_sync(0xffffffffu, a1, off);
                    if (lane >= off) {
                        a0 += y0;
                        a1 += y1;
                    }
                }
                a1 += __shfl_sync(0xffffffffu, a0, 31);
                const float lc = __shfl_sync(0xffffffffu, a1, 31);
                gt->lam[lane] = a0;
                gt->lam[32 + lane] = a1;
                gt->ea[lane] = __expf(a0);
                gt->ea[32 + lane] = __expf(a1);
                gt->eb[lane] = __expf(lc - a0);
                gt->eb[32 + lane] = __expf(lc - a1);
            }
            if (named_vote_or(NB_INTRA, N_INTRA, !wait_or_abort(&bars[GRAM_FULL], par, abort_flag)))
                break;
            tc_fence_after();
            // decay masks: rows 0-63 of the Gram are Q K^T (-> L), rows 64-127 K K^T (-> M)
            {
                const int j0 = 32 * h;
                float gv0[16], gv1[16];
                tmem_ld16(tq + T_GRAM + j0, gv0);
                tmem_ld16(tq + T_GRAM + j0 + 16, gv1);
                tmem_ld_wait();
                const bool qrow = R < CC;
                const int t = qrow ? R : R - CC;
                const float lt = gt->lam[t];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int jb = j0 + 16 * hh;
                    float lj[16], bj[16], out[16];
#pragma unroll
                    for (int u = 0; u < 16; u += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(&gt->lam[jb + u]);
                        const float4 b4 = *reinterpret_cast<const float4 *>(&gt->beta[jb + u]);
                        lj[u] = l4.x; lj[u + 1] = l4.y; lj[u + 2] = l4.z; lj[u + 3] = l4.w;
                        bj[u] = b4.x; bj[u + 1] = b4.y; bj[u + 2] = b4.z; bj[u + 3] = b4.w;
                    }
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int j = jb + u;
                        const float g = hh ? gv1[u] : gv0[u];
                        const float d = __expf(lt - lj[u]) * g;
                        out[u] = qrow ? ((j <= t) ? d : 0.f) : ((j < t) ? bj[u] * d : 0.f);
                    }
                    if (qrow) {
                        st_tile8(vl, 128, CC + t, jb, &out[0]);
                        st_tile8(vl, 128, CC + t, jb + 8, &out[8]);
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; u += 4)
                            *reinterpret_cast<float4 *>(&Mf[t * LDM + jb + u]) =
                                make_float4(out[u], out[u + 1], out[u + 2], out[u + 3]);
                    }
                }
            }
            tc_fence_before();
            // Qbar = diag(e^Lambda) Q, in place (the Gram MMA that read Q is done)
            {
                const int t = itid >> 2;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = (itid & 3) * 32 + 8 * u;
                    const uint32_t addr = wqk + sw128_off(192, 64 + t, col);
                    uint32_t a0, a1, a2, a3;
                    ld_shared_v4(addr, a0, a1, a2, a3);
                    const float e = gt->ea[t];
                    st_shared_v4(addr, pack_bf16(e * bf16lo(a0), e * bf16hi(a0)),
                                 pack_bf16(e * bf16lo(a1), e * bf16hi(a1)),
                                 pack_bf16(e * bf16lo(a2), e * bf16hi(a2)),
                                 pack_bf16(e * bf16lo(a3), e * bf16hi(a3)));
                }
            }
            fence_proxy_async_smem();
            named_sync(NB_INTRA, N_INTRA);
            if (itid == 0)
                mbar_arrive(&bars[GRAM_FREE]);
            // A = (I + M)^{-1}: exact 16 x 16 diagonal blocks (fp32) ...
            if (itid < 64) {
                const int blk = itid >> 4, cc = itid & 15, o = 16 * blk;
                float x[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float *mrow = Mf + (o + t) * LDM + o;
                    float acc = (t == cc) ? 1.f : 0.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (j < t)
                            acc -= mrow[j] * x[j];
                    x[t] = acc;
                }
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    Af[(o + t) * LDM + o + cc] = x[t];
            }
            named_sync(NB_INTRA, N_INTRA);
            // ... merged pairwise: X21 = -X22 (M21 X11), 16 -> 32
            {
                const int pr = itid >> 7, r = (itid >> 3) & 15, c2 = (itid & 7) * 2, o = 32 * pr;
                float mr[16];
#pragma unroll
                for (int l = 0; l < 16; l += 4) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(&Mf[(o + 16 + r) * LDM + o + l]);
                    mr[l] = m4.x; mr[l + 1] = m4.y; mr[l + 2] = m4.z; mr[l + 3] = m4.w;
                }
                float t0 = 0.f, t1 = 0.f;
#pragma unroll
                for (int l = 0; l < 16; ++l) {
                    const float2 a2 = *reinterpret_cast<const float2 *>(&Af[(o + l) * LDM + o + c2]);
                    t0 += mr[l] * a2.x;
                    t1 += mr[l] * a2.y;
                }
                *reinterpret_cast<float2 *>(&Tf[(pr * 16 + r) * LDT + c2]) = make_float2(t0, t1);
                named_sync(NB_INTRA, N_INTRA);
                float ar[16];
#pragma unroll
                for (int l = 0; l < 16; l += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(&Af[(o + 16 + r) * LDM + o + 16 + l]);
                    ar[l] = a4.x; ar[l + 1] = a4.y; ar[l + 2] = a4.z; ar[l + 3] = a4.w;
                }
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int l = 0; l < 16; ++l) {
                    const float2 t2 = *reinterpret_cast<const float2 *>(&Tf[(pr * 16 + l) * LDT + c2]);
                    x0 += ar[l] * t2.x;
                    x1 += ar[l] * t2.y;
                }
                *reinterpret_cast<float2 *>(&Af[(o + 16 + r) * LDM + o + c2]) = make_float2(-x0, -x1);
            }
            named_sync(NB_INTRA, N_INTRA);
            // ... and 32 -> 64
            {
                const int r = itid >> 3, c4 = (itid & 7) * 4;
                float mr[32];
#pragma unroll
                for (int l = 0; l < 32; l += 4) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(&Mf[(32 + r) * LDM + l]);
                    mr[l] = m4.x; mr[l + 1] = m4.y; mr[l + 2] = m4.z; mr[l + 3] = m4.w;
                }
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f), acc2 = acc;
#pragma unroll
                for (int l = 0; l < 32; l += 2) {
                    const float4 a = *reinterpret_cast<const float4 *>(&Af[l * LDM + c4]);
                    const float4 b2 = *reinterpret_cast<const float4 *>(&Af[(l + 1) * LDM + c4]);
                    acc.x += mr[l] * a.x; acc.y += mr[l] * a.y; acc.z += mr[l] * a.z; acc.w += mr[l] * a.w;
                    acc2.x += mr[l + 1] * b2.x; acc2.y += mr[l + 1] * b2.y;
                    acc2.z += mr[l + 1] * b2.z; acc2.w += mr[l + 1] * b2.w;
                }
                *reinterpret_cast<float4 *>(&Tf[r * LDT + c4]) =
                    make_float4(acc.x + acc2.x, acc.y + acc2.y, acc.z + acc2.z, acc.w + acc2.w);
                named_sync(NB_INTRA, N_INTRA);
                float ar[32];
#pragma unroll
                for (int l = 0; l < 32; l += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(&Af[(32 + r) * LDM + 32 + l]);
                    ar[l] = a4.x; ar[l + 1] = a4.y; ar[l + 2] = a4.z; ar[l + 3] = a4.w;
                }
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f), x2 = x;
#pragma unroll
                for (int l = 0; l < 32; l += 2) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(&Tf[l * LDT + c4]);
                    const float4 u4 = *reinterpret_cast<const float4 *>(&Tf[(l + 1) * LDT + c4]);
                    x.x += ar[l] * t4.x; x.y += ar[l] * t4.y; x.z += ar[l] * t4.z; x.w += ar[l] * t4.w;
                    x2.x += ar[l + 1] * u4.x; x2.y += ar[l + 1] * u4.y;
                    x2.z += ar[l + 1] * u4.z; x2.w += ar[l + 1] * u4.w;
                }
                *reinterpret_cast<float4 *>(&Af[(32 + r) * LDM + c4]) =
                    make_float4(-(x.x + x2.x), -(x.y + x2.y), -(x.z + x2.z), -(x.w + x2.w));
            }
            named_sync(NB_INTRA, N_INTRA);
            // [Ab; Abe] = [diag(beta) A; diag(beta) A diag(e^Lambda)]  (bf16, 128 x 64)
#pragma unroll
            for (int rep = 0; rep < (CC * 8) / N_INTRA; ++rep) {
                const int u = itid + rep * N_INTRA;
                const int t = u >> 3, j = (u & 7) * 8;
                const float bt = gt->beta[t];
                const float4 a0 = *reinterpret_cast<const float4 *>(&Af[t * LDM + j]);
                const float4 a1 = *reinterpret_cast<const float4 *>(&Af[t * LDM + j + 4]);
                const float4 e0 = *reinterpret_cast<const float4 *>(&gt->ea[j]);
                const float4 e1 = *reinterpret_cast<const float4 *>(&gt->ea[j + 4]);
                const float a[8] = {bt * a0.x, bt * a0.y, bt * a0.z, bt * a0.w,
                                    bt * a1.x, bt * a1.y, bt * a1.z, bt * a1.w};
                const float ae[8] = {a[0] * e0.x, a[1] * e0.y, a[2] * e0.z, a[3] * e0.w,
                                     a[4] * e1.x, a[5] * e1.y, a[6] * e1.z, a[7] * e1.w};
                st_tile8(base_u32 + Ly.AB, 128, t, j, a);
                st_tile8(base_u32 + Ly.AB, 128, CC + t, j, ae);
            }
            fence_proxy_async_smem();
            named_sync(NB_INTRA, N_INTRA);
            if (itid == 0)
                mbar_arrive(&bars[AB_READY]);
            if (named_vote_or(NB_INTRA, N_INTRA, !wait_or_abort(&bars[WU_FULL], par, abort_flag)))
                break;
            tc_fence_after();
            // W (TMEM rows 64-127) -> rows 0-63 of the W | Q | K blocks
            if (q4 >= 2) {
                const int t = R - CC;
#pragma unroll
                for (int cb = 0; cb < 64; cb += 16) {
                    float wv[16];
                    tmem_ld16(tq + T_W + 64 * h + cb, wv);
                    tmem_ld_wait();
                    st_tile8(wqk, 192, t, 64 * h + cb, &wv[0]);
                    st_tile8(wqk, 192, t, 64 * h + cb + 8, &wv[8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_INTRA, N_INTRA);
            if (itid == 0)
                mbar_arrive(&bars[W_READY]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <bool OB>
int launch(const Params &p, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, KD, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mk, p.k, KD, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CC))
        return 6;
    const Plan Ly = plan();
    auto kern = ws_kernel<OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    TcArgs a;
    a.p = p;
    a.nvt = p.dv / NVC;
    dim3 grid(a.nvt * p.Hv, p.B);
    kern<<<grid, NTHR, Ly.total, stream>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

inline bool supports(const Params &p)
{
    return p.in_bf16 && p.G == 1 && p.C == CC && p.dk == KD && p.dv % NVC == 0 && !p.neumann &&
           p.T >= 1 && p.B <= 65535;
}

}  // namespace ws
