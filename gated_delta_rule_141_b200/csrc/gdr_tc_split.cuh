// gdr_tc_split.cuh -- second pass of the two-pass tensor-core path: the
// inter-chunk state recurrence and the readout, for key width dk = 128, chunk
// C = 64, 64 value columns per CTA, any decay grouping.  The chunk-local
// factors T = diag(beta) (I + M)^{-1} and L come from the first pass
// (gdr_tc_prep.cuh), so the serial chain per chunk holds only the state
// products ("Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta
// Attention for TPUs", §2.1, §2.3 Table 2, §2.4.2):
//   W = T Kbar,  U = T V                     (off the chain, one chunk ahead)
//   P = W S,  E = U - P                      (chain)
//   S <- F S + Khat^T E,  O = Qbar S + L E   (chain; O leaves off the chain)
// with Kbar = k e^{Lambda_t}, Khat = k e^{Lambda_C - Lambda_t},
// Qbar = q e^{Lambda_t}, F = diag(e^{Lambda_C}) -- all factors <= 1.
// For the scalar gate the factors are row / column scalings:
// W = (T diag(e^Lambda)) K, Khat^T E = K^T (diag(e^{Lambda_C - Lambda}) E) and
// Qbar S = diag(e^Lambda) (Q S), applied by the epilogue.
//
// Roles (warp-specialised, hand-offs through mbarriers):
//   warp 0      producer: TMA q, k, v; bulk copies of T and L; 2-stage ring
//   warp 1      MMA issuer (one thread)
//   warps 2-9   state chain: S (fp32, TMEM) -> bf16 operand, E = U - P; two
//               warps per TMEM lane quarter, each lane on 32 of the 64 columns
//   warps 10-13 W read-back: TMEM fp32 -> bf16 operand tile (one chunk ahead)
//   warps 14-15 epilogue: O = f (Q S) + L E from TMEM to global memory
// Everything decayed (Abe, Qbar, Khat, Kbar, the per-token factors, F) comes
// from the first pass's record, so no role here evaluates an exponential.
// Stage s holds [W | Q | K] (rows 0-63 | 64-127 | 128-191, 128 columns),
// [V | L] (rows 0-63 | 64-127, 64 columns) and [Ab | Abe] (T, and for the
// scalar gate T diag(e^Lambda)).  MMA operands are stacked so that M = 128:
//   [Ab; Abe] V -> U (rows 0-63),  [Ab; Abe] K -> W (rows 64-127, scalar gate)
//   or [Ab; *] Kbar -> W (rows 0-63),  [W; Q] S -> P, Q S (Q = Qbar for
//   grouped / per-channel gates), Khat^T E onto S,  [V; L] E -> L E (rows 64-127).

namespace split {

constexpr int NWARP = 16;
constexpr int NTHR = NWARP * 32;   // 512
constexpr int CC = 64;
constexpr int KD = 128;
constexpr int NVC = 64;
constexpr int W_PROD = 0, W_MMA = 1, W_STATE0 = 2, W_PREP0 = 10, W_EPI0 = 14;
constexpr int N_STATE = 256, N_PREP = 128, N_EPI = 64;
constexpr int NB_STATE = 1, NB_PREP = 2, NB_EPI = 3;   // named barriers

constexpr uint32_t T_U = 0;        // [Ab; *] V              64 cols
constexpr uint32_t T_W = 64;       // [Ab; Abe] K / [Ab; *] Kbar   128 cols
constexpr uint32_t T_PO = 192;     // two buffers of 64 cols: [W; Q] S
constexpr uint32_t T_S = 320;      // fp32 state, 64 cols
constexpr uint32_t T_LE = 384;     // two buffers of 64 cols: [V; L] E
constexpr uint32_t TMEM_COLS = 512;

enum Bar { FULL0, FULL1, FREE0, FREE1, WU_FULL, W_READY, S_READY, P_FULL, E_READY,
           UPD_DONE, OUT0, OUT1, OFREE0, OFREE1, DRAIN, NBARS };

struct Gates {                        // landed by bulk copies from the first pass's record
    float ea[CC], eb[CC];             // scalar gate: e^{Lambda_t}, e^{Lambda_C - Lambda_t}
    float F[KD];                      // e^{Lambda_C} per key channel (F[0] for the scalar gate)
};

struct Plan {
    uint32_t wqk[2], vl[2], ab[2], gates[2], kb[2];
    uint32_t S, E, Eh, bar, misc, total;
};

// Scalar gate: an E_hat tile; grouped / per-channel gates: a Kbar tile per stage.
__host__ __device__ inline Plan plan(bool scalar)
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
        s.ab[i] = take(128 * 128);
        s.gates[i] = take(sizeof(Gates));
        s.kb[i] = scalar ? 0 : take((KD / 64) * CC * 128);
    }
    s.S = take(KD * NVC * 2);
    s.E = take(CC * NVC * 2);
    s.Eh = scalar ? take(CC * NVC * 2) : s.E;
    s.bar = take(NBARS * 8 + 16);
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

struct SplitArgs {
    Params p;
    const uint8_t *factors;   // first-pass output, [B * Hk * nchunks][rec_bytes]
    uint32_t rec_bytes;       // prep::CHUNK_BYTES (scalar gate) or prep::EXT_BYTES
    int nvt;
    int nchunks;
};

template <bool OUT_BF16>
__global__ void __launch_bounds__(NTHR, 1)
split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const SplitArgs args)
{
    using namespace ptx;
    using ws::wait_or_abort;
    using ws::named_sync;
    using ws::named_vote_or;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const bool scalar = p.G == 1;
    const Plan Ly = plan(scalar);
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
    const int N = args.nchunks;

    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 4);
    auto gates_of = [&](int s) { return reinterpret_cast<Gates *>(base + Ly.gates[s]); };
    auto wqk_of = [&](int s) { return base_u32 + Ly.wqk[s]; };
    auto vl_of = [&](int s) { return base_u32 + Ly.vl[s]; };
    auto ab_of = [&](int s) { return base_u32 + Ly.ab[s]; };
    const uint32_t S_T = base_u32 + Ly.S, E_T = base_u32 + Ly.E, EH_T = base_u32 + Ly.Eh;

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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int R = 32 * (warp & 3) + lane;     // TMEM lane of this thread

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        uint32_t pend = 0, par0 = 0, par1 = 0;
        for (int c = 0; c < N; ++c) {
            const int s = c & 1;
            if (c >= 2) {
                const bool ok = wait_or_abort(&bars[FREE0 + s], ((c >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            const long c0 = (long)c * CC;
            if (lane == 0) {
                const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
                uint64_t *full = &bars[FULL0 + s];
                if (scalar) {
                    // q, k as loaded; Abe and the per-token factors from the first pass
                    constexpr uint32_t fac_bytes = prep::SC_BYTES - prep::SC_EA;
                    mbar_arrive_expect_tx(full, 2u * CC * KD * 2 + CC * NVC * 2 + 3 * prep::IMG + fac_bytes);
                    for (int kb = 0; kb < KD / 64; ++kb) {
                        uint8_t *blk = base + Ly.wqk[s] + kb * 192 * 128;
                        tma_load_3d(blk + 64 * 128, &tm_q, full, 64 * kb, (int)c0, (int)kh);
                        tma_load_3d(blk + 128 * 128, &tm_k, full, 64 * kb, (int)c0, (int)kh);
                    }
                    bulk_load(base + Ly.ab[s] + 64 * 128, fac + prep::SC_ABE, prep::IMG, full);
                    bulk_load(gates_of(s)->ea, fac + prep::SC_EA, fac_bytes, full);
                } else {
                    // Qbar, Khat (per 64-column block), Kbar and F, decayed by the first pass
                    mbar_arrive_expect_tx(full, 8u * prep::IMG + KD * 4 + CC * NVC * 2);
                    for (int kb = 0; kb < KD / 64; ++kb) {
                        uint8_t *blk = base + Ly.wqk[s] + kb * 192 * 128;
                        bulk_load(blk + 64 * 128, fac + prep::EXT_QB + kb * prep::IMG, prep::IMG, full);
                        bulk_load(blk + 128 * 128, fac + prep::EXT_KH + kb * prep::IMG, prep::IMG, full);
                    }
                    bulk_load(base + Ly.kb[s], fac + prep::EXT_KB, 2 * prep::IMG, full);
                    bulk_load(gates_of(s)->F, fac + prep::EXT_F, KD * 4, full);
                }
                tma_load_3d(base + Ly.vl[s], &tm_v, full, n0, (int)c0, (int)vh);
                bulk_load(base + Ly.ab[s], fac, prep::IMG, full);
                bulk_load(base + Ly.vl[s] + 64 * 128, fac + prep::IMG, prep::IMG, full);
            }
            pend |= 1u << s;
            if (s)
                par1 = (c >> 1) & 1;
            else
                par0 = (c >> 1) & 1;
        }
        if (lane == 0) {   // drain loads that may still be landing (bounded)
            if (pend & 1u)
                mbar_wait(&bars[FULL0], par0, 200000000ull);
            if (pend & 2u)
                mbar_wait(&bars[FULL1], par1, 200000000ull);
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_u = idesc_bf16(128, NVC, false, true);
            const uint32_t id_w = idesc_bf16(128, KD, false, true);
            const uint32_t id_po = idesc_bf16(128, NVC, false, true);
            const uint32_t id_s = idesc_bf16(KD, NVC, true, true);
            // descriptors at k = 0; a K step adds its byte offset / 16 to the start field
            // (K-major: 32 bytes per 16 columns inside a 64-column block, rows * 128 per
            // block; MN-major: 16 rows of 128 bytes per 16-deep step)
            // (stage 1 sits a fixed byte distance after stage 0: one more add)
            const uint64_t d_ab0 = desc_kmajor(ab_of(0), 128, 0, 0);
            const uint64_t d_v0 = desc_mnmajor(vl_of(0), 128, 0, 0);
            const uint64_t d_wq0 = desc_kmajor(wqk_of(0), 192, 0, 0);
            const uint64_t d_kt0 = desc_mnmajor(wqk_of(0), 192, 128, 0);
            const uint64_t d_vl0 = desc_kmajor(vl_of(0), 128, 0, 0);
            const uint64_t d_kb0 = scalar ? 0 : desc_mnmajor(base_u32 + Ly.kb[0], CC, 0, 0);
            const uint64_t dkb = (Ly.kb[1] - Ly.kb[0]) >> 4;
            const uint64_t dab = (Ly.ab[1] - Ly.ab[0]) >> 4, dvl = (Ly.vl[1] - Ly.vl[0]) >> 4;
            const uint64_t dwq = (Ly.wqk[1] - Ly.wqk[0]) >> 4;
            const uint64_t d_s = desc_mnmajor(S_T, KD, 0, 0);
            const uint64_t d_e = desc_mnmajor(scalar ? EH_T : E_T, CC, 0, 0);
            const uint64_t d_eo = desc_mnmajor(E_T, CC, 0, 0);
            auto kstep = [](int k0, int rows) {
                return static_cast<uint64_t>(((k0 >> 6) * rows * 128 + (k0 & 63) * 2) >> 4);
            };
            auto mstep = [](int k0) { return static_cast<uint64_t>(k0 * 8); };
            auto wu = [&](int st) {
                const uint64_t a0 = d_ab0 + st * dab, v0 = d_v0 + st * dvl;
                const uint64_t k0d = scalar ? d_kt0 + st * dwq : d_kb0 + st * dkb;
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    mma_bf16(tmem + T_U, a0 + kstep(k0, 128), v0 + mstep(k0), id_u, k0 > 0);
                    mma_bf16(tmem + T_W, a0 + kstep(k0, 128), k0d + mstep(k0), id_w, k0 > 0);
                }
                mma_commit(&bars[WU_FULL]);
            };
            bool ok = true;
            if (N > 0) {
                ok = wait_or_abort(&bars[FULL0], 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    wu(0);
                }
            }
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1, ob = c & 1;
                const uint32_t par = c & 1;
                if (!(ok = wait_or_abort(&bars[W_READY], par, abort_flag)))
                    break;
                if (!(ok = wait_or_abort(&bars[S_READY], par, abort_flag)))
                    break;
                if (c >= 2 && !(ok = wait_or_abort(&bars[OFREE0 + ob], ((c >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint64_t wq = d_wq0 + s * dwq, kt = d_kt0 + s * dwq, vl = d_vl0 + s * dvl;
                for (int k0 = 0; k0 < KD; k0 += 16)
                    mma_bf16(tmem + T_PO + 64 * ob, wq + kstep(k0, 192), d_s + mstep(k0), id_po, k0 > 0);
                mma_commit(&bars[P_FULL]);
                if (!(ok = wait_or_abort(&bars[E_READY], par, abort_flag)))
                    break;
                tc_fence_after();
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_S, kt + mstep(k0), d_e + mstep(k0), id_s, 1u);
                mma_commit(&bars[UPD_DONE]);
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_LE + 64 * ob, vl + kstep(k0, 128), d_eo + mstep(k0), id_po, k0 > 0);
                mma_commit(&bars[OUT0 + ob]);
                mma_commit(&bars[FREE0 + s]);
                if (c + 1 < N) {
                    if (!(ok = wait_or_abort(&bars[FULL0 + (s ^ 1)], ((c + 1) >> 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    wu(s ^ 1);
                }
            }
            // whatever was issued must finish before tensor memory is released
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, 200000000ull);
        }
    } else if (warp < W_PREP0) {
        // ------------------------------------------------------------ state chain
        const int stid = tid - W_STATE0 * 32;
        const int cs = 32 * ((warp - W_STATE0) >> 2);   // this lane's 32 of the 64 columns
        {
            float sv[32];
#pragma unroll
            for (int n = 0; n < 32; ++n)
                sv[n] = 0.f;
            if (p.S0 != nullptr) {
                const float *src = p.S0 + (vh * KD + R) * p.dv + n0 + cs;
#pragma unroll
                for (int n = 0; n < 32; n += 4) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(src + n);
                    sv[n] = v4.x; sv[n + 1] = v4.y; sv[n + 2] = v4.z; sv[n + 3] = v4.w;
                }
            }
            tmem_st16(tq + T_S + cs, *reinterpret_cast<float(*)[16]>(&sv[0]));
            tmem_st16(tq + T_S + cs + 16, *reinterpret_cast<float(*)[16]>(&sv[16]));
        }
        tmem_st_wait();
        bool ok = true;
        for (int c = 0; c < N; ++c) {
            const int s = c & 1, ob = c & 1;
            const uint32_t par = c & 1;
            if (c >= 1 &&
                named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[UPD_DONE], (c - 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            if (named_vote_or(NB_STATE, N_STATE,
                              !wait_or_abort(&bars[FULL0 + s], (c >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const Gates *gt = gates_of(s);
            const float F = scalar ? gt->F[0] : gt->F[R];
            // S_{c-1} -> bf16 operand; T_S <- F S_{c-1} (the update MMA accumulates onto it)
            {
                float s0[16], s1[16];
                tmem_ld16(tq + T_S + cs, s0);
                tmem_ld16(tq + T_S + cs + 16, s1);
                tmem_ld_wait();
                st_tile8(S_T, KD, R, cs, &s0[0]);
                st_tile8(S_T, KD, R, cs + 8, &s0[8]);
                st_tile8(S_T, KD, R, cs + 16, &s1[0]);
                st_tile8(S_T, KD, R, cs + 24, &s1[8]);
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    s0[n] *= F;
                    s1[n] *= F;
                }
                tmem_st16(tq + T_S + cs, s0);
                tmem_st16(tq + T_S + cs + 16, s1);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[S_READY]);
            if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[P_FULL], par, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (R < CC) {   // warps of lane quarters 0 and 1: rows t of E
                const float f = scalar ? gt->eb[R] : 1.f;
                float p0[16], p1[16], u0[16], u1[16];
                tmem_ld16(tq + T_PO + 64 * ob + cs, p0);
                tmem_ld16(tq + T_PO + 64 * ob + cs + 16, p1);
                tmem_ld16(tq + T_U + cs, u0);
                tmem_ld16(tq + T_U + cs + 16, u1);
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    u0[n] -= p0[n];
                    u1[n] -= p1[n];
                }
                st_tile8(E_T, CC, R, cs, &u0[0]);
                st_tile8(E_T, CC, R, cs + 8, &u0[8]);
                st_tile8(E_T, CC, R, cs + 16, &u1[0]);
                st_tile8(E_T, CC, R, cs + 24, &u1[8]);
                if (scalar) {
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        u0[n] *= f;
                        u1[n] *= f;
                    }
                    st_tile8(EH_T, CC, R, cs, &u0[0]);
                    st_tile8(EH_T, CC, R, cs + 8, &u0[8]);
                    st_tile8(EH_T, CC, R, cs + 16, &u1[0]);
                    st_tile8(EH_T, CC, R, cs + 24, &u1[8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[E_READY]);
        }
        if (ok && N > 0 &&
            named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[UPD_DONE], (N - 1) & 1, abort_flag)))
            ok = false;
        if (ok && p.S_final != nullptr) {
            tc_fence_after();
            float *dst = p.S_final + (vh * KD + R) * p.dv + n0 + cs;
            float s0[16], s1[16];
            tmem_ld16(tq + T_S + cs, s0);
            tmem_ld16(tq + T_S + cs + 16, s1);
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 16; n += 4) {
                *reinterpret_cast<float4 *>(dst + n) = make_float4(s0[n], s0[n + 1], s0[n + 2], s0[n + 3]);
                *reinterpret_cast<float4 *>(dst + 16 + n) = make_float4(s1[n], s1[n + 1], s1[n + 2], s1[n + 3]);
            }
        }
    } else if (warp < W_EPI0) {
        // ------------------------------------------------------------ W read-back
        const int ptid = tid - W_PREP0 * 32;
        for (int c = 0; c < N; ++c) {
            const uint32_t wqk = wqk_of(c & 1);
            // W read-back: rows 64-127 of T_W (scalar gate) or rows 0-63
            if (named_vote_or(NB_PREP, N_PREP, !wait_or_abort(&bars[WU_FULL], c & 1, abort_flag)))
                break;
            tc_fence_after();
            const bool mine = scalar ? (R >= CC) : (R < CC);
            if (mine) {
                const int t = scalar ? R - CC : R;
#pragma unroll
                for (int cb = 0; cb < KD; cb += 16) {
                    float wv[16];
                    tmem_ld16(tq + T_W + cb, wv);
                    tmem_ld_wait();
                    st_tile8(wqk, 192, t, cb, &wv[0]);
                    st_tile8(wqk, 192, t, cb + 8, &wv[8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_PREP, N_PREP);
            if (ptid == 0)
                mbar_arrive(&bars[W_READY]);
        }
    } else {
        // ------------------------------------------------------------ epilogue (O rows in lanes 64-127)
        const int etid = tid - W_EPI0 * 32;
        const int t = R - CC;
        for (int c = 0; c < N; ++c) {
            const int ob = c & 1;
            const long c0 = (long)c * CC;
            const int Cl = (int)min((long)CC, T - c0);
            // Qbar S = e^{Lambda_t} (Q S) for the scalar gate (factor from the record)
            const float f = scalar ? reinterpret_cast<const float *>(
                                         args.factors + (size_t)(kh * N + c) * args.rec_bytes +
                                         prep::SC_EA)[t]
                                   : 1.f;
            if (named_vote_or(NB_EPI, N_EPI, !wait_or_abort(&bars[OUT0 + ob], (c >> 1) & 1, abort_flag)))
                break;
            tc_fence_after();
            const bool live = t < Cl;
            const long orow = (vh * T + c0 + t) * p.dv + n0;
#pragma unroll
            for (int cb = 0; cb < NVC; cb += 16) {
                float qs[16], le[16], ov[16];
                tmem_ld16(tq + T_PO + 64 * ob + cb, qs);
                tmem_ld16(tq + T_LE + 64 * ob + cb, le);
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 16; ++n)
                    ov[n] = f * qs[n] + le[n];
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
            tc_fence_before();
            named_sync(NB_EPI, N_EPI);
            if (etid == 0)
                mbar_arrive(&bars[OFREE0 + ob]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

inline bool supports(const Params &p)
{
    return prep::supports(p) && p.dk == KD && p.dv % NVC == 0 && p.G <= KD && p.T >= 1;
}

template <bool OB>
int launch(const Params &p, const void *factors, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, KD, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mk, p.k, KD, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CC))
        return 6;
    const Plan Ly = plan(p.G == 1);
    auto kern = split_kernel<OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    SplitArgs a;
    a.p = p;
    a.factors = static_cast<const uint8_t *>(factors);
    a.rec_bytes = prep::rec_bytes(p);
    a.nvt = p.dv / NVC;
    a.nchunks = prep::nchunks(p);
    dim3 grid(a.nvt * p.Hv, p.B);
    kern<<<grid, NTHR, Ly.total, stream>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace split
