// gdr_tc_ab128.cuh -- first launch of the segment-parallel 128-column state pass:
// each segment's end state from zero and its transition, two chains in one CTA.
// Included by gdr_tc.cu after gdr_tc_split.cuh (its launch is in gdr_tc_split128.cuh).
//
// A segment of chunks maps the state it starts from affinely, S -> Atil S + Btil,
// with Atil = prod (F_c - Khat_c^T W_c) and Btil its end state from S = 0 ("Systolic
// Linear Attention: Co-Designing Tile-Grouped Gated Delta Attention for TPUs",
// §2.1, §2.4.2; the chunk recurrence E = T V - W S, S <- F S + Khat^T E).  Both are
// the same chain over the same chunk operands: Btil runs it on 128 value columns
// from zero with the values injected (E = U - W S), Atil on the 128 columns of the
// identity with none (E = -W S).  One CTA runs the two chains of a (key head,
// segment) side by side:
//   * the chunk operands (W, Khat, F) are loaded once for both;
//   * the state warps alternate between the chains (S_A, S_B, E_A, E_B), so that
//     each chain's products run on the tensor core while the warps convert the
//     other chain's tensor-memory results to bf16 operands.
// Value tiles beyond the first of a key head (dv > 128, or several value heads per
// key head) run the value chain alone.
//
// The chunk's rows need only M = 64 products (the 64-row accumulator puts row m in
// tensor-memory lane 32 (m / 16) + m % 16):
//   T V -> U,  -W S onto it -> E = U - W S,  Khat^T E onto F S (M = dk = 128).
// Tensor memory: R_A 0, R_B 128, S_A 256, S_B 384 (fp32, 128 columns each).
// Pairs (the chunk-128 Neumann inverses run as 64-token halves): a second half adds
// the first half's correction, E2 += Y E1, as one more product [Y; *] E1 onto its R
// before the E phase; E1 is still the chain's bf16 E operand then, and Y (from the
// first half's record) lands just above the second-half stage's [-W; Khat].
//
// Roles: warp 0 producer (W, Khat, F), warp 1 MMA issuer, warp 2 producer (T, V),
// warp 3 idle, warps 4-19 state (S row in TMEM lane 32 (w % 4) + lane, 32 of the
// 128 columns each; E row 16 (w % 4) + lane in lanes 0-15 of every warp).

namespace split {

namespace ab {

constexpr int NV = 128;            // value columns per chain
constexpr int NWARP = 20;
constexpr int NTHR = NWARP * 32;   // 640
constexpr int W_PX = 0, W_MMA = 1, W_PY = 2, W_STATE0 = 4;
constexpr int N_STATE = 512;
constexpr int NB_STATE = 1;
constexpr uint32_t T_RA = 0, T_RB = 128, T_SA = 256, T_SB = 384;

enum Bar { FULL0, FULL1, FREE0, FREE1, S_READY_A, S_READY_B, P_FULL_A, P_FULL_B, E_READY_A,
           E_READY_B, UPD_A, UPD_B, DRAIN, NBARS };

struct Plan {
    uint32_t y, wk[2], tv[2], gates[2];
    uint32_t S[2], E[2], bar, misc, total;
};

// Stage: [-W | Khat] (rows 0-63 | 64-127, two 64-column blocks), then T (64 rows)
// and V (64 rows, two 64-column blocks).
__host__ __device__ inline Plan plan(bool pair = false)
{
    Plan s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    s.y = 0;
    for (int i = 0; i < 2; ++i) {
        if (pair && i == 1)   // second halves (segments start at even chunks)
            s.y = take(prep::IMG);
        s.wk[i] = take((KD / 64) * 128 * 128);
        s.tv[i] = take(prep::IMG + 2 * 64 * 128);
    }
    for (int i = 0; i < 2; ++i) {
        s.S[i] = take(KD * NV * 2);
        s.E[i] = take(CC * NV * 2);
    }
    s.gates[0] = take(2 * KD * 4 + NBARS * 8 + 16);
    s.gates[1] = s.gates[0] + KD * 4;
    s.bar = s.gates[0] + 2 * KD * 4;
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

__global__ void __launch_bounds__(NTHR, 1)
ab128_kernel(const __grid_constant__ CUtensorMap tm_v, const SplitArgs args)
{
    using namespace ptx;
    using ws::named_sync;
    using ws::named_vote_or;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const bool pair = args.pair != 0;
    const Plan Ly = plan(pair);
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = (int)blockIdx.x % args.nvt;
    const int hv = (int)blockIdx.x / args.nvt;
    const int b = blockIdx.y;
    const int hk = hv / p.R;
    const bool dual = nt == 0 && hv % p.R == 0;   // this CTA also runs the key head's transition
    const int n0 = nt * NV;
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int N = args.nchunks;
    const int seg = blockIdx.z;
    const int cbeg = seg * args.seg_len;
    const int nloc = min(args.seg_len, N - cbeg);

    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 4);
    auto fgate = [&](int s) { return reinterpret_cast<float *>(base + stage(Ly.gates, s)); };

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)   // FULL: two producers; FREE: the MMAs and the state warps
            mbar_init(&bars[i], i <= FREE1 ? 2 : 1);
        *abort_flag = 0;
        fence_barrier_init();
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

    if (warp == W_PX || warp == W_PY) {
        // ------------------------------------------------------------ producers
        const bool px = warp == W_PX;
        int armed0 = 0, armed1 = 0;   // copies issued on each stage's barrier
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, s = i & 1;
            const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
            if (i >= 2) {
                const bool ok = wait_or_abort(&bars[FREE0 + s], ((i >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (lane == 0) {
                uint64_t *full = &bars[FULL0 + s];
                if (px) {   // -W and Khat of both 64-column blocks, F (and a pair's Y)
                    const bool with_y = pair && s == 1;
                    mbar_arrive_expect_tx(full, (with_y ? 5u : 4u) * prep::IMG + KD * 4);
                    if (with_y)
                        bulk_load(base + Ly.y, fac - args.rec_bytes + args.pair_y, prep::IMG, full);
                    uint8_t *wk = base + stage(Ly.wk, s);
                    for (int kb = 0; kb < KD / 64; ++kb) {
                        bulk_load(wk + kb * 128 * 128, fac + prep::REC_W + kb * prep::IMG, prep::IMG, full);
                        bulk_load(wk + kb * 128 * 128 + 64 * 128, fac + prep::EXT_KH + kb * prep::IMG,
                                  prep::IMG, full);
                    }
                    bulk_load(fgate(s), fac + prep::EXT_F, KD * 4, full);
                } else {    // T, then V
                    mbar_arrive_expect_tx(full, prep::IMG + CC * NV * 2);
                    uint8_t *tv = base + stage(Ly.tv, s);
                    const long c0 = (long)c * CC;
                    bulk_load(tv, fac, prep::IMG, full);
                    tma_load_3d(tv + prep::IMG, &tm_v, full, n0, (int)c0, (int)vh);
                    tma_load_3d(tv + prep::IMG + 64 * 128, &tm_v, full, n0 + 64, (int)c0, (int)vh);
                }
            }
            armed0 += s == 0;
            armed1 += s == 1;
        }
        if (lane == 0)   // no copy may still be in flight when the CTA exits
            for (int s = 0; s < 2; ++s)
                if ((s == 0 ? armed0 : armed1) > 0)
                    mbar_wait(&bars[FULL0 + s], ((s == 0 ? armed0 : armed1) - 1) & 1, 200000000ull);
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id64 = idesc_bf16(64, NV, false, true);
            const uint32_t id_s = idesc_bf16(KD, NV, true, true);
            auto kstep = [](int k0) {   // K-major A of 128 rows, 64-column blocks
                return static_cast<uint64_t>(((k0 >> 6) * 128 * 128 + (k0 & 63) * 2) >> 4);
            };
            auto mstep = [](int k0) { return static_cast<uint64_t>(k0 * 8); };
            // per chain x (arithmetic, so that nothing lives in local memory)
            const uint32_t dSE = Ly.S[1] - Ly.S[0];
            auto d_s = [&](int x) { return desc_mnmajor(base_u32 + Ly.S[0] + x * dSE, KD, 0, 0); };
            auto d_e = [&](int x) { return desc_mnmajor(base_u32 + Ly.E[0] + x * dSE, CC, 0, 0); };
            auto tr = [&](int x) { return tmem + T_RA + (T_RB - T_RA) * x; };
            auto ts = [&](int x) { return tmem + T_SA + (T_SB - T_SA) * x; };
            const int nch = dual ? 2 : 1;
            bool ok = true;
            for (int i = 0; i < nloc && ok; ++i) {
                const int s = i & 1;
                const uint32_t par = i & 1;
                const uint32_t wk = base_u32 + stage(Ly.wk, s), tv = base_u32 + stage(Ly.tv, s);
                if (!(ok = wait_or_abort(&bars[FULL0 + s], (i >> 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                // U = [T; *] V into R_A (E_A of the previous chunk has been read)
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tr(0), desc_kmajor(tv, 64, 0, k0), desc_mnmajor(tv + prep::IMG, 64, k0, 0),
                             id64, k0 > 0);
                // -W S: E = U - W S (value chain), -W S (transition)
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (x >= nch || !ok)
                        break;
                    if (!(ok = wait_or_abort(&bars[S_READY_A + x], par, abort_flag)))
                        break;
                    tc_fence_after();
                    for (int k0 = 0; k0 < KD; k0 += 16)
                        mma_bf16(tr(x), desc_kmajor(wk, 128, 0, 0) + kstep(k0), d_s(x) + mstep(k0), id64,
                                 (x == 0 || k0 > 0) ? 1u : 0u);
                    if (pair && s == 1)   // second half: + Y E1
                        for (int k0 = 0; k0 < CC; k0 += 16)
                            mma_bf16(tr(x), desc_kmajor(base_u32 + Ly.y, 128, 0, k0), d_e(x) + mstep(k0),
                                     id64, 1u);
                    mma_commit(&bars[P_FULL_A + x]);
                }
                // S <- F S + Khat^T E
                const uint64_t kt = desc_mnmajor(wk, 128, 64, 0);
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (x >= nch || !ok)
                        break;
                    if (!(ok = wait_or_abort(&bars[E_READY_A + x], par, abort_flag)))
                        break;
                    tc_fence_after();
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(ts(x), kt + mstep(k0), d_e(x) + mstep(k0), id_s, 1u);
                    mma_commit(&bars[UPD_A + x]);
                }
                mma_commit(&bars[FREE0 + s]);
            }
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, 200000000ull);
        }
    } else if (warp >= W_STATE0) {
        // ------------------------------------------------------------ state chains
        const int stid = tid - W_STATE0 * 32;
        const int R = 32 * (warp & 3) + lane;            // S row (key channel), E row if < 64
        const int cs = 32 * ((warp - W_STATE0) >> 2);    // this thread's 32 of the 128 columns
        const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        const uint32_t dSE = Ly.S[1] - Ly.S[0];
        auto tr = [&](int x) { return tq + T_RA + (T_RB - T_RA) * x + cs; };
        auto ts = [&](int x) { return tq + T_SA + (T_SB - T_SA) * x + cs; };
        auto S_T = [&](int x) { return base_u32 + Ly.S[0] + x * dSE; };
        auto E_T = [&](int x) { return base_u32 + Ly.E[0] + x * dSE; };
        const int nch = dual ? 2 : 1;
        // chain A from zero; chain B from the identity
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            if (x >= nch)
                break;
            float sv[32];
#pragma unroll
            for (int n = 0; n < 32; ++n)
                sv[n] = (x == 1 && R == cs + n) ? 1.f : 0.f;
            tmem_st16(ts(x), *reinterpret_cast<const float(*)[16]>(&sv[0]));
            tmem_st16(ts(x) + 16, *reinterpret_cast<const float(*)[16]>(&sv[16]));
        }
        tmem_st_wait();
        bool ok = true;
        for (int i = 0; i < nloc && ok; ++i) {
            const int s = i & 1;
            const uint32_t par = i & 1;
            // S phases: S_{c-1} -> bf16 operand, then F S_{c-1} back (the update accumulates onto it)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                if (x >= nch)
                    break;
                if (i >= 1 && named_vote_or(NB_STATE, N_STATE,
                                            !wait_or_abort(&bars[UPD_A + x], par ^ 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float sv[32];
                tmem_ld16(ts(x), *reinterpret_cast<float(*)[16]>(&sv[0]));
                tmem_ld16(ts(x) + 16, *reinterpret_cast<float(*)[16]>(&sv[16]));
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 32; n += 8)
                    st_tile8(S_T(x), KD, R, cs + n, &sv[n]);
                fence_proxy_async_smem();
                tc_fence_before();
                named_sync(NB_STATE, N_STATE);
                if (stid == 0)
                    mbar_arrive(&bars[S_READY_A + x]);
                if (x == 0 && named_vote_or(NB_STATE, N_STATE,
                                            !wait_or_abort(&bars[FULL0 + s], (i >> 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                const float F = fgate(s)[R];
#pragma unroll
                for (int n = 0; n < 32; ++n)
                    sv[n] *= F;
                tmem_st16(ts(x), *reinterpret_cast<const float(*)[16]>(&sv[0]));
                tmem_st16(ts(x) + 16, *reinterpret_cast<const float(*)[16]>(&sv[16]));
            }
            if (!ok)
                break;
            // E phases: E from R -> bf16 operand of the update
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                if (x >= nch)
                    break;
                if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[P_FULL_A + x], par, abort_flag))) {
                    ok = false;
                    break;
                }
                if (x == 0 && stid == 0)   // every state thread has read F (the vote above)
                    mbar_arrive(&bars[FREE0 + s]);
                tc_fence_after();
                {   // E row t = 16 (w % 4) + lane in lanes 0-15 (M = 64 accumulator)
                    float ev[32];
                    tmem_ld16(tr(x), *reinterpret_cast<float(*)[16]>(&ev[0]));
                    tmem_ld16(tr(x) + 16, *reinterpret_cast<float(*)[16]>(&ev[16]));
                    tmem_ld_wait();
                    if (lane < 16) {
                        const int t = 16 * (warp & 3) + lane;
#pragma unroll
                        for (int n = 0; n < 32; n += 8)
                            st_tile8(E_T(x), CC, t, cs + n, &ev[n]);
                    }
                }
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                named_sync(NB_STATE, N_STATE);
                if (stid == 0)
                    mbar_arrive(&bars[E_READY_A + x]);
            }
        }
        tmem_st_wait();
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            if (x >= nch)
                break;
            if (ok && nloc > 0 &&
                named_vote_or(NB_STATE, N_STATE,
                              !wait_or_abort(&bars[UPD_A + x], (nloc - 1) & 1, abort_flag)))
                ok = false;
            if (!ok)
                break;
            tc_fence_after();
            float *dst = x == 0 ? args.seg_end + (((size_t)vh * args.nseg + seg) * KD + R) * p.dv + n0 + cs
                                : args.seg_trans + (((size_t)kh * args.nseg + seg) * KD + R) * KD + cs;
            float sv[32];
            tmem_ld16(ts(x), *reinterpret_cast<float(*)[16]>(&sv[0]));
            tmem_ld16(ts(x) + 16, *reinterpret_cast<float(*)[16]>(&sv[16]));
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 32; n += 4)
                *reinterpret_cast<float4 *>(dst + n) = make_float4(sv[n], sv[n + 1], sv[n + 2], sv[n + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace ab
}  // namespace split
