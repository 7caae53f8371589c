// gdr_tc_split128.cuh -- the state pass with 128 value columns per CTA, for
// few long sequences (the segment-parallel form).  Included by gdr_tc.cu after
// gdr_tc_split.cuh and gdr_tc_ab128.cuh: this kernel runs the whole sequence
// (MODE_SEQ) or each segment from its start state with outputs (MODE_SEG_C); the
// segments' end states and transitions (MODE_SEG_AB) come from ab128_kernel.
//
// The same chunk recurrence as split_kernel ("Systolic Linear Attention:
// Co-Designing Tile-Grouped Gated Delta Attention for TPUs", §2.1, §2.3 Table 2,
// §2.4.2), E = T V - W S, S <- F S + Khat^T E, O = Qbar S + L E, arranged for
// fewer, wider chain steps:
//   * one CTA holds 128 value columns (a whole dv = 128 head), so every product
//     has N = 128: an
//     N = 64 product reads as many operand bytes from shared memory per output
//     column as it computes, N = 128 half as many;
//   * U, P, E and O share one fp32 tensor-memory buffer R (two, alternating by
//     chunk): [0; T] V writes U into rows 64-127 (zeros into 0-63), the first pass
//     stores W negated so that [Qbar; -W] S accumulates Qbar S into rows 0-63 and
//     U - W S = E into rows 64-127 with no subtraction, and after the update
//     [L; 0] E accumulates L E into rows 0-63, leaving O there;
//   * [L | 0 | T] is one 192-row tile whose middle block of zeros serves both
//     [L; 0] and [0; T].
// Tensor memory: R 2 x 128 columns, S 128 columns.  Grouped / per-channel gates
// (records carry Qbar and Khat), dk = 128, dv a multiple of 128; the pair
// correction of the chunk-128 Neumann inverses is not implemented here.
//
// Roles: warps 0-1 epilogue (O rows in lanes 0-63), warps 2 and 12 producers,
// warp 3 MMA issuer, warps 4-11 state chain (S in all 128 lanes; E in lanes
// 64-127, i.e. warps 6, 7, 10, 11).

namespace split {

constexpr int NVC2 = 128;                 // value columns per CTA
constexpr uint32_t T_R = 0;               // two buffers of 128 columns
constexpr uint32_t T_S2 = 256;            // fp32 state, 128 columns
constexpr uint32_t T_X = 384;             // pairs: Y E1 of the first half (rows 64-127)

struct Plan128 {
    uint32_t qwk[2], lzt[2], v[2], gates[2];
    uint32_t S, E, bar, misc, total;
};

// Stage: [Qbar | -W | Khat] (rows 0-63 | 64-127 | 128-191, 128 columns), [L | 0 | T]
// (3 x 64 rows, 64 columns), V (64 rows, 128 columns), F (128 fp32).  Pairs: stage 0
// (first halves) appends the pair's Y under T ([L | 0 | T | Y]) and V has one buffer
// (the 16 KB that pays for Y), refilled as soon as the chunk's U product is done.
__host__ __device__ inline Plan128 plan128(bool pair = false)
{
    Plan128 s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    for (int i = 0; i < 2; ++i) {
        s.qwk[i] = take((KD / 64) * 192 * 128);
        s.lzt[i] = take(((pair && i == 0) ? 256 : 192) * 128);
        s.v[i] = (pair && i == 1) ? s.v[0] : take(2 * 64 * 128);
    }
    s.S = take(KD * NVC2 * 2);
    s.E = take(CC * NVC2 * 2);
    // factors of both stages and the barriers share one kilobyte
    s.gates[0] = take(2 * KD * 4 + NBARS * 8 + 16);
    s.gates[1] = s.gates[0] + KD * 4;
    s.bar = s.gates[0] + 2 * KD * 4;
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(NTHR, 1)
split128_kernel(const __grid_constant__ CUtensorMap tm_v, const SplitArgs args)
{
    using namespace ptx;
    using ws::named_sync;
    using ws::named_vote_or;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const bool pair = args.pair != 0;
    const Plan128 Ly = plan128(pair);
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = (int)blockIdx.x % args.nvt;
    const int hv = (int)blockIdx.x / args.nvt;
    const int b = blockIdx.y;
    const int hk = hv / p.R;
    const int n0 = nt * NVC2;
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int T = p.T;
    const int N = args.nchunks;
    const int seg = blockIdx.z;
    const int cbeg = seg * args.seg_len;
    const int nloc = min(args.seg_len, N - cbeg);

    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 4);
    auto fgate = [&](int s) { return reinterpret_cast<float *>(base + stage(Ly.gates, s)); };
    const uint32_t S_T = base_u32 + Ly.S, E_T = base_u32 + Ly.E;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)   // FREEX: the MMAs' commit and the state warps
            mbar_init(&bars[i], (i == FREEX0 || i == FREEX1) ? 2 : 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    // the zero block of [L | 0 | T] (never loaded)
    for (int i = tid; i < 2 * 64 * 8; i += NTHR) {
        const int st = i >> 9, r = (i >> 3) & 63, c = (i & 7) * 8;
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        st_tile8(base_u32 + stage(Ly.lzt, st), 192, 64 + r, c, z);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int R = 32 * (warp & 3) + lane;     // TMEM lane of this thread

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer: X group
        // [Qbar; -W] (Qbar only where o is written) and F; warp 12 adds T and V
        int narmx = 0;   // group X loads armed (both stages)
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, s = i & 1;
            const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
            uint8_t *qwk = base + stage(Ly.qwk, s);
            if (i >= 2) {
                const bool ok = wait_or_abort(&bars[FREEX0 + s], ((i >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (lane == 0) {
                uint64_t *full = &bars[FULLX0 + s];
                mbar_arrive_expect_tx(full, 5u * prep::IMG + CC * NVC2 * 2 + KD * 4);
                for (int kb = 0; kb < KD / 64; ++kb) {
                    uint8_t *blk = qwk + kb * 192 * 128;
                    bulk_load(blk + 64 * 128, fac + prep::REC_W + kb * prep::IMG, prep::IMG, full);
                    bulk_load(blk, fac + prep::EXT_QB + kb * prep::IMG, prep::IMG, full);
                }
                bulk_load(fgate(s), fac + prep::EXT_F, KD * 4, full);
            }
            ++narmx;
        }
        if (lane == 0) {
            for (int s = 0; s < 2; ++s)
                if ((narmx + 1 - s) / 2 > 0)   // loads armed on stage s
                    mbar_wait(&bars[FULLX0 + s], ((narmx + 1 - s) / 2 - 1) & 1, 200000000ull);
        }
    } else if (warp == W_PROD_Y) {
        // ------------------------------------------------------------ producer: T, V; Y group
        int narmy = 0;   // group Y loads armed (both stages)
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, s = i & 1;
            const long c0 = (long)c * CC;
            const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
            uint8_t *qwk = base + stage(Ly.qwk, s);
            uint8_t *lzt = base + stage(Ly.lzt, s);
            if (i >= 2) {
                const bool ok = wait_or_abort(&bars[FREEX0 + s], ((i >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (pair && i >= 1) {   // one V buffer: the previous chunk's U product has read it
                const bool ok = wait_or_abort(&bars[VFREE], (i - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (lane == 0) {
                uint64_t *full = &bars[FULLX0 + s];
                bulk_load(lzt + 128 * 128, fac, prep::IMG, full);   // T under the zeros
                tma_load_3d(base + stage(Ly.v, s), &tm_v, full, n0, (int)c0, (int)vh);
                tma_load_3d(base + stage(Ly.v, s) + 64 * 128, &tm_v, full, n0 + 64, (int)c0, (int)vh);
            }
            if (i >= 2) {
                const bool ok = wait_or_abort(&bars[FREEY0 + s], ((i >> 1) - 1) & 1, abort_flag);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (lane == 0) {
                // pairs: a first half (stage 0: segments start at even chunks) brings the
                // pair's Y under its T
                const bool with_y = pair && s == 0;
                uint64_t *full = &bars[FULLY0 + s];
                mbar_arrive_expect_tx(full, (with_y ? 4u : 3u) * prep::IMG);
                for (int kb = 0; kb < KD / 64; ++kb)
                    bulk_load(qwk + kb * 192 * 128 + 128 * 128, fac + prep::EXT_KH + kb * prep::IMG,
                              prep::IMG, full);
                bulk_load(lzt, fac + prep::IMG, prep::IMG, full);   // L above the zeros
                if (with_y)
                    bulk_load(lzt + 192 * 128, fac + args.pair_y, prep::IMG, full);
            }
            ++narmy;
        }
        if (lane == 0) {
            for (int s = 0; s < 2; ++s)
                if ((narmy + 1 - s) / 2 > 0)   // loads armed on stage s
                    mbar_wait(&bars[FULLY0 + s], ((narmy + 1 - s) / 2 - 1) & 1, 200000000ull);
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id128 = idesc_bf16(128, NVC2, false, true);
            const uint32_t id_s = idesc_bf16(KD, NVC2, true, true);
            auto kstep = [](int k0, int rows) {
                return static_cast<uint64_t>(((k0 >> 6) * rows * 128 + (k0 & 63) * 2) >> 4);
            };
            auto mstep = [](int k0) { return static_cast<uint64_t>(k0 * 8); };
            const uint64_t d_s = desc_mnmajor(S_T, KD, 0, 0);
            const uint64_t d_e = desc_mnmajor(E_T, CC, 0, 0);
            bool ok = true;
            for (int i = 0; i < nloc && ok; ++i) {
                const int s = i & 1;
                const uint32_t par = i & 1;
                const uint32_t qwk = base_u32 + stage(Ly.qwk, s), lzt = base_u32 + stage(Ly.lzt, s);
                const uint32_t rb = tmem + T_R + 128 * s;
                if (!(ok = wait_or_abort(&bars[FULLX0 + s], (i >> 1) & 1, abort_flag)))
                    break;
                // R(s) was last read by the epilogue for chunk i - 2
                if (i >= 2 && !(ok = wait_or_abort(&bars[OFREE0 + s], ((i >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                // U = [0; T] V into rows 64-127 of R(s), zeros into 0-63
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(rb, desc_kmajor(lzt + 64 * 128, 128, 0, k0),
                             desc_mnmajor(base_u32 + stage(Ly.v, s), 64, k0, 0), id128, k0 > 0);
                if (pair)
                    mma_commit(&bars[VFREE]);
                if (!(ok = wait_or_abort(&bars[S_READY], par, abort_flag)))
                    break;
                tc_fence_after();
                // [Qbar; -W] S: Qbar S into rows 0-63, U - W S = E into rows 64-127
                for (int k0 = 0; k0 < KD; k0 += 16)
                    mma_bf16(rb, desc_kmajor(qwk, 192, 0, 0) + kstep(k0, 192), d_s + mstep(k0), id128, 1u);
                mma_commit(&bars[P_FULL]);
                if (!pair)   // (pairs: T also feeds the first half's Y product below)
                    mma_commit(&bars[FREEX0 + s]);
                if (!(ok = wait_or_abort(&bars[E_READY], par, abort_flag)))
                    break;
                if (!(ok = wait_or_abort(&bars[FULLY0 + s], (i >> 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint64_t kt = desc_mnmajor(qwk, 192, 128, 0);
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_S2, kt + mstep(k0), d_e + mstep(k0), id_s, 1u);
                mma_commit(&bars[UPD_DONE]);
                // [L; 0] E onto R(s): O = Qbar S + L E in rows 0-63 (rows 64-127 unchanged)
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(rb, desc_kmajor(lzt, 128, 0, k0), d_e + mstep(k0), id128, 1u);
                if (pair && s == 0)   // [T; Y] E1: Y E1 into rows 64-127 of X for the second half
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_X, desc_kmajor(lzt + 128 * 128, 128, 0, k0), d_e + mstep(k0),
                                 id128, k0 > 0);
                if (pair)
                    mma_commit(&bars[FREEX0 + s]);
                mma_commit(&bars[OUT0 + s]);
                mma_commit(&bars[FREEY0 + s]);
            }
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, 200000000ull);
        }
    } else if (warp >= W_STATE0) {
        // ------------------------------------------------------------ state chain
        const int stid = tid - W_STATE0 * 32;
        const int cs = 64 * ((warp - W_STATE0) >> 2);   // this lane's 64 of the 128 columns
        {
            float sv[64];
#pragma unroll
            for (int n = 0; n < 64; ++n)
                sv[n] = 0.f;
            const float *src = nullptr;
            if (args.mode == MODE_SEQ && p.S0 != nullptr)
                src = p.S0 + (vh * KD + R) * p.dv + n0 + cs;
            else if (args.mode == MODE_SEG_C)
                src = args.seg_start + (((size_t)vh * args.nseg + seg) * KD + R) * p.dv + n0 + cs;
            if (src != nullptr)
#pragma unroll
                for (int n = 0; n < 64; n += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(src + n);
                    sv[n] = a4.x; sv[n + 1] = a4.y; sv[n + 2] = a4.z; sv[n + 3] = a4.w;
                }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_st16(tq + T_S2 + cs + 16 * q, *reinterpret_cast<const float(*)[16]>(&sv[16 * q]));
        }
        tmem_st_wait();
        bool ok = true;
        for (int i = 0; i < nloc; ++i) {
            const int s = i & 1;
            const uint32_t par = i & 1;
            if (i >= 1 &&
                named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[UPD_DONE], (i - 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // S_{c-1} -> bf16 operand, then F S_{c-1} back (the update accumulates onto it)
            float sv[64];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_ld16(tq + T_S2 + cs + 16 * q, *reinterpret_cast<float(*)[16]>(&sv[16 * q]));
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 64; n += 8)
                st_tile8(S_T, KD, R, cs + n, &sv[n]);
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[S_READY]);
            if (named_vote_or(NB_STATE, N_STATE,
                              !wait_or_abort(&bars[FULLX0 + s], (i >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            {
                const float F = fgate(s)[R];
#pragma unroll
                for (int n = 0; n < 64; ++n)
                    sv[n] *= F;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_st16(tq + T_S2 + cs + 16 * q, *reinterpret_cast<const float(*)[16]>(&sv[16 * q]));
            }
            if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[P_FULL], par, abort_flag))) {
                ok = false;
                break;
            }
            if (stid == 0)   // every state thread has read its factor (the vote above)
                mbar_arrive(&bars[FREEX0 + s]);
            tc_fence_after();
            if (R >= CC && pair && s == 1) {   // second half of a pair: E2 + Y E1 (X, same lanes)
                const int t = R - CC;
#pragma unroll
                for (int h = 0; h < 64; h += 32) {
                    float ev[32], xv[32];
                    tmem_ld16(tq + T_R + 128 * s + cs + h, *reinterpret_cast<float(*)[16]>(&ev[0]));
                    tmem_ld16(tq + T_R + 128 * s + cs + h + 16, *reinterpret_cast<float(*)[16]>(&ev[16]));
                    tmem_ld16(tq + T_X + cs + h, *reinterpret_cast<float(*)[16]>(&xv[0]));
                    tmem_ld16(tq + T_X + cs + h + 16, *reinterpret_cast<float(*)[16]>(&xv[16]));
                    tmem_ld_wait();
#pragma unroll
                    for (int n = 0; n < 32; ++n)
                        ev[n] += xv[n];
#pragma unroll
                    for (int n = 0; n < 32; n += 8)
                        st_tile8(E_T, CC, t, cs + h + n, &ev[n]);
                }
            } else if (R >= CC) {   // lanes 64-127: E of token t = R - 64, straight from R(s)
                const int t = R - CC;
                float ev[64];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld16(tq + T_R + 128 * s + cs + 16 * q, *reinterpret_cast<float(*)[16]>(&ev[16 * q]));
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 64; n += 8)
                    st_tile8(E_T, CC, t, cs + n, &ev[n]);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[E_READY]);
        }
        tmem_st_wait();
        if (ok && nloc > 0 &&
            named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[UPD_DONE], (nloc - 1) & 1, abort_flag)))
            ok = false;
        float *dst = nullptr;
        if (p.S_final != nullptr && seg == args.nseg - 1)
            dst = p.S_final + (vh * KD + R) * p.dv + n0 + cs;
        if (ok && dst != nullptr) {
            tc_fence_after();
            float sv[64];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_ld16(tq + T_S2 + cs + 16 * q, *reinterpret_cast<float(*)[16]>(&sv[16 * q]));
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 64; n += 4)
                *reinterpret_cast<float4 *>(dst + n) = make_float4(sv[n], sv[n + 1], sv[n + 2], sv[n + 3]);
        }
    } else {
        // ------------------------------------------------------------ epilogue (rows t in lanes 0-63)
        const int etid = tid - W_EPI0 * 32;
        const int t = R;
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, ob = i & 1;
            const long c0 = (long)c * CC;
            const int Cl = (int)min((long)CC, T - c0);
            if (named_vote_or(NB_EPI, N_EPI, !wait_or_abort(&bars[OUT0 + ob], (i >> 1) & 1, abort_flag)))
                break;
            tc_fence_after();
            const bool live = t < Cl;
            const long orow = (vh * T + c0 + t) * p.dv + n0;
            // 64 columns per tensor-memory wait: the epilogue must finish within about one
            // chunk period, or the next chunk but one waits for its buffer
#pragma unroll
            for (int half = 0; half < NVC2; half += 64) {
                float ov[64];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld16(tq + T_R + 128 * ob + half + 16 * q, *reinterpret_cast<float(*)[16]>(&ov[16 * q]));
                tmem_ld_wait();
                if (live) {
#pragma unroll
                    for (int cb = 0; cb < 64; cb += 16) {
                        const float *v = &ov[cb];
                        if constexpr (OUT_BF16) {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow + half + cb);
                            dst[0] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
                            dst[1] = make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]),
                                                pack_bf16(v[12], v[13]), pack_bf16(v[14], v[15]));
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow + half + cb);
#pragma unroll
                            for (int n = 0; n < 4; ++n)
                                dst[n] = make_float4(v[4 * n], v[4 * n + 1], v[4 * n + 2], v[4 * n + 3]);
                        }
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

// The 128-column state pass serves grouped / per-channel gates at dk = 128 when the
// sequences are few and long enough to run segment-parallel.
inline bool supports128(const Params &p)
{
    return supports(p) && p.dk == KD && p.G > 1 && p.dv % NVC2 == 0 && !p.momentum;
}

// Segment plan of the 128-column pass (one CTA per head and 128 value columns in
// both launches, the transitions riding with the first value tile of each key
// head); its chain step does twice the columns of the 64-column pass's for about
// 1.3 times its time.
inline SegPlan seg_plan128(const Params &p)
{
    const int N = prep::nchunks(p);
    const long nvh = (long)(p.dv / NVC2) * p.Hv * p.B;
    auto waves = [](long ctas) { return (ctas + kSMs - 1) / kSMs; };
    const int even = p.pair ? 2 : 1;   // pairs never straddle a segment boundary
    SegPlan best{1, N};
    long best_cost = waves(nvh) * (long)N;
    for (int ns = 2; ns <= N / kMinSegChunks; ++ns) {
        const int L = ((N + ns - 1) / ns + even - 1) / even * even;
        const int nsg = (N + L - 1) / L;
        const long cost = 2 * waves(nvh * nsg) * (long)L + nsg;
        if (cost < best_cost) {
            best_cost = cost;
            best = SegPlan{nsg, L};
        }
    }
    return best;
}

// Use it when both plans are segment-parallel and its cost (scaled by the wider
// step's time) is the lower.
inline bool use128(const Params &p)
{
    if (!supports128(p))
        return false;
    if (p.wide_state)
        return true;
    const SegPlan a = seg_plan(p), w = seg_plan128(p);
    if (a.nseg == 1 || w.nseg == 1)
        return false;
    auto waves = [](long ctas) { return (ctas + kSMs - 1) / kSMs; };
    const long nvh = (long)(p.dv / NVC) * p.Hv * p.B, ntr = (long)(KD / NVC) * p.Hk * p.B;
    const long nvh2 = (long)(p.dv / NVC2) * p.Hv * p.B;
    const long ca = (waves((nvh + ntr) * a.nseg) + waves(nvh * a.nseg)) * (long)a.seg_len * 10;
    const long cw = 2 * waves(nvh2 * w.nseg) * (long)w.seg_len * 13;
    return cw < ca;
}

template <bool OB>
int launch128(const Params &p, const void *factors, cudaStream_t stream)
{
    CUtensorMap mv;
    if (!make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CC))
        return 6;
    const Plan128 Ly = plan128(p.pair != 0);
    auto kern = split128_kernel<OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    SplitArgs a;
    a.p = p;
    a.factors = static_cast<const uint8_t *>(factors);
    a.rec_bytes = prep::rec_bytes(p);
    a.nvt = p.dv / NVC2;
    a.nchunks = prep::nchunks(p);
    const SegPlan sp = seg_plan128(p);
    a.nseg = sp.nseg;
    a.seg_len = sp.seg_len;
    a.pair = p.pair;
    a.pair_y = prep::kind_bytes(prep::record_kind(p), p.dk) + prep::PAIR_Y;
    a.seg_end = a.seg_trans = a.seg_start = nullptr;
    if (sp.nseg == 1) {   // one segment: the whole sequence from S0, with outputs
        a.mode = MODE_SEQ;
        kern<<<dim3(a.nvt * p.Hv, p.B, 1), NTHR, Ly.total, stream>>>(mv, a);
        return cudaGetLastError() == cudaSuccess ? 0 : 6;
    }
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    uint8_t *w = static_cast<uint8_t *>(const_cast<void *>(factors)) + al(prep::ws_bytes(p));
    const size_t per_v = al((size_t)p.B * p.Hv * sp.nseg * KD * p.dv * 4);
    a.seg_end = reinterpret_cast<float *>(w);
    a.seg_start = reinterpret_cast<float *>(w + per_v);
    a.seg_trans = reinterpret_cast<float *>(w + 2 * per_v);
    if (cudaFuncSetAttribute(seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)CMB_SMEM) != cudaSuccess)
        return 6;
    const ab::Plan La = ab::plan(p.pair != 0);
    if (cudaFuncSetAttribute(ab::ab128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)La.total) != cudaSuccess)
        return 6;
    a.mode = MODE_SEG_AB;
    ab::ab128_kernel<<<dim3(a.nvt * p.Hv, p.B, sp.nseg), ab::NTHR, La.total, stream>>>(mv, a);
    seg_combine_kernel<<<dim3((p.dv / CMB_COLS) * p.Hv, p.B), CMB_THREADS, CMB_SMEM, stream>>>(a);
    a.mode = MODE_SEG_C;
    kern<<<dim3(a.nvt * p.Hv, p.B, sp.nseg), NTHR, Ly.total, stream>>>(mv, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

// The segment plan and the segment buffers of the state pass a request runs.
inline SegPlan state_seg_plan(const Params &p) { return use128(p) ? seg_plan128(p) : seg_plan(p); }

inline size_t state_seg_bytes(const Params &p)
{
    const SegPlan sp = state_seg_plan(p);
    if (sp.nseg == 1)
        return 0;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t per_v = (size_t)p.B * p.Hv * sp.nseg * KD * p.dv * 4;
    return 2 * al(per_v) + al((size_t)p.B * p.Hk * sp.nseg * KD * KD * 4);
}

}  // namespace split
