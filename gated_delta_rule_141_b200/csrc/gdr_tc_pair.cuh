// gdr_tc_pair.cuh -- the truncated Neumann inverse at chunk 2C = 128 on the
// two-pass path, with the state pass stepping by C = 64.  Included by gdr_tc.cu.
//
// "When Good Enough Is Optimal: Multiplication-Only Matrix Inversion
// Approximation for Quantized Gated DeltaNet" (§4.1, Lemma 3.1) truncates the
// Neumann series of (I + M)^{-1} for a whole chunk; the result depends on the
// chunk length, so a 128-token request cannot simply be blocked by 64 as the
// exact inverse can.  Split the chunk into halves 1 and 2.  With G the chunk's
// decayed Gram (G_tj = sum_i k_ti k_ji e^{Lambda_ti - Lambda_ji}, t > j),
// M = G diag(beta), A the truncated series with its Newton steps and
// T = diag(beta) A, the blocks of powers and products of block-lower-triangular
// matrices are the products of their blocks, so T11 and T22 are exactly the
// 64-token factors of each half (what the first pass writes).  Only T21 is
// unseen by a state pass that steps half by half.  Stepping half 2 from the
// state at the half boundary gives
//   E2' = T22 (V2 - Kbar2 S) - T22 G21 E1,
// while the 128-token chunk has E2 = T21 (V1 - Kbar1 S) + T22 (V2 - Kbar2 S),
// with S the pair's start state and E1 = T11 (V1 - Kbar1 S) the first half's E.
// In the similar form Atil = diag(beta) A diag(beta)^{-1} (the same series of
// Ntil = diag(beta) G, beta on the rows; unit lower triangular),
// T21 = Atil21 diag(beta1) and T11 = Atil11 diag(beta1), hence
//   E2 = E2' + Y E1,   Y = Atil21 Atil11^{-1} + Atil22 Ntil21,
// and the half's output and state update follow from that E2 unchanged.  (For
// the exact inverse Y = 0: that is why exact requests at 128 run by 64.)
//
// pair_kernel, one CTA (256 threads) per (batch, key head, pair of halves):
//   1. bulk copies of Ntil11, Ntil22 (first-pass images) and the operands of
//      G21 = Kbar2' Khat1^T (Kbar2' = k2 e^{Lambda_t - Lambda_mid},
//      Khat1 = k1 e^{Lambda_mid - Lambda_j}: both <= 1, no pivot needed);
//   2. G21 on tcgen05, Ntil21 = diag(beta2) G21 into the 128 x 128 Ntil tile;
//   3. Atil by Horner's rule (X <- I - Ntil X, m times) and r Newton steps
//      (X <- X + X (I - X - Ntil X)), all products M = N = K = 128 on tcgen05,
//      X kept in fp32 in tensor memory and as a bf16 operand in shared memory;
//   4. Atil11^{-1} exactly in fp32 (block doubling), then Y on tcgen05 from split
//      bf16 operands (hi + lo parts: fp32-level products, which the cancellation
//      between Y's two terms needs); (the 1-Step Neumann inverse of §2.4.3 instead
//      of 3: Atil from the diagonal 16 x 16 blocks in fp32, Y the same way;)
//   5. Y as a bf16 image into the first half's record.
// The state passes add Y E1 to the second half's E: the 64-column pass through an
// [L; Y] tile whose E product of the first half leaves Y E1 in tensor memory, the
// 128-column passes through their own products with Y.

namespace pair {

constexpr int NT = 256;
constexpr int CC = 64;
constexpr int LDM = gen::LDM;
constexpr uint32_t TMEM_COLS = 256;   // product (128 columns), X in fp32 (128 columns)
constexpr uint32_t T_D = 0, T_X = 128;

struct Plan {
    uint32_t NTL, XT, RT, Tf, beta, bar, misc, total;
};

template <int DK>
__host__ __device__ inline Plan plan()
{
    Plan s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    s.NTL = take(2 * 128 * 128);        // Ntil, 128 x 128 bf16
    s.XT = take(2 * 128 * 128);         // X, 128 x 128 bf16
    // Newton residual; first the G21 operands (two 64 x dk tiles)
    s.RT = take(2 * 128 * 128 > 2 * CC * DK * 2 ? 2 * 128 * 128 : 2 * CC * DK * 2);
    s.Tf = take(32 * 36 * 4 + 1024);    // scratch of the fp32 block inverse
    s.beta = take(4 * CC * 4);          // beta2, then (scalar gate) ea2, eb1, then beta1
    s.bar = take(64);
    s.misc = s.bar + 32;
    s.total = o + 1024;
    return s;
}

struct PairArgs {
    Params p;                 // the request at the half length (C = 64, pair = 1)
    uint8_t *rec;             // the first pass's records, [B * Hk * nchunks][rec_bytes]
    int nchunks;              // halves per sequence
    uint32_t rec_bytes;
    uint32_t base_bytes;      // offset of the pair extras in a record
    int ext;                  // grouped / per-channel records (else the scalar gate's)
    int defer_tw;             // the first pass left the halves' T and W to this kernel
    int neg_w;                // ... and the state pass reads -W
};

// fp32 views of the regions freed once the series is done (stride LDM)
__device__ __forceinline__ float *f32(uint8_t *base, uint32_t off) { return reinterpret_cast<float *>(base + off); }

template <int DK>
__global__ void __launch_bounds__(NT, 2)
pair_kernel(const __grid_constant__ CUtensorMap tm_k, const PairArgs a)
{
    using namespace ptx;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = a.p;
    const Plan Ly = plan<DK>();
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));
    const uint32_t NTL = base_u32 + Ly.NTL, XT = base_u32 + Ly.XT, RT = base_u32 + Ly.RT;
    float *Tf = f32(base, Ly.Tf);
    float *sbeta = f32(base, Ly.beta);          // beta of half 2
    float *ea2 = sbeta + CC, *eb1 = sbeta + 2 * CC, *beta1 = sbeta + 3 * CC;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pr = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const long kh = (long)b * p.Hk + hk;
    const int c1 = 2 * pr, c2 = c1 + 1;
    const int T = p.T;
    uint8_t *rec1 = a.rec + (size_t)(kh * a.nchunks + c1) * a.rec_bytes;
    uint8_t *img_Y = rec1 + a.base_bytes + prep::PAIR_Y;

    // no second half (odd number of halves): nothing follows, Y = 0
    if (c2 >= a.nchunks) {
        for (int u = tid; u < CC * 8; u += NT)
            reinterpret_cast<uint4 *>(img_Y)[u] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    const uint8_t *rec2 = rec1 + a.rec_bytes;
    const long c0_2 = (long)c2 * CC;
    const int Cl2 = (int)min((long)CC, T - c0_2);

    if (tid == 0) {
        mbar_init(&bars[0], 1);   // loads
        mbar_init(&bars[1], 1);   // MMA
        mbar_init(&bars[2], 1);   // Kbar of the first half (deferred T and W)
        fence_barrier_init();
        uint64_t *full = &bars[0];
        const uint32_t opnd = (uint32_t)(CC * DK * 2);   // one 64-row operand tile
        mbar_arrive_expect_tx(full, 2u * prep::IMG + 2u * opnd);
        bulk_load(base + Ly.NTL, rec1 + a.base_bytes + prep::PAIR_N, prep::IMG, full);
        bulk_load(base + Ly.NTL + 128 * 128 + 64 * 128, rec2 + a.base_bytes + prep::PAIR_N, prep::IMG, full);
        if (a.ext) {
            // Khat1 (the first half's record) and Kbar2 (the second half's pair extra),
            // 64-row tiles of DK / 64 column blocks, as the records store them
            bulk_load(base + Ly.RT, rec1 + prep::ext_kh(DK), opnd, full);
            bulk_load(base + Ly.RT + opnd, rec2 + a.base_bytes + prep::PAIR_KB, opnd, full);
        } else {
            for (int kb = 0; kb < DK / 64; ++kb) {
                tma_load_3d(base + Ly.RT + kb * 64 * 128, &tm_k, full, 64 * kb, c1 * CC, (int)kh);
                tma_load_3d(base + Ly.RT + opnd + kb * 64 * 128, &tm_k, full, 64 * kb, (int)c0_2, (int)kh);
            }
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    for (int t = tid; t < CC; t += NT) {
        sbeta[t] = t < Cl2 ? p.beta[kh * T + c0_2 + t] : 0.f;
        if (a.defer_tw)
            beta1[t] = p.beta[kh * T + (long)c1 * CC + t];   // a first half is whole
        if (!a.ext) {   // e^{Lambda_t} of half 2, e^{Lambda_mid - Lambda_j} of half 1
            ea2[t] = reinterpret_cast<const float *>(rec2 + prep::SC_EA)[t];
            eb1[t] = reinterpret_cast<const float *>(rec1 + prep::SC_EB)[t];
        }
    }
    // the zero block of Ntil (rows 0-63 of columns 64-127), X = I
    for (int u = tid; u < 64 * 8; u += NT) {
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        st_tile8(NTL, 128, u >> 3, 64 + (u & 7) * 8, z);
    }
    for (int u = tid; u < 128 * 16; u += NT) {
        const int r = u >> 4, c = (u & 15) * 8;
        float x8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            x8[e] = (r == c + e) ? 1.f : 0.f;
        st_tile8(XT, 128, r, c, x8);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);

    uint32_t ph_mma = 0;
    bool failed = false;
    int kb_loads = 0;        // (thread 0) phases armed on the Kbar barrier
    auto wait_bar = [&](int i, uint32_t ph) {
        const bool gave_up = !mbar_wait(&bars[i], ph);
        if (gave_up)
            atomicExch(&g_device_status, kTimeoutStatus);
        return __syncthreads_or(gave_up ? 1 : 0) != 0;
    };
    failed = wait_bar(0, 0);
    const uint32_t KH1 = RT, KB2 = RT + (uint32_t)(CC * DK * 2);
    if (!failed && !a.ext) {   // scalar gate: scale the raw k rows by their decay factors
        for (int u = tid; u < 2 * CC * (DK / 8); u += NT) {
            const int h = u / (CC * (DK / 8)), r = (u / (DK / 8)) % CC, i0 = (u % (DK / 8)) * 8;
            const uint32_t tile = h == 0 ? KH1 : KB2;
            const float f = h == 0 ? eb1[r] : ea2[r];
            float v8[8];
            ld_tile8(tile, 64, r, i0, v8);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                v8[e] *= f;
            st_tile8(tile, 64, r, i0, v8);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- G21 = Kbar2' Khat1^T (M = 64, N = 64, K = DK)
    if (!failed) {
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, 64, false, false);
            for (int k0 = 0; k0 < DK; k0 += 16)
                mma_bf16(tmem + T_D, desc_kmajor(KB2, 64, 0, k0), desc_kmajor(KH1, 64, 0, k0), id, k0 > 0);
            mma_commit(&bars[1]);
        }
        failed = wait_bar(1, ph_mma);
        ph_mma ^= 1u;
    }
    if (!failed) {
        tc_fence_after();
        const int rr = gen::row64g(warp, lane);
        const int cb = 32 * (warp >> 2);
        float d0[16], d1[16];
        tmem_ld16(tq + T_D + cb, d0);
        tmem_ld16(tq + T_D + cb + 16, d1);
        tmem_ld_wait();
        if (rr >= 0) {
            const float bt = sbeta[rr];
            float n[32];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                n[u] = bt * d0[u];
                n[16 + u] = bt * d1[u];
            }
#pragma unroll
            for (int u = 0; u < 32; u += 8)
                st_tile8(NTL, 128, 64 + rr, cb + u, &n[u]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- the 128 x 128 series: products D = A B with M = N = K = 128
    const int R = 32 * (warp & 3) + lane;   // row of this thread (lane of its quarter)
    const int ch = 64 * (warp >> 2);        // its 64 columns
    const uint32_t id128 = idesc_bf16(128, 128, false, true);
    auto product = [&](uint32_t a_tile, uint32_t b_tile) {
        if (tid == 0) {
            tc_fence_after();
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma_bf16(tmem + T_D, desc_kmajor(a_tile, 128, 0, k0), desc_mnmajor(b_tile, 128, k0, 0),
                         id128, k0 > 0);
            mma_commit(&bars[1]);
        }
        const bool f = wait_bar(1, ph_mma);
        ph_mma ^= 1u;
        if (!f)
            tc_fence_after();
        return f;
    };
    // X (fp32, tensor memory) and its bf16 operand: this thread's row R, 16 columns at a time
    auto put_x = [&](int c, const float (&x)[16]) {
        tmem_st16(tq + T_X + c, x);
        st_tile8(XT, 128, R, c, &x[0]);
        st_tile8(XT, 128, R, c + 8, &x[8]);
    };
    if (!failed && p.neu_order == 0) {
        for (int c = ch; c < ch + 64; c += 16) {
            float x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                x[e] = (R == c + e) ? 1.f : 0.f;
            tmem_st16(tq + T_X + c, x);
        }
    }
    // order 4 (the default): X = I - N + N^2 - N^3 + N^4 = (I + P2) - N (I + P2) + P2 P2 with
    // P2 = N^2, two product round trips instead of Horner's four (the same series, other
    // rounding); the B operand -(I + P2) makes the sum one accumulation
    const bool quad = p.neu_order == 4;
    if (!failed && quad) {
        if (!(failed = product(NTL, NTL))) {
            for (int c = ch; c < ch + 64; c += 16) {
                float d[16], x[16];
                tmem_ld16(tq + T_D + c, d);
                tmem_ld_wait();
                tmem_st16(tq + T_X + c, d);                      // P2, fp32
                st_tile8(RT, 128, R, c, &d[0]);                  // P2 (bf16, both operands)
                st_tile8(RT, 128, R, c + 8, &d[8]);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] = -(((R == c + e) ? 1.f : 0.f) + d[e]);
                st_tile8(XT, 128, R, c, &x[0]);                  // -(I + P2)
                st_tile8(XT, 128, R, c + 8, &x[8]);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
        }
        if (!failed) {
            if (tid == 0) {
                tc_fence_after();
                for (int k0 = 0; k0 < 128; k0 += 16)
                    mma_bf16(tmem + T_D, desc_kmajor(NTL, 128, 0, k0), desc_mnmajor(XT, 128, k0, 0), id128,
                             k0 > 0);
                for (int k0 = 0; k0 < 128; k0 += 16)
                    mma_bf16(tmem + T_D, desc_kmajor(RT, 128, 0, k0), desc_mnmajor(RT, 128, k0, 0), id128, 1u);
                mma_commit(&bars[1]);
            }
            failed = wait_bar(1, ph_mma);
            ph_mma ^= 1u;
        }
        if (!failed) {
            tc_fence_after();
            for (int c = ch; c < ch + 64; c += 16) {
                float d[16], x[16];
                tmem_ld16(tq + T_D + c, d);
                tmem_ld16(tq + T_X + c, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] += ((R == c + e) ? 1.f : 0.f) + d[e];
                put_x(c, x);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
        }
    }
    for (int pw = 1; pw <= (quad ? 0 : p.neu_order) && !failed; ++pw) {   // X <- I - Ntil X
        if ((failed = product(NTL, XT)))
            break;
        for (int c = ch; c < ch + 64; c += 16) {
            float d[16], x[16];
            tmem_ld16(tq + T_D + c, d);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                x[e] = ((R == c + e) ? 1.f : 0.f) - d[e];
            put_x(c, x);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    for (int st = 0; st < p.neu_resid && !failed; ++st) {   // Newton: X <- X + X (I - X - Ntil X)
        if ((failed = product(NTL, XT)))
            break;
        for (int c = ch; c < ch + 64; c += 16) {
            float d[16], x[16];
            tmem_ld16(tq + T_D + c, d);
            tmem_ld16(tq + T_X + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                d[e] = ((R == c + e) ? 1.f : 0.f) - x[e] - d[e];
            st_tile8(RT, 128, R, c, &d[0]);
            st_tile8(RT, 128, R, c + 8, &d[8]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if ((failed = product(XT, RT)))
            break;
        for (int c = ch; c < ch + 64; c += 16) {
            float d[16], x[16];
            tmem_ld16(tq + T_D + c, d);
            tmem_ld16(tq + T_X + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                x[e] += d[e];
            put_x(c, x);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    // ---- the halves' own T and W, left by the first pass: T_h = diag(beta_h) A_hh =
    //      Atil_hh diag(beta_h), Atil_hh the h-th diagonal block of X (the half's own
    //      series), and W_h = T_h Kbar_h (M = 64, N = dk, K = 64), into the halves' records
    //      as the first pass would have written them (W negated for the 128-column pass)
    const bool tw_series = a.defer_tw && !p.neumann1;   // (1-Step Neumann: in its branch below)
    if (!failed && tw_series && tid == 0) {   // both halves' Kbar over the dead residual tile
        const uint32_t opnd = (uint32_t)(CC * DK * 2);
        kb_loads = 1;
        mbar_arrive_expect_tx(&bars[2], 2u * opnd);
        bulk_load(base + Ly.RT, rec1 + a.base_bytes + prep::PAIR_KB, opnd, &bars[2]);
        bulk_load(base + Ly.RT + opnd, rec2 + a.base_bytes + prep::PAIR_KB, opnd, &bars[2]);
    }
    for (int h = 0; h < 2 && !failed && tw_series; ++h) {
        uint8_t *rec = h == 0 ? rec1 : rec1 + a.rec_bytes;
        const float *bh = h == 0 ? beta1 : sbeta;
        const uint32_t TBh = XT + h * 8192;      // X's bf16 operand is dead
        tc_fence_after();
        if ((R < 64) == (h == 0) && ch == 64 * h) {   // warps holding rows of the block
            const int r = R - 64 * h;
            for (int c = 0; c < 64; c += 16) {
                float x[16];
                tmem_ld16(tq + T_X + ch + c, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] *= bh[c + e];
                prep::st_img8(rec, r, c, &x[0]);
                prep::st_img8(rec, r, c + 8, &x[8]);
                st_tile8(TBh, 64, r, c, &x[0]);
                st_tile8(TBh, 64, r, c + 8, &x[8]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (h == 0 && (failed = wait_bar(2, 0)))
            break;
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(64, DK, false, true);
            const uint32_t KBh = RT + h * (uint32_t)(CC * DK * 2);
            for (int k0 = 0; k0 < CC; k0 += 16)
                mma_bf16(tmem + T_D, desc_kmajor(TBh, 64, 0, k0), desc_mnmajor(KBh, 64, k0, 0), id, k0 > 0);
            mma_commit(&bars[1]);
        }
        failed = wait_bar(1, ph_mma);
        ph_mma ^= 1u;
        if (!failed) {
            tc_fence_after();
            const int rr = gen::row64g(warp, lane);
            const int cw = (DK / 2) * (warp >> 2);   // this warp's half of the dk columns
#pragma unroll
            for (int cb = 0; cb < DK / 2; cb += 32) {
                float w0[16], w1[16];
                tmem_ld16(tq + T_D + cw + cb, w0);
                tmem_ld16(tq + T_D + cw + cb + 16, w1);
                tmem_ld_wait();
                if (rr >= 0) {
                    if (a.neg_w) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            w0[e] = -w0[e];
                            w1[e] = -w1[e];
                        }
                    }
                    const int col = cw + cb;   // 32 columns inside one 64-column image
                    uint8_t *img_W = rec + prep::REC_W + (col >> 6) * prep::IMG;
                    prep::st_img8(img_W, rr, col & 63, &w0[0]);
                    prep::st_img8(img_W, rr, (col & 63) + 8, &w0[8]);
                    prep::st_img8(img_W, rr, (col & 63) + 16, &w1[0]);
                    prep::st_img8(img_W, rr, (col & 63) + 24, &w1[8]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();   // the product is read back before the next one lands there
    }

    if (!p.neumann1) {
        // ---- Y = Atil21 Atil11^{-1} + Atil22 Ntil21 on tcgen05 (M = N = K = 64) in split
        //      bf16 terms: with P = Ph + Pl (Ph the bf16 rounding of the fp32 P, Pl that of
        //      the rest), P Q ~ Ph Qh + Ph Ql + Pl Qh in fp32, the dropped Pl Ql being 2^-16
        //      of the product; Ntil21 is exactly the bf16 operand the series used.  The
        //      inverse Atil11^{-1} stays in fp32 on the CUDA cores (block doubling).
        float *A11f = f32(base, Ly.XT);                  // strict lower part: I + H form
        const uint32_t A21H = RT, A21L = RT + 8192, A22H = RT + 16384, A22L = RT + 24576;
        const uint32_t IH = NTL + 128 * 128, IL = IH + 8192;   // the dead columns 64-127 of Ntil
        auto split_store = [&](uint32_t th, uint32_t tl, int r, int c, const float *v) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const uint32_t h = pack_bf16(v[e], v[e + 1]);
                hi[e] = bf16lo(h);
                hi[e + 1] = bf16hi(h);
                lo[e] = v[e] - hi[e];
                lo[e + 1] = v[e + 1] - hi[e + 1];
            }
            st_tile8(th, 64, r, c, hi);
            st_tile8(tl, 64, r, c, lo);
        };
        if (!failed) {
            tc_fence_after();
            // Atil from tensor memory: Atil11 (strict lower part) to fp32 for the inverse,
            // Atil21 and Atil22 straight to their split operand tiles
            for (int c = 0; c < 64; c += 16) {
                float x[16];
                tmem_ld16(tq + T_X + ch + c, x);
                tmem_ld_wait();
                if (ch == 0 && R < 64) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        A11f[R * LDM + c + e] = (R > c + e) ? x[e] : 0.f;
                } else if (R >= 64) {
                    const uint32_t th = ch == 0 ? A21H : A22H, tl = ch == 0 ? A21L : A22L;
                    split_store(th, tl, R - 64, c, &x[0]);
                    split_store(th, tl, R - 64, c + 8, &x[8]);
                }
            }
        }
        __syncthreads();
        if (!failed) {
            gen::inverse64_mid(A11f, Tf, tid);            // Atil11^{-1}, unit lower triangular
            for (int u = tid; u < CC * 8; u += NT) {
                const int r = u >> 3, c = (u & 7) * 8;
                split_store(IH, IL, r, c, A11f + r * LDM + c);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (!failed) {
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id64 = idesc_bf16(64, 64, false, true);
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    const uint64_t a21h = desc_kmajor(A21H, 64, 0, k0), a21l = desc_kmajor(A21L, 64, 0, k0);
                    const uint64_t a22h = desc_kmajor(A22H, 64, 0, k0), a22l = desc_kmajor(A22L, 64, 0, k0);
                    const uint64_t ih = desc_mnmajor(IH, 64, k0, 0), il = desc_mnmajor(IL, 64, k0, 0);
                    const uint64_t n21 = desc_mnmajor(NTL, 128, 64 + k0, 0);
                    mma_bf16(tmem + T_D, a21h, ih, id64, k0 > 0);
                    mma_bf16(tmem + T_D, a21h, il, id64, 1u);
                    mma_bf16(tmem + T_D, a21l, ih, id64, 1u);
                    mma_bf16(tmem + T_D, a22h, n21, id64, 1u);
                    mma_bf16(tmem + T_D, a22l, n21, id64, 1u);
                }
                mma_commit(&bars[1]);
            }
            failed = wait_bar(1, ph_mma);
            ph_mma ^= 1u;
        }
        if (!failed) {   // Y (M = 64 accumulator: rows in lanes 0-15 of each quarter) as an image
            tc_fence_after();
            const int rr = gen::row64g(warp, lane);
            const int cb = 32 * (warp >> 2);
            float d0[16], d1[16];
            tmem_ld16(tq + T_D + cb, d0);
            tmem_ld16(tq + T_D + cb + 16, d1);
            tmem_ld_wait();
            if (rr >= 0) {
                prep::st_img8(img_Y, rr, cb, &d0[0]);
                prep::st_img8(img_Y, rr, cb + 8, &d0[8]);
                prep::st_img8(img_Y, rr, cb + 16, &d1[0]);
                prep::st_img8(img_Y, rr, cb + 24, &d1[8]);
            }
        }
    } else {
        // ---- the 1-Step Neumann inverse: Atil21 from the diagonal blocks, Y in fp32
        float *N21f = f32(base, Ly.XT);                  // 64 x LDM each
        float *A11f = N21f + CC * LDM;
        float *A21f = A11f + CC * LDM;
        float *A22f = f32(base, Ly.NTL);                 // once Ntil21 is copied out
        if (!failed) {
            // 1-Step Neumann ("Systolic Linear Attention ...", §2.4.3), in fp32 from the bf16
            // blocks: Atil = Dtil^{-1} - Dtil^{-1} Ntil_off Dtil^{-1}, Dtil the diagonal 16 x 16
            // blocks of I + Ntil; per half that is the first pass's 64-token factor, and across
            // the halves Atil21 = -bd(Atil22) Ntil21 bd(Atil11) (bd: the diagonal blocks)
            for (int u = tid; u < CC * 8; u += NT) {
                const int t = u >> 3, j0 = (u & 7) * 8;
                float a8[8], n8[8];
                ld_tile8(NTL, 128, t, j0, a8);
                ld_tile8(NTL, 128, 64 + t, j0, n8);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    A11f[t * LDM + j0 + e] = (t > j0 + e) ? a8[e] : 0.f;
                    N21f[t * LDM + j0 + e] = n8[e];
                }
            }
            __syncthreads();
            for (int u = tid; u < CC * 8; u += NT) {   // Ntil22 lies past the bytes of A22f
                const int t = u >> 3, j0 = (u & 7) * 8;
                float a8[8];
                ld_tile8(NTL, 128, 64 + t, 64 + j0, a8);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    A22f[t * LDM + j0 + e] = (t > j0 + e) ? a8[e] : 0.f;
            }
            __syncthreads();
            gen::block_neumann1_64_inplace(A11f, Tf, tid);
            gen::block_neumann1_64_inplace(A22f, Tf, tid);
            // the halves' own T and W, left by the first pass: T_h = Atil_hh diag(beta_h) from
            // the fp32 blocks, W_h = T_h Kbar_h, one half at a time in the residual tile's
            // dead tail (Atil11's last rows end 2 KB into it)
            for (int h = 0; h < 2 && a.defer_tw && !failed; ++h) {
                uint8_t *rec = h == 0 ? rec1 : rec1 + a.rec_bytes;
                const float *Ah = h == 0 ? A11f : A22f;
                const float *bh = h == 0 ? beta1 : sbeta;
                const uint32_t TBs = RT + 8192, KBs = RT + 16384;
                if (tid == 0) {
                    const uint32_t opnd = (uint32_t)(CC * DK * 2);
                    kb_loads = h + 1;
                    mbar_arrive_expect_tx(&bars[2], opnd);
                    bulk_load(base + Ly.RT + 16384, rec + a.base_bytes + prep::PAIR_KB, opnd, &bars[2]);
                }
                for (int u = tid; u < CC * 8; u += NT) {
                    const int r = u >> 3, c = (u & 7) * 8;
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v[e] = Ah[r * LDM + c + e] * bh[c + e];
                    prep::st_img8(rec, r, c, v);
                    st_tile8(TBs, 64, r, c, v);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if ((failed = wait_bar(2, (uint32_t)h)))
                    break;
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(64, DK, false, true);
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_D, desc_kmajor(TBs, 64, 0, k0), desc_mnmajor(KBs, 64, k0, 0), id,
                                 k0 > 0);
                    mma_commit(&bars[1]);
                }
                failed = wait_bar(1, ph_mma);
                ph_mma ^= 1u;
                if (failed)
                    break;
                tc_fence_after();
                const int rr = gen::row64g(warp, lane);
                const int cw = (DK / 2) * (warp >> 2);
#pragma unroll
                for (int cb = 0; cb < DK / 2; cb += 32) {
                    float w0[16], w1[16];
                    tmem_ld16(tq + T_D + cw + cb, w0);
                    tmem_ld16(tq + T_D + cw + cb + 16, w1);
                    tmem_ld_wait();
                    if (rr >= 0) {
                        if (a.neg_w) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                w0[e] = -w0[e];
                                w1[e] = -w1[e];
                            }
                        }
                        const int col = cw + cb;
                        uint8_t *img_W = rec + prep::REC_W + (col >> 6) * prep::IMG;
                        prep::st_img8(img_W, rr, col & 63, &w0[0]);
                        prep::st_img8(img_W, rr, (col & 63) + 8, &w0[8]);
                        prep::st_img8(img_W, rr, (col & 63) + 16, &w1[0]);
                        prep::st_img8(img_W, rr, (col & 63) + 24, &w1[8]);
                    }
                }
                tc_fence_before();
                __syncthreads();   // read back (and the tiles read) before the next half
            }
            const int rg = tid >> 4, c0 = 4 * (tid & 15), lb = c0 & ~15, lr = 16 * (rg >> 2);
            float acc[4][4];
            // Z = Ntil21 bd(Atil11): rows rg + 16 i, columns c0..c0+3 (one 16-column block)
            gen::block_product4x4<16>(acc, N21f + rg * LDM + lb, 16 * LDM, A11f + lb * LDM + c0, LDM, 0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    A21f[(rg + 16 * i) * LDM + c0 + n] = acc[i][n];
            __syncthreads();
            // Atil21 = -bd(Atil22) Z: rows 4 rg .. 4 rg + 3 (one 16-row block)
            gen::block_product4x4<16>(acc, A22f + (4 * rg) * LDM + lr, LDM, A21f + lr * LDM + c0, LDM, 0);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    A21f[(4 * rg + i) * LDM + c0 + n] = -acc[i][n];
            for (int u = tid; u < CC * CC; u += NT) {   // Atil11 as I + H for the exact inverse
                const int t = u / CC, j = u % CC;
                if (t <= j)
                    A11f[t * LDM + j] = 0.f;
            }
            __syncthreads();
        }
        // ---- Y = Atil21 Atil11^{-1} + Atil22 Ntil21 on tcgen05 from split bf16 operands, as in
        //      the truncated series' branch, in two stages for want of free tiles beside the
        //      fp32 blocks: Atil22 Ntil21 (Ntil21 exact in bf16), then Atil21 Atil11^{-1} onto it
        auto split_store = [&](uint32_t th, uint32_t tl, int r, int c, const float *v) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const uint32_t hh = pack_bf16(v[e], v[e + 1]);
                hi[e] = bf16lo(hh);
                hi[e + 1] = bf16hi(hh);
                lo[e] = v[e] - hi[e];
                lo[e + 1] = v[e + 1] - hi[e + 1];
            }
            st_tile8(th, 64, r, c, hi);
            st_tile8(tl, 64, r, c, lo);
        };
        const uint32_t id64 = idesc_bf16(64, 64, false, true);
        if (!failed) {
            gen::inverse64_mid(A11f, Tf, tid);                // Atil11^{-1}, lower triangular
            // stage 1 tiles: Ntil21 over the first 8 KB of its fp32 copy (read out first),
            // Atil22 high / low past the fp32 blocks in the residual and Ntil tiles
            const uint32_t N21T = XT, A22H = RT + 20480, A22L = NTL + 18432;
            float nv[2][8];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int u = tid + NT * k, r = u >> 3, c = (u & 7) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    nv[k][e] = N21f[r * LDM + c + e];
                split_store(A22H, A22L, r, c, A22f + r * LDM + c);
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int u = tid + NT * k;
                st_tile8(N21T, 64, u >> 3, (u & 7) * 8, nv[k]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    const uint64_t n21 = desc_mnmajor(N21T, 64, k0, 0);
                    mma_bf16(tmem + T_D, desc_kmajor(A22H, 64, 0, k0), n21, id64, k0 > 0);
                    mma_bf16(tmem + T_D, desc_kmajor(A22L, 64, 0, k0), n21, id64, 1u);
                }
                mma_commit(&bars[1]);
            }
            failed = wait_bar(1, ph_mma);
            ph_mma ^= 1u;
        }
        if (!failed) {
            // stage 2 tiles: over the dead fp32 Ntil21 / Atil22 and stage 1's Atil22 high part
            const uint32_t A21H = XT + 8192, A21L = NTL, IH = NTL + 8192, IL = RT + 20480;
            for (int u = tid; u < CC * 8; u += NT) {
                const int r = u >> 3, c = (u & 7) * 8;
                split_store(A21H, A21L, r, c, A21f + r * LDM + c);
                split_store(IH, IL, r, c, A11f + r * LDM + c);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                for (int k0 = 0; k0 < CC; k0 += 16) {
                    const uint64_t a21h = desc_kmajor(A21H, 64, 0, k0), a21l = desc_kmajor(A21L, 64, 0, k0);
                    const uint64_t ih = desc_mnmajor(IH, 64, k0, 0), il = desc_mnmajor(IL, 64, k0, 0);
                    mma_bf16(tmem + T_D, a21h, ih, id64, 1u);
                    mma_bf16(tmem + T_D, a21h, il, id64, 1u);
                    mma_bf16(tmem + T_D, a21l, ih, id64, 1u);
                }
                mma_commit(&bars[1]);
            }
            failed = wait_bar(1, ph_mma);
            ph_mma ^= 1u;
        }
        if (!failed) {   // Y (M = 64 accumulator: rows in lanes 0-15 of each quarter) as an image
            tc_fence_after();
            const int rr = gen::row64g(warp, lane);
            const int cb = 32 * (warp >> 2);
            float d0[16], d1[16];
            tmem_ld16(tq + T_D + cb, d0);
            tmem_ld16(tq + T_D + cb + 16, d1);
            tmem_ld_wait();
            if (rr >= 0) {
                prep::st_img8(img_Y, rr, cb, &d0[0]);
                prep::st_img8(img_Y, rr, cb + 8, &d0[8]);
                prep::st_img8(img_Y, rr, cb + 16, &d1[0]);
                prep::st_img8(img_Y, rr, cb + 24, &d1[8]);
            }
        }
    }
    if (tid == 0 && failed) {   // drain what was started before releasing tensor memory
        mma_commit(&bars[1]);
        mbar_wait(&bars[1], ph_mma, 200000000ull);
        mbar_wait(&bars[0], 0, 200000000ull);
        if (kb_loads > 0)
            mbar_wait(&bars[2], (kb_loads - 1) & 1, 200000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

inline int npairs(int nchunks) { return (nchunks + 1) / 2; }

template <int DK>
int launch(const Params &p, void *records, cudaStream_t stream, int neg_w = 0)
{
    const int N = prep::nchunks(p);
    if (N == 0 || p.B == 0)
        return 0;
    CUtensorMap mk;
    if (!make_map(&mk, p.k, DK, p.T, (long)p.B * p.Hk, CC))
        return 6;
    const Plan Ly = plan<DK>();
    if (cudaFuncSetAttribute(pair_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    PairArgs a;
    a.p = p;
    a.rec = static_cast<uint8_t *>(records);
    a.nchunks = N;
    a.rec_bytes = prep::rec_bytes(p);
    a.base_bytes = prep::kind_bytes(prep::record_kind(p), DK);
    a.ext = prep::record_kind(p) == prep::REC_EXT;
    // the first pass leaves T and W of paired halves here (both Neumann inverses, dk = 128,
    // grouped / per-channel records): the same condition as its own
    a.defer_tw = DK == 128 && a.ext && (p.neumann || p.neumann1);
    a.neg_w = neg_w;
    pair_kernel<DK><<<dim3(npairs(N), p.Hk, p.B), NT, Ly.total, stream>>>(mk, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace pair
