// gdr_tc_prep.cuh -- first pass of the two-pass tensor-core path: the
// chunk-local factors of every (batch, key head, chunk), computed for all
// chunks in parallel.  Included by gdr_tc.cu.
//
// Per chunk of C = 64 tokens ("Systolic Linear Attention: Co-Designing
// Tile-Grouped Gated Delta Attention for TPUs", §2.1, §2.3 Table 2, §2.4.2;
// "Kimi Linear" chunkwise KDA, decay pivots):
//   1. TMA: q and k as one [q; k] tile of 128 rows (zero past T); beta and the
//      log-gates g through plain loads (zero past T: the recurrence is then
//      left untouched by the padding rows).
//   2. Lambda = cumsum g per decay group (fp32).
//   3. Decayed Grams on tcgen05, never dividing by a decay prefix:
//        scalar gate: [Q; K] K^T once, then the factor e^{Lambda_t - Lambda_j}
//          (t >= j, so <= 1) on the way out of TMEM;
//        grouped / per-channel gate: when each half of the chunk spans at most
//          kGuard nats of decay, one pivot p = 32 in the middle of the chunk (rows
//          scaled by e^{Lambda_t - Lambda_p}, columns by e^{Lambda_p - Lambda_j}, each
//          at most e^{kGuard}, from two exponentials per element: every decayed
//          operand of the record is these times a per-channel constant); otherwise
//          two row blocks of 32 tokens, each with
//          its own pivot p in the middle of the block.  Rows t of the block
//          carry e^{Lambda_t - Lambda_p}, columns j carry e^{Lambda_p - Lambda_j};
//          both factors are at most e^{(half-block decay span)}, and their
//          product is the exact e^{Lambda_t - Lambda_j}.  A block whose half
//          span exceeds kGuard nats is recomputed element by element in fp32.
//      L_tj = (t >= j) q_t . k_j decayed,  M_tj = (t > j) beta_j k_t . k_j decayed.
//   4. A = (I + M)^{-1}: exact fp32 block doubling, or the truncated Neumann
//      series with Newton residual steps on tcgen05 ("When Good Enough Is
//      Optimal: Multiplication-Only Matrix Inversion Approximation for
//      Quantized Gated DeltaNet", Lemma 3.1, §4.1).
//   5. Output, per chunk, two bf16 C x C tiles: T = diag(beta) A and L, each as
//      the byte image of a 128-byte-swizzled shared-memory tile (64 rows x 128
//      bytes, 16-byte chunk index XOR (row % 8)), so that the second pass can
//      bring them in with one bulk copy each.  For grouped / per-channel gates
//      the record the state pass reads also carries the decayed operands
//      Qbar = q e^{Lambda_t}, Khat = k e^{Lambda_C - Lambda_t}, Kbar = k e^{Lambda_t}
//      (C x dk bf16 images, 64-column blocks of 64 rows) and F = e^{Lambda_C}
//      (dk fp32): every factor is the exponential of a non-positive difference.

namespace prep {

constexpr int NT = 256;
constexpr int CC = 64;
constexpr int LDM = gen::LDM;              // row stride of the fp32 C x C scratch
constexpr int NROUND = 2;                  // pivot blocks of 32 rows
constexpr float kGuard = 64.f;             // largest exponent a pivoted factor may take
constexpr uint32_t IMG = CC * CC * 2;      // one bf16 C x C tile image
constexpr uint32_t CHUNK_BYTES = 2 * IMG;  // T, then L
// Records of the two-pass path's workspace (key width 128).  Both start with T,
// L and W = diag(beta) A Kbar (64 x 128 bf16: two 64-column images).
// scalar gate: then e^{Lambda_t}, e^{Lambda_C - Lambda_t}, e^{Lambda_C}
constexpr uint32_t REC_W = 2 * IMG;
constexpr uint32_t SC_EA = 4 * IMG, SC_EB = SC_EA + CC * 4, SC_F = SC_EB + CC * 4;
constexpr uint32_t SC_BYTES = SC_F + 16;
// grouped / per-channel gates: then Qbar, Khat (64 x dk bf16 each, dk / 64 images)
// and F (dk fp32); offsets for key width dk:
__host__ __device__ constexpr uint32_t ext_qb(int dk) { return (2u + dk / 64) * IMG; }
__host__ __device__ constexpr uint32_t ext_kh(int dk) { return (2u + 2 * (dk / 64)) * IMG; }
__host__ __device__ constexpr uint32_t ext_f(int dk) { return (2u + 3 * (dk / 64)) * IMG; }
__host__ __device__ constexpr uint32_t ext_bytes(int dk) { return ext_f(dk) + dk * 4; }
constexpr uint32_t EXT_QB = ext_qb(128), EXT_KH = ext_kh(128), EXT_F = ext_f(128);
constexpr uint32_t EXT_BYTES = ext_bytes(128);
enum RecordKind { REC_PLAIN = 0, REC_SCALAR = 1, REC_EXT = 2 };
// Pair records (the truncated Neumann inverse at C = 128 run as two 64-token
// halves): the base record, then Y (the pair's correction, written by
// pair_kernel into the record of the pair's first half), Ntil = diag(beta) x the
// decayed Gram of the half (beta on the rows: strictly lower, bf16 image) and,
// for grouped / per-channel gates, Kbar = k e^{Lambda_t} (64 x dk bf16, dk / 64
// images).
constexpr uint32_t PAIR_Y = 0, PAIR_N = IMG, PAIR_KB = 2 * IMG;   // offsets past the base record
__host__ __device__ constexpr uint32_t pair_extra(int kind, int dk = 128)
{
    return kind == REC_EXT ? (2u + dk / 64) * IMG : 2 * IMG;
}

__host__ __device__ constexpr int gmax(int dk) { return dk == 256 ? 8 : 128; }

struct Plan {
    uint32_t QK, RA, KC, Mf, Tf, NB, XB, RB, TB, lam, beta, piv, bar, misc, total, tmem_cols, tn;
};

// Rows of Lambda that the register-resident form (rl) keeps in shared memory.
enum LamRow { LR_0 = 0, LR_P = 1, LR_C = 2, LR_16 = 3, LR_48 = 4, LR_N = 5 };

// rl: per-channel Lambda lives in registers (dk = 128, grouped / per-channel gates,
// extended records), so the 32 KB Lambda tile is gone and three CTAs fit on an SM.
__host__ __device__ inline Plan plan(int dk, int G, bool neumann, bool rl = false)
{
    Plan s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    // The k rows of QK outlive the inverse (W = T Kbar reads them at the end);
    // the q rows are dead after the Grams and hold T (bf16) for that product.
    s.QK = take((dk / 64) * 128 * 128);          // rows 0-63 q, 64-127 k
    s.TB = s.QK;
    if (G > 1) {
        s.RA = take((dk / 64) * 64 * 128);        // round rows: 16 of q, 16 of k
        s.KC = take((dk / 64) * 64 * 128);        // round columns
        s.Mf = s.RA;                              // fp32 scratch, once the Grams are read
    } else {
        s.RA = s.KC = 0;
        s.Mf = take(CC * LDM * 4 + 32 * 36 * 4);
    }
    s.Tf = s.Mf + CC * LDM * 4;
    const uint32_t lam_bytes = rl ? LR_N * dk * 4 : CC * G * 4;
    s.lam = take(lam_bytes + CC * 4 + NROUND * 4 + 64);   // Lambda, beta, flags, barriers
    s.beta = s.lam + lam_bytes;
    if (neumann && rl) {
        // the q rows of QK (dead after the Grams) and the end of the inverse's scratch
        s.NB = s.QK;
        s.XB = s.QK + 2 * 8192;
        s.RB = s.Mf + ((CC * LDM * 4 + 32 * 36 * 4 + 1023u) & ~1023u);
    } else if (neumann) {   // in the Lambda tile (dead by the inverse) when it is large enough
        s.NB = CC * G * 4 >= 3 * 8192 ? s.lam : take(3 * 8192);
        s.XB = s.NB + 8192;
        s.RB = s.NB + 16384;
    } else {
        s.NB = s.XB = s.RB = 0;
    }
    s.piv = G > 1 ? take(2 * dk * 4) : 0;   // per channel: e^{Lambda_p}, e^{Lambda_C - Lambda_p}
    s.bar = (s.beta + CC * 4 + NROUND * 4 + 7u) & ~7u;
    s.misc = s.bar + 24;
    s.total = o + 1024;
    // W (M = 64, N = dk) needs dk columns; three CTAs a SM (rl) share the 512 columns, so
    // their Neumann products reuse the Grams' columns 64-127 (read out by then)
    s.tmem_cols = ((G > 1 && !rl) || dk > 128) ? 256u : 128u;
    s.tn = (G > 1 && !rl) ? 192u : 64u;           // Neumann products
    return s;
}

struct PrepArgs {
    Params p;
    uint8_t *out;      // [B * Hk * nchunks][rec_bytes]
    int nchunks;
    int kind;          // RecordKind: what besides T and L the record carries
    uint32_t rec_bytes;
    uint32_t base_bytes;   // the kind's own record; pair extras follow it (pair != 0)
    int pair;              // also write the pair extras (Ntil, and Kbar for REC_EXT)
    int neg_w;             // store -W (the 128-column state pass accumulates U - W S)
};

// Store 8 floats as bf16 into the 16-byte chunk of row r holding columns [c, c+8)
// of a 64 x 64 tile image in global memory.
__device__ __forceinline__ void st_img8(uint8_t *img, int r, int c, const float *v)
{
    const int cc = (c >> 3) ^ (r & 7);
    *reinterpret_cast<uint4 *>(img + r * 128 + cc * 16) =
        make_uint4(ptx::pack_bf16(v[0], v[1]), ptx::pack_bf16(v[2], v[3]),
                   ptx::pack_bf16(v[4], v[5]), ptx::pack_bf16(v[6], v[7]));
}

// Lambda of row t at the eight channels [i0, i0 + 8).  Per-channel gates read two
// vectors; grouped gates (64 or more channels a group) one broadcast value.
__device__ __forceinline__ void lam8(const float *lam, int G, int wsh, int t, int i0, float *o)
{
    if (wsh == 0) {
        const float4 a = *reinterpret_cast<const float4 *>(lam + t * G + i0);
        const float4 b = *reinterpret_cast<const float4 *>(lam + t * G + i0 + 4);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    } else if (wsh >= 3) {
        const float x = lam[t * G + (i0 >> wsh)];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            o[e] = x;
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            o[e] = lam[t * G + ((i0 + e) >> wsh)];
    }
}

// SCALAR: the scalar-gate instantiation (no pivoting machinery, four CTAs per SM);
// otherwise grouped / per-channel gates: RL keeps Lambda in registers (dk = 128,
// extended records; three CTAs per SM), else in a shared-memory tile (two per SM).
//
// RL: thread (tb, cg) = (tid / 16, tid % 16) owns tokens 4 tb .. 4 tb + 3 at the
// eight channels 8 cg .. 8 cg + 7 in every elementwise sweep; its Lambda values are
// a blocked scan (within its four tokens, then over the 16 token blocks), and the
// rows every thread needs (0, 16, 32, 48, 63) go to shared memory.
template <int DK, bool SCALAR, bool RL = false>
__global__ void __launch_bounds__(NT, SCALAR ? 4 : RL ? 3 : 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const PrepArgs a)
{
    using namespace ptx;
    static_assert(!RL || (DK == 128 && !SCALAR), "register-resident Lambda: dk = 128, gated by group");
    extern __shared__ uint8_t smem_raw[];
    const Params &p = a.p;
    const int G = SCALAR ? 1 : p.G;
    const bool neu = p.neumann != 0;
    const Plan Ly = plan(DK, G, neu, RL);
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t pad = base_u32 - smem_u32(smem_raw);
    uint8_t *base = smem_raw + pad;
    float *lam = reinterpret_cast<float *>(base + Ly.lam);
    float *sbeta = reinterpret_cast<float *>(base + Ly.beta);
    int *flag = reinterpret_cast<int *>(sbeta + CC);
    float *Mf = reinterpret_cast<float *>(base + Ly.Mf);
    float *Tf = reinterpret_cast<float *>(base + Ly.Tf);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const long kh = (long)b * p.Hk + hk;
    const int T = p.T;
    const long c0 = (long)c * CC;
    const int Cl = (int)min((long)CC, T - c0);
    const int wsh = __ffs(DK / G) - 1;      // channels per decay group = 2^wsh
    const uint32_t QK = base_u32 + Ly.QK, RA = base_u32 + Ly.RA, KC = base_u32 + Ly.KC;
    // L and W leave as whole images by bulk copies from shared memory (a thread holds
    // one row of them, so direct stores would each touch 16 or 32 lines): L is staged
    // in the q rows (scalar gate; read before T lands there) or in the second half of
    // the Grams' column tile, W in the inverse's scratch (dk = 128, read back before)
    // or the column tile (dk = 256, after L has left).
    const uint32_t Ls = SCALAR ? QK : KC + 8192;
    const uint32_t Ws = DK == 128 ? base_u32 + Ly.Mf : KC;
    constexpr bool W_STAGE = !(SCALAR && DK > 128);
    uint8_t *img_T = a.out + (size_t)(kh * a.nchunks + c) * a.rec_bytes;
    uint8_t *img_L = img_T + IMG;

    // The log-gates of a grouped / per-channel chunk are one contiguous run of Cl x G
    // floats: one bulk copy when it is 16-byte aligned (RL: into the Gram tiles, free
    // until the scan has read it), else plain loads.
    const float *g_src = p.g + (kh * T + c0) * G;
    const uint32_t g_bytes = (uint32_t)(Cl * G * 4);
    const bool g_bulk = !SCALAR && (g_bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(g_src) & 15u) == 0;
    float *g_tile = RL ? reinterpret_cast<float *>(base + Ly.RA) : lam;
    // beta of a full chunk: one 256-byte bulk copy on the q, k barrier when aligned
    const float *b_src = p.beta + kh * T + c0;
    const bool b_bulk = Cl == CC && (reinterpret_cast<uintptr_t>(b_src) & 15u) == 0;
    if (tid == 0) {
        mbar_init(&bars[0], 1);     // TMA of q, k
        mbar_init(&bars[1], 1);     // MMA
        mbar_init(&bars[2], 1);     // bulk copy of the log-gates
        fence_barrier_init();
        if (g_bulk) {
            mbar_arrive_expect_tx(&bars[2], g_bytes);
            bulk_load(g_tile, g_src, g_bytes, &bars[2]);
        }
        mbar_arrive_expect_tx(&bars[0], 2u * CC * DK * 2u + (b_bulk ? CC * 4u : 0u));
        if (b_bulk)
            bulk_load(sbeta, b_src, CC * 4u, &bars[0]);
        for (int kb = 0; kb < DK / 64; ++kb) {
            tma_load_3d(base + Ly.QK + kb * 128 * 128, &tm_q, &bars[0], 64 * kb, (int)c0, (int)kh);
            tma_load_3d(base + Ly.QK + kb * 128 * 128 + 64 * 128, &tm_k, &bars[0], 64 * kb, (int)c0,
                        (int)kh);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Ly.tmem_cols);
        tmem_relinquish();
    }
    if (!b_bulk)
        for (int t = tid; t < CC; t += NT)
            sbeta[t] = t < Cl ? b_src[t] : 0.f;
    // RL: this thread's log-gates (zero past T) into registers, from the bulk-copied
    // tile or straight from global memory
    const int cg = tid & 15, tb = tid >> 4, i0r = 8 * cg;
    float lv[RL ? 4 : 1][8];
    auto load_gates = [&](const float *src, bool vec) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int t = 4 * tb + k;
            if (t >= Cl) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    lv[k][e] = 0.f;
            } else if (vec) {
                const float4 x0 = *reinterpret_cast<const float4 *>(src + t * G + i0r);
                const float4 x1 = *reinterpret_cast<const float4 *>(src + t * G + i0r + 4);
                lv[k][0] = x0.x; lv[k][1] = x0.y; lv[k][2] = x0.z; lv[k][3] = x0.w;
                lv[k][4] = x1.x; lv[k][5] = x1.y; lv[k][6] = x1.z; lv[k][7] = x1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    lv[k][e] = src[t * G + ((i0r + e) >> wsh)];
            }
        }
    };
    if constexpr (RL) {
        if (!g_bulk)
            load_gates(g_src, wsh == 0 && (reinterpret_cast<uintptr_t>(p.g) & 15u) == 0);
    } else if (g_bulk) {
        for (int u = Cl * G + tid; u < CC * G; u += NT)   // rows past T (not copied)
            lam[u] = 0.f;
    } else {
        for (int u = tid; u < CC * G; u += NT)
            lam[u] = (u / G) < Cl ? g_src[u] : 0.f;
    }
    if (tid < NROUND)
        flag[tid] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);

    uint32_t ph_mma = 0;
    bool failed = false;
    auto wait_bar = [&](int i, uint32_t ph) {
        const bool gave_up = !mbar_wait(&bars[i], ph);
        if (gave_up)
            atomicExch(&g_device_status, kTimeoutStatus);
        return __syncthreads_or(gave_up ? 1 : 0) != 0;
    };
    if (g_bulk)
        failed = wait_bar(2, 0);

    // ---- Lambda = cumsum over the chunk per decay group
    if constexpr (RL) {
        if (g_bulk) {
            load_gates(g_tile, wsh == 0);
            __syncthreads();   // the gate tile has been read: its space takes the block totals
        }
        // blocked scan: the thread's four tokens, then the 16 token blocks in order
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int k = 1; k < 4; ++k)
                lv[k][e] += lv[k - 1][e];
        float *tot = reinterpret_cast<float *>(base + Ly.RA);   // [16][DK]: free until the Grams
        *reinterpret_cast<float4 *>(tot + tb * DK + i0r) = make_float4(lv[3][0], lv[3][1], lv[3][2], lv[3][3]);
        *reinterpret_cast<float4 *>(tot + tb * DK + i0r + 4) = make_float4(lv[3][4], lv[3][5], lv[3][6], lv[3][7]);
        __syncthreads();
        if (tid < DK) {   // exclusive prefix over the token blocks, one channel a thread
            float run = 0.f;
            for (int j = 0; j < 16; ++j) {
                const float x = tot[j * DK + tid];
                tot[j * DK + tid] = run;
                run += x;
            }
        }
        __syncthreads();
        {
            const float4 o0 = *reinterpret_cast<const float4 *>(tot + tb * DK + i0r);
            const float4 o1 = *reinterpret_cast<const float4 *>(tot + tb * DK + i0r + 4);
            const float off[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    lv[k][e] += off[e];
        }
        // the rows every thread reads: 0, 16, 32 (the pivot), 48 and 63 (the chunk's end)
        auto put = [&](int row, int k) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                lam[row * DK + i0r + e] = lv[k][e];
        };
        if (tb == 0) put(LR_0, 0);
        if (tb == 4) put(LR_16, 0);
        if (tb == 8) put(LR_P, 0);
        if (tb == 12) put(LR_48, 0);
        if (tb == 15) put(LR_C, 3);
        __syncthreads();
    } else if (G <= 8) {
        if (warp < G) {   // lane l holds rows 2l, 2l+1
            const float v0 = lam[(2 * lane) * G + warp], v1 = lam[(2 * lane + 1) * G + warp];
            float s = v0 + v1;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, d);
                if (lane >= d)
                    s += y;
            }
            const float r0 = (s - (v0 + v1)) + v0;
            lam[(2 * lane) * G + warp] = r0;
            lam[(2 * lane + 1) * G + warp] = r0 + v1;
        }
    } else {
        for (int gi = tid; gi < G; gi += NT) {
            float acc = 0.f;
            for (int t0 = 0; t0 < CC; t0 += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = lam[(t0 + e) * G + gi];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    acc += v[e];
                    lam[(t0 + e) * G + gi] = acc;
                }
            }
        }
    }
    // decay span of each half of the chunk per group: within kGuard nats a single
    // pivot in the middle of the chunk serves every pair; wider spans take the two
    // pivoted row blocks
    constexpr int PV = CC / 2;
    float *piv = reinterpret_cast<float *>(base + Ly.piv);   // e^{Lambda_p}, e^{Lambda_C - Lambda_p}
    // Lambda at the pivot and at the chunk's end, channel i
    auto lam_p = [&](int i) { return RL ? lam[LR_P * DK + i] : lam[PV * G + (i >> wsh)]; };
    auto lam_c = [&](int i) { return RL ? lam[LR_C * DK + i] : lam[(CC - 1) * G + (i >> wsh)]; };
    bool wide = false;
    if (RL) {
        if (tid < DK) {
            const float l0 = lam[LR_0 * DK + tid], lp = lam_p(tid), lc = lam_c(tid);
            wide = (l0 - lp) > kGuard || (lp - lc) > kGuard;
        }
    } else if (!SCALAR) {
        for (int gi = tid; gi < G; gi += NT) {
            const float l0 = lam[gi], lp = lam[PV * G + gi], lc = lam[(CC - 1) * G + gi];
            wide |= (l0 - lp) > kGuard || (lp - lc) > kGuard;
        }
    }
    wide = __syncthreads_or(wide ? 1 : 0) != 0;
    if (!SCALAR && !wide) {
        for (int i = tid; i < DK; i += NT) {
            const float lp = lam_p(i), lc = lam_c(i);
            piv[i] = __expf(lp);
            piv[DK + i] = __expf(lc - lp);
        }
        __syncthreads();
    }
    failed = wait_bar(0, 0) || failed;

    const bool ext = a.kind == REC_EXT;
    if (!failed && ext) {
        float *fo = reinterpret_cast<float *>(img_T + ext_f(DK));
        for (int i = tid; i < DK; i += NT)
            fo[i] = __expf(lam_c(i));   // F = e^{Lambda_C}
    }
    // Scalar gate: e^{Lambda_t - Lambda_j} = e^{Lambda_t - Lambda_p} e^{Lambda_p - Lambda_j} with
    // the pivot p in the middle of the chunk; while the chunk's decay span is within
    // 2 kGuard both factors stay below e^{kGuard}.  The row and column factors go to
    // the inverse's scratch (free until the inverse), read back with the Gram.
    const bool sc_piv = SCALAR && (lam[0] - lam[CC - 1]) <= 2.f * kGuard;
    if (!failed && sc_piv)
        for (int t = tid; t < CC; t += NT) {
            Tf[t] = __expf(lam[t] - lam[CC / 2]);
            Tf[CC + t] = __expf(lam[CC / 2] - lam[t]);
        }
    if (!failed && a.kind == REC_SCALAR) {   // per-token factors of the scalar gate
        float *ea = reinterpret_cast<float *>(img_T + SC_EA);
        float *eb = reinterpret_cast<float *>(img_T + SC_EB);
        const float lc = lam[CC - 1];
        for (int t = tid; t < CC; t += NT) {
            ea[t] = __expf(lam[t]);
            eb[t] = __expf(lc - lam[t]);
        }
        if (tid < 4)
            reinterpret_cast<float *>(img_T + SC_F)[tid] = __expf(lc);
    }
    // decayed operands for the state pass straight from the raw tiles (wide chunks):
    // Qbar = q e^{Lambda_t}, Khat = k e^{Lambda_C - Lambda_t} at row t, channels i0 .. i0 + 7
    auto raw_operands = [&](int t, int i0, const float *lt, const float *lc) {
        float qv[8], kv[8], qb[8], kh8[8];
        ld_tile8(QK, 128, t, i0, qv);
        ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            qb[e] = qv[e] * __expf(lt[e]);
            kh8[e] = kv[e] * __expf(lc[e] - lt[e]);
        }
        const uint32_t off = (i0 >> 6) * IMG + t * 128 + ((((i0 >> 3) & 7) ^ (t & 7)) << 4);
        *reinterpret_cast<uint4 *>(img_T + ext_qb(DK) + off) =
            make_uint4(pack_bf16(qb[0], qb[1]), pack_bf16(qb[2], qb[3]), pack_bf16(qb[4], qb[5]),
                       pack_bf16(qb[6], qb[7]));
        *reinterpret_cast<uint4 *>(img_T + ext_kh(DK) + off) =
            make_uint4(pack_bf16(kh8[0], kh8[1]), pack_bf16(kh8[2], kh8[3]),
                       pack_bf16(kh8[4], kh8[5]), pack_bf16(kh8[6], kh8[7]));
    };
    if (!RL && !failed && ext && wide)   // (RL: after the rounds, whose fp32 rows may need the area)
        for (int u = tid; u < CC * (DK / 8); u += NT) {
            const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
            float lt[8], lc[8];
            lam8(lam, G, wsh, t, i0, lt);
            lam8(lam, G, wsh, CC - 1, i0, lc);
            raw_operands(t, i0, lt, lc);
        }

    if (!failed && !wide) {
        if (!SCALAR) {
            // ---- one pivot p in the middle of the chunk: rows carry a_t = e^{Lambda_t - Lambda_p},
            //      columns b_j = e^{Lambda_p - Lambda_j} (each at most e^{kGuard}); the state
            //      pass's operands from the same two exponentials, Qbar = q a e^{Lambda_p} and
            //      Khat = k b e^{Lambda_C - Lambda_p}; the k rows keep k a (Kbar = k a e^{Lambda_p}
            //      is W's operand, its per-channel factor applied on the way out of TMEM)
            // fq, fk: e^{Lambda_p} and e^{Lambda_C - Lambda_p} at the eight channels
            auto item = [&](int t, int i0, const float *lt, const float *lp, const float *fq,
                            const float *fk) {
                float qv[8], kv[8], kc[8], kh8[8], qb[8];
                ld_tile8(QK, 128, t, i0, qv);
                ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float a = __expf(lt[e] - lp[e]), b = __expf(lp[e] - lt[e]);
                    qv[e] *= a;
                    kc[e] = kv[e] * b;
                    kv[e] *= a;
                    qb[e] = qv[e] * fq[e];
                    kh8[e] = kc[e] * fk[e];
                }
                st_tile8(QK, 128, t, i0, qv);
                st_tile8(QK, 128, 64 + t, i0, kv);
                st_tile8(KC, 64, t, i0, kc);
                if (ext) {
                    const uint32_t off = (i0 >> 6) * IMG + t * 128 + ((((i0 >> 3) & 7) ^ (t & 7)) << 4);
                    st_global_v4(img_T + ext_qb(DK) + off, pack_bf16(qb[0], qb[1]), pack_bf16(qb[2], qb[3]),
                                 pack_bf16(qb[4], qb[5]), pack_bf16(qb[6], qb[7]));
                    st_global_v4(img_T + ext_kh(DK) + off, pack_bf16(kh8[0], kh8[1]),
                                 pack_bf16(kh8[2], kh8[3]), pack_bf16(kh8[4], kh8[5]),
                                 pack_bf16(kh8[6], kh8[7]));
                }
            };
            if constexpr (RL) {
                // the thread's eight channels are the same for its four tokens: the
                // pivot's Lambda and the two per-channel factors are loaded once
                float lp[8], fq[8], fk[8];
                ld8f(lam + LR_P * DK + i0r, lp);
                ld8f(piv + i0r, fq);
                ld8f(piv + DK + i0r, fk);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    item(4 * tb + k, i0r, lv[k], lp, fq, fk);
            } else {
                for (int u = tid; u < CC * (DK / 8); u += NT) {
                    const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
                    float lt[8], lp[8], fq[8], fk[8];
                    lam8(lam, G, wsh, t, i0, lt);
                    lam8(lam, G, wsh, PV, i0, lp);
                    ld8f(piv + i0, fq);
                    ld8f(piv + DK + i0, fk);
                    item(t, i0, lt, lp, fq, fk);
                }
            }
            fence_proxy_async_smem();
            __syncthreads();
        }
        // ---- [Q; K] K^T (M = 128, N = 64, K = dk); for the scalar gate the decay and
        //      beta are applied on the way out, for the others beta only
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, CC, false, false);
            for (int k0 = 0; k0 < DK; k0 += 16)
                mma_bf16(tmem, desc_kmajor(QK, 128, 0, k0),
                         SCALAR ? desc_kmajor(QK, 128, 64, k0) : desc_kmajor(KC, 64, 0, k0), id, k0 > 0);
            mma_commit(&bars[1]);
        }
        failed = wait_bar(1, ph_mma);
        ph_mma ^= 1u;
        if (!failed) {
            tc_fence_after();
            const int R = 32 * (warp & 3) + lane, half = warp >> 2, j0 = 32 * half;
            float g0[16], g1[16];
            tmem_ld16(tq + j0, g0);
            tmem_ld16(tq + j0 + 16, g1);
            tmem_ld_wait();
            const bool qrow = R < CC;
            const int t = qrow ? R : R - CC;
            const float lt = SCALAR ? lam[t] : 0.f;   // (scalar gate: G = 1)
            // two halves of 16 columns (fewer live registers)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int jh = j0 + 16 * h;
                const bool with_beta = !qrow && !a.pair;   // pairs: the raw Gram, beta applied before the inverse
                float bj[16];   // (grouped / per-channel gates: beta of the 16 columns at once)
                if (!SCALAR && with_beta) {
                    ld8f(sbeta + jh, bj);
                    ld8f(sbeta + jh + 8, bj + 8);
                }
                float out[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j = jh + u;
                    const float d = h == 0 ? g0[u] : g1[u];
                    const bool keep = qrow ? (j <= t) : (j < t);
                    float v = 0.f;
                    if (keep)
                        v = !SCALAR ? d : sc_piv ? d * (Tf[t] * Tf[CC + j]) : d * __expf(lt - lam[j]);
                    if (with_beta)
                        v *= SCALAR ? sbeta[j] : bj[u];
                    out[u] = v;
                }
                if (qrow) {
                    st_tile8(Ls, 64, t, jh, &out[0]);
                    st_tile8(Ls, 64, t, jh + 8, &out[8]);
                } else {
                    // Mf holds the k rows' products in fp32
#pragma unroll
                    for (int u = 0; u < 16; u += 4)
                        *reinterpret_cast<float4 *>(&Mf[t * LDM + jh + u]) =
                            make_float4(out[u], out[u + 1], out[u + 2], out[u + 3]);
                }
            }
        }
    } else if (!failed) {
        // ---- two row blocks of 32 tokens, each pivoted at its middle row p = 32r + 16:
        //      rows t of the block carry e^{Lambda_t - Lambda_p}, columns j <= end of the
        //      block carry e^{Lambda_p - Lambda_j}; growth is bounded by a 16-token span
        // RL: Lambda goes to the record's T / L / W area (written after this path: L leaves
        // from its staging tile, T and W after the inverse) and is read back from there, so
        // that the common path keeps no registers for it
        const float *lsc = reinterpret_cast<const float *>(img_T);
        auto lam_row = [&](int t, float *o) {   // this thread's eight channels of row t
            const float4 a0 = *reinterpret_cast<const float4 *>(lsc + t * DK + i0r);
            const float4 a1 = *reinterpret_cast<const float4 *>(lsc + t * DK + i0r + 4);
            o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
            o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
        };
        if constexpr (RL) {
            float *lw = reinterpret_cast<float *>(img_T);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float *dst = lw + (4 * tb + k) * DK + i0r;
                *reinterpret_cast<float4 *>(dst) = make_float4(lv[k][0], lv[k][1], lv[k][2], lv[k][3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(lv[k][4], lv[k][5], lv[k][6], lv[k][7]);
            }
            __syncthreads();
        }
        for (int r = 0; r < 2 && !failed; ++r) {
            const int p0 = 32 * r, pv = p0 + 16, n_r = 32 * (r + 1);
            bool clamp = false;
            // rows 0-31 of RA: q of the block, 32-63: k of the block; the q and k rows of
            // a token share their factors.  Row operand of token t: factor e^{la - lb}
            // with (la, lb) = (Lambda_t, Lambda_p); column operand of token jj:
            // (Lambda_p, Lambda_jj).
            auto operand = [&](bool rowop, int t, int i0, const float *la, const float *lb) {
                float f8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float x = la[e] - lb[e];
                    if (x > kGuard) {
                        x = kGuard;
                        clamp = true;
                    }
                    f8[e] = __expf(x);
                }
                if (rowop) {
                    float q8[8], k8[8];
                    ld_tile8(QK, 128, t, i0, q8);
                    ld_tile8(QK, 128, 64 + t, i0, k8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        q8[e] *= f8[e];
                        k8[e] *= f8[e];
                    }
                    st_tile8(RA, 64, t - p0, i0, q8);
                    st_tile8(RA, 64, 32 + t - p0, i0, k8);
                } else {
                    float k8[8];
                    ld_tile8(QK, 128, 64 + t, i0, k8);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        k8[e] *= f8[e];
                    st_tile8(KC, 64, t, i0, k8);
                }
            };
            if constexpr (RL) {
                float lp[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    lp[e] = lam[(r == 0 ? LR_16 : LR_48) * DK + i0r + e];
#pragma unroll 1
                for (int k = 0; k < 4; ++k) {
                    const int t = 4 * tb + k;
                    float lt[8];
                    lam_row(t, lt);
                    if (t >= p0 && t < p0 + 32)
                        operand(true, t, i0r, lt, lp);
                    if (t < n_r)
                        operand(false, t, i0r, lp, lt);
                }
            } else {
                for (int u = tid; u < (32 + n_r) * (DK / 8); u += NT) {
                    const int row = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
                    float la[8], lb[8];
                    const bool rowop = row < 32;
                    const int t = rowop ? p0 + row : row - 32;
                    lam8(lam, G, wsh, rowop ? t : pv, i0, la);
                    lam8(lam, G, wsh, rowop ? pv : t, i0, lb);
                    operand(rowop, t, i0, la, lb);
                }
            }
            if (clamp)
                flag[r] = 1;
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(64, n_r, false, false);
                for (int k0 = 0; k0 < DK; k0 += 16)
                    mma_bf16(tmem + 32 * r, desc_kmajor(RA, 64, 0, k0), desc_kmajor(KC, 64, 0, k0), id,
                             k0 > 0);
                mma_commit(&bars[1]);
            }
            failed = wait_bar(1, ph_mma);
            ph_mma ^= 1u;
        }
        if (!failed) {
            tc_fence_after();
            // M = 64 accumulator: row m at lane 32 (m / 16) + m % 16.  Block rows of q
            // (m < 32) are in quarters 0-1, of k in quarters 2-3; row t = 32r + 16 (q & 1)
            // + lane.  Each warp takes half of the round's columns; Mf aliases the round tiles.
            const int q4 = warp & 3, half = warp >> 2;
            const bool qrow = q4 < 2;
            for (int r = 0; r < 2; ++r) {
                const int n_r = 32 * (r + 1), w = n_r / 2, c0 = half * w;
                const int t = 32 * r + 16 * (q4 & 1) + (lane & 15);
                for (int cb = 0; cb < w; cb += 16) {
                    float d[16];
                    tmem_ld16(tq + 32 * r + c0 + cb, d);
                    tmem_ld_wait();
                    if (lane < 16) {
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int jj = c0 + cb + e;
                            v[e] = qrow ? ((jj <= t) ? d[e] : 0.f)
                                        : ((jj < t) ? (a.pair ? d[e] : sbeta[jj] * d[e]) : 0.f);
                        }
                        if (qrow) {
                            st_tile8(Ls, 64, t, c0 + cb, &v[0]);
                            st_tile8(Ls, 64, t, c0 + cb + 8, &v[8]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; e += 4)
                                *reinterpret_cast<float4 *>(&Mf[t * LDM + c0 + cb + e]) =
                                    make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                        }
                    }
                }
                if (r == 0 && lane < 16) {   // columns 32-63 of block 0's rows: above the diagonal
                    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    const int zc = 32 + 16 * half;
                    if (qrow) {
                        st_tile8(Ls, 64, t, zc, z);
                        st_tile8(Ls, 64, t, zc + 8, z);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<float4 *>(&Mf[t * LDM + zc + e]) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
            __syncthreads();
            // blocks whose decay span overran the guard: exact fp32 rows from the raw tiles
            // (RL: Lambda from the record)
            for (int r = 0; r < 2; ++r) {
                if (!flag[r])
                    continue;
                for (int u = tid; u < 32 * 8; u += NT) {
                    const int t = 32 * r + (u >> 3), j0 = (u & 7) * 8;
                    float lv2[8], mv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        lv2[e] = mv[e] = 0.f;
                    for (int i0 = 0; i0 < DK; i0 += 8) {
                        float qt[8], kt[8];
                        ld_tile8(QK, 128, t, i0, qt);
                        ld_tile8(QK, 128, 64 + t, i0, kt);
                        for (int e = 0; e < 8; ++e) {
                            const int j = j0 + e;
                            if (j > t)
                                break;
                            float kj[8];
                            ld_tile8(QK, 128, 64 + j, i0, kj);
#pragma unroll
                            for (int f = 0; f < 8; ++f) {
                                const int gi = (i0 + f) >> wsh;
                                const float dcy = RL ? __expf(lsc[t * DK + i0 + f] - lsc[j * DK + i0 + f])
                                                     : __expf(lam[t * G + gi] - lam[j * G + gi]);
                                lv2[e] += qt[f] * kj[f] * dcy;
                                mv[e] += kt[f] * kj[f] * dcy;
                            }
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = j0 + e;
                        mv[e] = (j < t) ? (a.pair ? mv[e] : sbeta[j] * mv[e]) : 0.f;
                        lv2[e] = (j <= t) ? lv2[e] : 0.f;
                        Mf[t * LDM + j] = mv[e];
                    }
                    st_tile8(Ls, 64, t, j0, lv2);
                }
            }
            if constexpr (RL) {
                // the state pass's decayed operands and Kbar = k e^{Lambda_t} in place in the
                // raw k rows (every fp32 row has read them: the barrier), the same rows the same
                // thread reads for the operands
                __syncthreads();
                float lc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    lc[e] = lam[LR_C * DK + i0r + e];
#pragma unroll 1
                for (int k = 0; k < 4; ++k) {
                    const int t = 4 * tb + k;
                    float lt[8];
                    lam_row(t, lt);
                    raw_operands(t, i0r, lt, lc);
                    float kv[8];
                    ld_tile8(QK, 128, 64 + t, i0r, kv);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        kv[e] *= __expf(lt[e]);
                    st_tile8(QK, 128, 64 + t, i0r, kv);
                }
            }
        }
    }
    if (!failed) {   // L leaves in one bulk copy
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_store(img_L, Ls, IMG);
            bulk_commit();
        }
    }
    if (!RL && !failed && a.kind != REC_PLAIN && !SCALAR && wide) {
        // Kbar = k e^{Lambda_t} in place in the raw k rows of the pivoted blocks, before the
        // inverse: the last use of Lambda there, whose tile then holds the Neumann operands
        // (RL: at the end of the pivoted blocks' path)
        __syncthreads();
        auto kbar = [&](int t, int i0, const float *lt) {
            float kv[8];
            ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                kv[e] *= __expf(lt[e]);
            st_tile8(QK, 128, 64 + t, i0, kv);
        };
        for (int u = tid; u < CC * (DK / 8); u += NT) {
            const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
            float lt[8];
            lam8(lam, G, wsh, t, i0, lt);
            kbar(t, i0, lt);
        }
    }
    if (!failed && a.pair) {
        // Mf holds the decayed Gram of the k rows (strictly lower): the pair kernel's
        // Ntil = diag(beta) Gram (beta on the rows) as an image, then M = Gram diag(beta)
        __syncthreads();
        uint8_t *img_N = img_T + a.base_bytes + PAIR_N;
        for (int u = tid; u < CC * 8; u += NT) {
            const int t = u >> 3, j0 = (u & 7) * 8;
            float nv[8], mv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gr = Mf[t * LDM + j0 + e];
                nv[e] = sbeta[t] * gr;
                mv[e] = gr * sbeta[j0 + e];
            }
            st_img8(img_N, t, j0, nv);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                Mf[t * LDM + j0 + e] = mv[e];
        }
    }
    // A chunk-128 Neumann pair (grouped / per-channel records, dk = 128) leaves its halves'
    // T and W to the pair kernel, which holds both halves' own factors as the diagonal
    // blocks of its 128-token one; an unpaired last half computes its own.
    const bool defer = DK == 128 && a.pair && (neu || p.neumann1) && ext && ((c & 1) || c + 1 < a.nchunks);
    if (!failed && !defer) {
        if (tid == 0 && (SCALAR || (RL && neu)))   // T or the Neumann operands land on L's staging
            bulk_wait_read();
        __syncthreads();
        if (!neu) {
            if (p.neumann1)
                gen::block_neumann1_64_inplace(Mf, Tf, tid);
            else
                gen::inverse64_mid(Mf, Tf, tid);
        } else {
            // ---- truncated Neumann series (Horner) + Newton residual steps, M = 64 on tcgen05
            const uint32_t NB = base_u32 + Ly.NB, XB = base_u32 + Ly.XB, RB = base_u32 + Ly.RB;
            const uint32_t tn = tmem + Ly.tn, tqn = tq + Ly.tn;
            for (int u = tid; u < CC * 8; u += NT) {
                const int t = u >> 3, j = (u & 7) * 8;
                float v8[8], x8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v8[e] = Mf[t * LDM + j + e];
                    x8[e] = (t == j + e) ? 1.f : 0.f;
                }
                st_tile8(NB, 64, t, j, v8);
                st_tile8(XB, 64, t, j, x8);
            }
            fence_proxy_async_smem();
            __syncthreads();
            const int rr = gen::row64g(warp, lane);
            const int cb = 32 * (warp >> 2);
            const uint32_t id = idesc_bf16(64, 64, false, true);
            auto product = [&](uint32_t a_tile, uint32_t b_tile) {   // tn = A (K-major) * B (MN-major)
                if (tid == 0) {
                    tc_fence_after();
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tn, desc_kmajor(a_tile, 64, 0, k0), desc_mnmajor(b_tile, 64, k0, 0), id,
                                 k0 > 0);
                    mma_commit(&bars[1]);
                }
                const bool f = wait_bar(1, ph_mma);
                ph_mma ^= 1u;
                return f;
            };
            for (int pw = 1; pw <= p.neu_order && !failed; ++pw) {
                if ((failed = product(NB, XB)))
                    break;
                tc_fence_after();
                float d0[16], d1[16];
                tmem_ld16(tqn + cb, d0);
                tmem_ld16(tqn + cb + 16, d1);
                tmem_ld_wait();
                if (rr >= 0) {
                    float x[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        x[u] = ((rr == cb + u) ? 1.f : 0.f) - (u < 16 ? d0[u] : d1[u - 16]);
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(XB, 64, rr, cb + u, &x[u]);
                    if (pw == p.neu_order)
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            Mf[rr * LDM + cb + u] = x[u];
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
            }
            if (!failed && p.neu_order == 0) {
                for (int u = tid; u < CC * CC; u += NT)
                    Mf[(u / CC) * LDM + (u % CC)] = ((u / CC) == (u % CC)) ? 1.f : 0.f;
                __syncthreads();
            }
            // Newton: Rm = I - X - N X ; X <- X + X Rm
            for (int st = 0; st < p.neu_resid && !failed; ++st) {
                if ((failed = product(NB, XB)))
                    break;
                tc_fence_after();
                float d0[16], d1[16];
                tmem_ld16(tqn + cb, d0);
                tmem_ld16(tqn + cb + 16, d1);
                tmem_ld_wait();
                if (rr >= 0) {
                    float rm[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        rm[u] = ((rr == cb + u) ? 1.f : 0.f) - Mf[rr * LDM + cb + u] -
                                (u < 16 ? d0[u] : d1[u - 16]);
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(RB, 64, rr, cb + u, &rm[u]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                if ((failed = product(XB, RB)))
                    break;
                tc_fence_after();
                tmem_ld16(tqn + cb, d0);
                tmem_ld16(tqn + cb + 16, d1);
                tmem_ld_wait();
                if (rr >= 0) {
                    float x[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        x[u] = Mf[rr * LDM + cb + u] + (u < 16 ? d0[u] : d1[u - 16]);
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        Mf[rr * LDM + cb + u] = x[u];
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(XB, 64, rr, cb + u, &x[u]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
            }
        }
    }
    const bool with_w = a.kind != REC_PLAIN;
    if (!failed) {
        __syncthreads();
        // After the middle pivot the k rows hold k e^{Lambda_t - Lambda_p}: W is then
        // (T that) diag(e^{Lambda_p}), the column factors applied on the way out of TMEM
        // (copied into the inverse's scratch, free by now).
        const bool w_cols = with_w && !SCALAR && !wide;
        if (w_cols)
            for (int i = tid; i < DK; i += NT)
                Tf[i] = piv[i];
        if (a.pair && !SCALAR) {
            // Kbar = k e^{Lambda_t} for the pair kernel: the k rows hold it after the
            // pivoted blocks; after the chunk-end pivot they hold k e^{Lambda_t - Lambda_C}
            __syncthreads();
            uint8_t *img_K = img_T + a.base_bytes + PAIR_KB;
            for (int u = tid; u < CC * (DK / 8); u += NT) {
                const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
                float kv[8];
                ld_tile8(QK, 128, 64 + t, i0, kv);
                if (w_cols)   // Tf holds e^{Lambda_p} per channel here
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        kv[e] *= Tf[i0 + e];
                st_img8(img_K + (i0 >> 6) * IMG, t, i0 & 63, kv);
            }
        }
        if (SCALAR && with_w) {   // e^{Lambda_j} for W's operand, once per token
            for (int t = tid; t < CC; t += NT)
                Tf[2 * CC + t] = __expf(lam[t]);
            __syncthreads();
        }
        // ---- T = diag(beta) A as a tile image: thread u writes 16-byte chunk u (coalesced).
        //      For W the same chunk goes to the bf16 operand tile in the dead q rows,
        //      scaled by e^{Lambda_j} for the scalar gate (W = T diag(e^Lambda) K).
        const uint32_t TB = base_u32 + Ly.TB;
        for (int u = tid; u < (defer ? 0 : CC * 8); u += NT) {
            const int r = u >> 3, cc = (u & 7) ^ (r & 7);
            const float bt = sbeta[r];
            const float4 x0 = *reinterpret_cast<const float4 *>(&Mf[r * LDM + 8 * cc]);
            const float4 x1 = *reinterpret_cast<const float4 *>(&Mf[r * LDM + 8 * cc + 4]);
            const uint4 tv =
                make_uint4(pack_bf16(bt * x0.x, bt * x0.y), pack_bf16(bt * x0.z, bt * x0.w),
                           pack_bf16(bt * x1.x, bt * x1.y), pack_bf16(bt * x1.z, bt * x1.w));
            *reinterpret_cast<uint4 *>(img_T + 16 * u) = tv;
            if (with_w) {
                if (SCALAR) {
                    float e[8];
#pragma unroll
                    for (int f = 0; f < 8; ++f)
                        e[f] = bt * Tf[2 * CC + 8 * cc + f];
                    st_shared_v4(TB + 16 * u, pack_bf16(e[0] * x0.x, e[1] * x0.y),
                                 pack_bf16(e[2] * x0.z, e[3] * x0.w), pack_bf16(e[4] * x1.x, e[5] * x1.y),
                                 pack_bf16(e[6] * x1.z, e[7] * x1.w));
                } else {
                    st_shared_v4(TB + 16 * u, tv.x, tv.y, tv.z, tv.w);
                }
            }
        }
        if (with_w && !defer) {
            // ---- W = TB Kbar (M = 64, N = dk, K = 64) on tcgen05, read back as an image
            fence_proxy_async_smem();
            if (tid == 0 && DK > 128)   // W's staging is L's
                bulk_wait_read();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(64, DK, false, true);
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem, desc_kmajor(TB, 64, 0, k0), desc_mnmajor(QK, 128, 64 + k0, 0), id,
                             k0 > 0);
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
                    tmem_ld16(tq + cw + cb, w0);
                    tmem_ld16(tq + cw + cb + 16, w1);
                    tmem_ld_wait();
                    if (rr >= 0) {
                        if (w_cols) {
#pragma unroll
                            for (int e0 = 0; e0 < 16; e0 += 8) {
                                float f0[8], f1[8];
                                ld8f(Tf + cw + cb + e0, f0);
                                ld8f(Tf + cw + cb + 16 + e0, f1);
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    w0[e0 + e] *= f0[e];
                                    w1[e0 + e] *= f1[e];
                                }
                            }
                        }
                        if (a.neg_w) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                w0[e] = -w0[e];
                                w1[e] = -w1[e];
                            }
                        }
                        const int col = cw + cb;   // 32 columns inside one 64-column image
                        if constexpr (W_STAGE) {
                            const uint32_t wi = Ws + (col >> 6) * IMG;
                            st_tile8(wi, 64, rr, col & 63, &w0[0]);
                            st_tile8(wi, 64, rr, (col & 63) + 8, &w0[8]);
                            st_tile8(wi, 64, rr, (col & 63) + 16, &w1[0]);
                            st_tile8(wi, 64, rr, (col & 63) + 24, &w1[8]);
                        } else {
                            uint8_t *img_W = img_T + REC_W + (col >> 6) * IMG;
                            st_img8(img_W, rr, col & 63, &w0[0]);
                            st_img8(img_W, rr, (col & 63) + 8, &w0[8]);
                            st_img8(img_W, rr, (col & 63) + 16, &w1[0]);
                            st_img8(img_W, rr, (col & 63) + 24, &w1[8]);
                        }
                    }
                }
                if constexpr (W_STAGE) {   // W leaves in one bulk copy
                    fence_proxy_async_smem();
                    __syncthreads();
                    if (tid == 0) {
                        bulk_store(img_T + REC_W, Ws, (DK / 64) * IMG);
                        bulk_commit();
                    }
                }
            }
        }
    }
    // shared memory must outlive the bulk copies' reads of it
    if (tid == 0)
        bulk_wait_read();
    // drain: whatever was started must finish before tensor memory is released (bounded)
    if (tid == 0 && failed) {
        mma_commit(&bars[1]);
        mbar_wait(&bars[1], ph_mma, 200000000ull);
        mbar_wait(&bars[0], 0, 200000000ull);
        if (g_bulk)
            mbar_wait(&bars[2], 0, 200000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Ly.tmem_cols);
    }
}

inline int nchunks(const Params &p) { return (p.T + CC - 1) / CC; }

inline size_t bytes(const Params &p)
{
    return (size_t)p.B * p.Hk * nchunks(p) * CHUNK_BYTES;
}

// Record of the two-pass path's workspace.
inline int record_kind(const Params &p) { return p.G > 1 ? REC_EXT : REC_SCALAR; }

inline uint32_t kind_bytes(int kind, int dk = 128)
{
    return kind == REC_EXT ? ext_bytes(dk) : (kind == REC_SCALAR ? SC_BYTES : CHUNK_BYTES);
}

inline uint32_t rec_bytes(const Params &p)
{
    return kind_bytes(record_kind(p), p.dk) + (p.pair ? pair_extra(record_kind(p), p.dk) : 0u);
}

inline size_t ws_bytes(const Params &p) { return (size_t)p.B * p.Hk * nchunks(p) * rec_bytes(p); }

inline bool supports(const Params &p)
{
    return p.in_bf16 && p.C == CC && (p.dk == 128 || p.dk == 256) && p.G >= 1 &&
           p.G <= gmax(p.dk) && p.Hk <= 65535 && p.B <= 65535;
}

template <int DK>
int launch(const Params &p, void *out, int kind, cudaStream_t stream, int pair = 0, int neg_w = 0)
{
    const int N = nchunks(p);
    if (N == 0 || p.B == 0)
        return 0;
    CUtensorMap mq, mk;
    const long sk = (long)p.B * p.Hk;
    if (!make_map(&mq, p.q, DK, p.T, sk, CC) || !make_map(&mk, p.k, DK, p.T, sk, CC))
        return 6;
    // Lambda in registers where it pays (per-channel / grouped gates at dk = 128 with the
    // state pass's records: its fp32 rows use the record as scratch)
    const bool rl = DK == 128 && p.G > 1 && kind == REC_EXT;
    const Plan Ly = plan(DK, p.G, p.neumann != 0, rl);
    auto kern = p.G == 1 ? prep_kernel<DK, true> : rl ? prep_kernel<DK, false, DK == 128> : prep_kernel<DK, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return 6;
    PrepArgs a;
    a.p = p;
    a.out = static_cast<uint8_t *>(out);
    a.nchunks = N;
    a.kind = kind;
    a.base_bytes = kind_bytes(kind, DK);
    a.pair = pair;
    a.neg_w = neg_w;
    a.rec_bytes = a.base_bytes + (pair ? pair_extra(kind, DK) : 0u);
    dim3 grid(N, p.Hk, p.B);
    kern<<<grid, NT, Ly.total, stream>>>(mq, mk, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace prep
