// gdr_tc_gen.cuh -- tensor-core kernel for grouped and per-channel decay
// (G = dk/64 or dk), key width 128 or 256, chunk C = 64, exact or truncated
// Neumann chunk inverse.  Included by gdr_tc.cu.
//
// One CTA (256 threads) owns one (batch, value head, 64 value columns) and runs
// the chunk steps in order ("Systolic Linear Attention: Co-Designing
// Tile-Grouped Gated Delta Attention for TPUs", §2.1, §2.3 Table 2, §2.4.2):
//   1. TMA: q, k (as one [q; k] block of 128 rows), v and (for G >= 4) the
//      chunk's log-gates, zero-filled past T; beta (and the gates when G < 4)
//      are prefetched a chunk ahead through registers, zero past T.  Zero gates
//      and beta leave the recurrence untouched.
//   2. Lambda = cumsum g per decay group.  Decayed operands in place, with the
//      chunk boundaries as pivots (no division by a decay prefix):
//        Khat = k e^{Lambda_C - Lambda_t} (<= 1), and for the Gram
//        Kr = k e^{Lambda_t - Lambda_C}, Qr = q e^{Lambda_t - Lambda_C}, whose
//      factor is bounded by e^{-Lambda_C}; the kernel uses this single-MMA Gram
//      only while max_i(-Lambda_C,i) <= 60, and otherwise forms the chunk's
//      Gram exactly in fp32 from exp(Lambda_t - Lambda_j) (t >= j).
//   3. tcgen05: [Qr; Kr] Khat^T -> L (rows 0-63) and M (rows 64-127, beta_j).
//   4. A = (I + M)^{-1}: exact fp32 block doubling in place (16 x 16 diagonal
//      blocks, merges X21 = -X22 M21 X11), or the truncated Neumann series by
//      Horner's rule plus Newton residual steps, both products on tcgen05
//      ("When Good Enough Is Optimal: Multiplication-Only Matrix Inversion
//      Approximation for Quantized Gated DeltaNet", Lemma 3.1, §4.1).
//   5. Kbar = Kr e^{Lambda_C} = k e^{Lambda_t}, Qbar likewise (in place).
//   6. tcgen05: [Qbar; Kbar] S -> Q S, Kbar S;  RHS = V - Kbar S (bf16).
//   7. tcgen05: E = diag(beta) A RHS   (= U - W S of Table 2).
//   8. tcgen05: dS = Khat^T E, O = Qbar S + L E;  S <- diag(e^{Lambda_C}) S + dS.

namespace gen {

constexpr int NT = 256;
constexpr int CC = 64;
constexpr int NVC = 64;
constexpr int LDM = 68;
constexpr float kGrowthLimit = 60.f;

// Widest gate tile per key width: G <= 128 for dk = 128 (per channel); for
// dk = 256 only the scalar and 64-channel-tile gates (G <= 4) run here.
__host__ __device__ constexpr int gmax(int dk) { return dk == 256 ? 8 : 128; }

constexpr uint32_t T_G = 0;      // [Qr;Kr] Khat^T : rows 0-63 L', 64-127 M'
constexpr uint32_t T_Y = 64;     // [Qbar;Kbar] S : rows 0-63 QS (+ L E), 64-127 Kbar S
constexpr uint32_t T_E = 128;    // [Ab;0] RHS : rows 0-63 E
constexpr uint32_t T_N = 192;    // Neumann products (M = 64)
constexpr uint32_t T_DS = 256;   // dS, 64 columns per 128 key channels
constexpr uint32_t TMEM_COLS = 512;

enum Bar { TMA_QK, TMA_V, TMA_G, MMA, NBARS };

template <int DK>
struct Plan {
    uint32_t QK, KH, V, S, L, AB, RHS, E, gates, beta, Mf, Tf, fac, bar, misc, total;
};

template <int DK>
__host__ __device__ inline Plan<DK> plan()
{
    Plan<DK> s;
    uint32_t o = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t at = o;
        o += (bytes + 1023u) & ~1023u;
        return at;
    };
    s.QK = take((DK / 64) * 128 * 128);   // rows 0-63 q, 64-127 k
    s.KH = take((DK / 64) * 64 * 128);
    s.V = take(64 * 128);
    s.S = take(DK * 128);
    s.L = take(128 * 128);                // rows 64-127 stay zero
    s.AB = take(128 * 128);               // rows 64-127 stay zero
    s.RHS = take(64 * 128);
    s.E = take(64 * 128);
    s.gates = take(CC * gmax(DK) * 4);    // C x G fp32
    s.beta = take(CC * 4 + 2 * DK * 4);   // beta, then Lambda_C and e^{Lambda_C} per channel
    s.Mf = take(CC * LDM * 4);
    s.Tf = take(32 * 36 * 4);
    s.fac = take(2 * CC * 8 * 4);         // per (t, group) factors when G <= 8
    s.bar = take(NBARS * 8 + 16);
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

struct GenArgs {
    Params p;
    int nvt;
    int g_flat;                           // G < 4: gates prefetched through registers
};

// Row of an M = 64 accumulator held by this thread (lanes 0-15 of each quarter).
__device__ __forceinline__ int row64g(int warp, int lane) { return lane < 16 ? 16 * (warp & 3) + lane : -1; }

// acc[i][n] = sum over l in [l0, K) of A[i * a_step + l] * B[l * ldb + n], n < 4: a 4 x 4
// block of a product, the inner index in ascending order.
template <int K>
__device__ __forceinline__ void block_product4x4(float (&acc)[4][4], const float *A, int a_step,
                                                 const float *B, int ldb, int l0)
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int n = 0; n < 4; ++n)
            acc[i][n] = 0.f;
#pragma unroll 4
    for (int l = l0; l < K; ++l) {
        float a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            a[i] = A[i * a_step + l];
        const float4 b = *reinterpret_cast<const float4 *>(B + l * ldb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[i][0] += a[i] * b.x;
            acc[i][1] += a[i] * b.y;
            acc[i][2] += a[i] * b.z;
            acc[i][3] += a[i] * b.w;
        }
    }
}

// The four diagonal 16 x 16 blocks of I + M (64 x 64, M strictly lower) replaced
// in place by their exact inverses; the blocks below them are left as they are.
__device__ __forceinline__ void diag16_inverse_inplace(float *Mf, int tid)
{
    // Exact forward substitution, column cc of a block's inverse a thread, in
    // registers.  Right-looking: once x_j is final it is applied to every later row
    // at once, so the dependent chain is 15 steps long (each x_t still sums its
    // terms in the order j = 0, 1, ...).  The columns go back over the blocks once
    // every thread has read them (a barrier, no staging copy).
    const int blk = tid >> 4, cc = tid & 15, o = 16 * blk;
    float x[16];
    if (tid < 64) {
#pragma unroll
        for (int t = 0; t < 16; ++t)
            x[t] = (t == cc) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < 15; ++j) {
            const float xj = x[j];
#pragma unroll
            for (int t = j + 1; t < 16; ++t)
                x[t] -= Mf[(o + t) * LDM + o + j] * xj;
        }
    }
    __syncthreads();
    if (tid < 64)
#pragma unroll
        for (int t = 0; t < 16; ++t)
            Mf[(o + t) * LDM + o + cc] = x[t];
    __syncthreads();
}

// In-place exact inverse of I + M (64 x 64, M strictly lower) by block doubling.
__device__ __forceinline__ void inverse64_inplace(float *Mf, float *Tf, int tid)
{
    diag16_inverse_inplace(Mf, tid);
    // The doubling steps are products of small dense blocks.  Each thread owns a
    // 4 x 4 block of the product: per step of the inner index it loads four A
    // values (shared by the lanes of a row group) and one float4 of B, which is
    // half the shared-memory traffic per FMA of one output row per thread.
    const int warp = tid >> 5, lane = tid & 31;
    // 16 -> 32, pair pr in warp pr (lanes 0-15): T = M21 X11, X21 = -X22 T (16 x 16 blocks)
    if (warp < 2 && lane < 16) {
        const int pr = warp, rg = lane >> 2, c0 = 4 * (lane & 3), o = 32 * pr;
        float acc[4][4];
        block_product4x4<16>(acc, Mf + (o + 16 + rg) * LDM + o, 4 * LDM, Mf + o * LDM + o + c0, LDM, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Tf[(pr * 16 + rg + 4 * i) * 36 + c0]) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        __syncwarp(0x0000ffffu);
        block_product4x4<16>(acc, Mf + (o + 16 + rg) * LDM + o + 16, 4 * LDM, Tf + pr * 16 * 36 + c0, 36, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Mf[(o + 16 + rg + 4 * i) * LDM + o + c0]) =
                make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]);
    }
    __syncthreads();
    // 32 -> 64 on warps 0-1: rows rg + 8i of the 32-row block, columns 16 warp + c0.
    // X11 is lower triangular, so its rows above 16 warp vanish in those columns.
    const int rg = lane >> 2, c0 = 16 * warp + 4 * (lane & 3);
    if (warp < 2) {
        float acc[4][4];
        block_product4x4<32>(acc, Mf + (32 + rg) * LDM, 8 * LDM, Mf + c0, LDM, 16 * warp);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Tf[(rg + 8 * i) * 36 + c0]) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
    __syncthreads();
    if (warp < 2) {
        float acc[4][4];
        block_product4x4<32>(acc, Mf + (32 + rg) * LDM + 32, 8 * LDM, Tf + c0, 36, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Mf[(32 + rg + 8 * i) * LDM + c0]) =
                make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]);
    }
    __syncthreads();
}

// In-place exact inverse of I + M (64 x 64, M strictly lower) by block doubling,
// the merges spread over the CTA: after the exact 16 x 16 diagonal blocks, each
// merge X21 = -X22 (M21 X11) is two small dense products with a loop over the full
// inner index (the zero triangles multiply as zeros, so every lane of a warp runs
// the same trip count).  The 16 -> 32 merges give every output pair its own thread
// (all 256); the 32 -> 64 one runs on warps 0-3, thread (rg, c0) owning rows rg
// and rg + 16 of the 32-row block at columns c0 .. c0 + 3, so each step of the
// inner index loads two values of the left factor and one float4 of the right one
// for eight products: fewer shared-memory wavefronts than one output row a thread
// (what bounds pass 1, several CTAs to an SM), shorter chains than 4 x 4 blocks on
// two warps.  Same arithmetic as inverse64_inplace (inner index ascending, fp32);
// Tf needs 32 x 36 floats.
__device__ __forceinline__ void inverse64_mid(float *Mf, float *Tf, int tid)
{
    diag16_inverse_inplace(Mf, tid);
    {   // 16 -> 32: pair pr (rows 32 pr + 16 .. +31, columns 32 pr .. +15)
        const int pr = tid >> 7, q = tid & 127, r = q >> 3, c0 = (q & 7) * 2, o = 32 * pr;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) {   // T = M21 X11
            const float m = Mf[(o + 16 + r) * LDM + o + l];
            const float2 x = *reinterpret_cast<const float2 *>(&Mf[(o + l) * LDM + o + c0]);
            a0 += m * x.x;
            a1 += m * x.y;
        }
        *reinterpret_cast<float2 *>(&Tf[(16 * pr + r) * 36 + c0]) = make_float2(a0, a1);
        __syncthreads();
        a0 = a1 = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) {   // X21 = -X22 T
            const float x = Mf[(o + 16 + r) * LDM + o + 16 + l];
            const float2 t = *reinterpret_cast<const float2 *>(&Tf[(16 * pr + l) * 36 + c0]);
            a0 += x * t.x;
            a1 += x * t.y;
        }
        *reinterpret_cast<float2 *>(&Mf[(o + 16 + r) * LDM + o + c0]) = make_float2(-a0, -a1);
        __syncthreads();
    }
    // 32 -> 64: rows 32 + rg and 48 + rg, columns c0 .. c0 + 3
    const int rg = (tid >> 3) & 15, c0 = (tid & 7) * 4;
    if (tid < 128) {
        float a[2][4] = {};
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {   // T = M21 X11
            const float m0 = Mf[(32 + rg) * LDM + l], m1 = Mf[(48 + rg) * LDM + l];
            const float4 x = *reinterpret_cast<const float4 *>(&Mf[l * LDM + c0]);
            a[0][0] += m0 * x.x; a[0][1] += m0 * x.y; a[0][2] += m0 * x.z; a[0][3] += m0 * x.w;
            a[1][0] += m1 * x.x; a[1][1] += m1 * x.y; a[1][2] += m1 * x.z; a[1][3] += m1 * x.w;
        }
        *reinterpret_cast<float4 *>(&Tf[rg * 36 + c0]) = make_float4(a[0][0], a[0][1], a[0][2], a[0][3]);
        *reinterpret_cast<float4 *>(&Tf[(rg + 16) * 36 + c0]) = make_float4(a[1][0], a[1][1], a[1][2], a[1][3]);
    }
    __syncthreads();
    if (tid < 128) {
        float a[2][4] = {};
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {   // X21 = -X22 T
            const float x0 = Mf[(32 + rg) * LDM + 32 + l], x1 = Mf[(48 + rg) * LDM + 32 + l];
            const float4 t = *reinterpret_cast<const float4 *>(&Tf[l * 36 + c0]);
            a[0][0] += x0 * t.x; a[0][1] += x0 * t.y; a[0][2] += x0 * t.z; a[0][3] += x0 * t.w;
            a[1][0] += x1 * t.x; a[1][1] += x1 * t.y; a[1][2] += x1 * t.z; a[1][3] += x1 * t.w;
        }
        *reinterpret_cast<float4 *>(&Mf[(32 + rg) * LDM + c0]) =
            make_float4(-a[0][0], -a[0][1], -a[0][2], -a[0][3]);
        *reinterpret_cast<float4 *>(&Mf[(48 + rg) * LDM + c0]) =
            make_float4(-a[1][0], -a[1][1], -a[1][2], -a[1][3]);
    }
    __syncthreads();
}

// In-place 1-Step Neumann approximation of (I + M)^{-1} ("Systolic Linear
// Attention ...", §2.4.3): with D the block-diagonal part of I + M in 16-row
// blocks and N = D^{-1} M_off, A = (I - N) D^{-1}, i.e. the exact inverses D_ii^{-1}
// on the diagonal and A_ij = -D_ii^{-1} M_ij D_jj^{-1} below it (i > j).  The six
// products T_ij = M_ij D_jj^{-1} go to the (zero) block above the diagonal at
// (j, i) first, one 16-thread group per block (4 x 4 outputs a thread).
__device__ __forceinline__ void block_neumann1_64_inplace(float *Mf, float *Tf, int tid)
{
    diag16_inverse_inplace(Mf, tid);
    const int pi = tid >> 4;                      // block pair 0..5 for tid < 96
    const int bi = pi < 1 ? 1 : pi < 3 ? 2 : 3;   // (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
    const int bj = pi < 1 ? 0 : pi < 3 ? pi - 1 : pi - 3;
    const int rg = (tid & 15) >> 2, c0 = 4 * (tid & 3);
    if (tid < 96) {
        float acc[4][4];
        block_product4x4<16>(acc, Mf + (16 * bi + rg) * LDM + 16 * bj, 4 * LDM,
                             Mf + 16 * bj * LDM + 16 * bj + c0, LDM, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Mf[(16 * bj + rg + 4 * i) * LDM + 16 * bi + c0]) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
    __syncthreads();
    if (tid < 96) {
        float acc[4][4];
        block_product4x4<16>(acc, Mf + (16 * bi + rg) * LDM + 16 * bi, 4 * LDM,
                             Mf + 16 * bj * LDM + 16 * bi + c0, LDM, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Mf[(16 * bi + rg + 4 * i) * LDM + 16 * bj + c0]) =
                make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]);
    }
    __syncthreads();
    for (int u = tid; u < 6 * 256; u += NT) {     // the scratch blocks back to zero
        const int q = u >> 8, r = (u >> 4) & 15, c = u & 15;
        const int qi = q < 1 ? 1 : q < 3 ? 2 : 3, qj = q < 1 ? 0 : q < 3 ? q - 1 : q - 3;
        Mf[(16 * qj + r) * LDM + 16 * qi + c] = 0.f;
    }
    __syncthreads();
}

template <int DK, bool OUT_BF16>
__global__ void __launch_bounds__(NT, 1)
gen_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
           const GenArgs args)
{
    using namespace ptx;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const Plan<DK> Ly = plan<DK>();
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t pad = base_u32 - smem_u32(smem_raw);
    uint8_t *base = smem_raw + pad;
    float *gts = reinterpret_cast<float *>(smem_raw + pad + Ly.gates);
    float *sbeta = reinterpret_cast<float *>(smem_raw + pad + Ly.beta);
    float *lamc = sbeta + CC;          // Lambda_C per channel
    float *fch = lamc + DK;            // e^{Lambda_C} per channel
    float *Mf = reinterpret_cast<float *>(smem_raw + pad + Ly.Mf);
    float *Tf = reinterpret_cast<float *>(smem_raw + pad + Ly.Tf);
    float *fac = reinterpret_cast<float *>(smem_raw + pad + Ly.fac);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + pad + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + pad + Ly.misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = blockIdx.x % args.nvt, hv = blockIdx.x / args.nvt, b = blockIdx.y;
    const int hk = hv / p.R, n0 = nt * NVC;
    const long kh = (long)b * p.Hk + hk, vh = (long)b * p.Hv + hv;
    const int T = p.T, G = p.G, width = DK / G;
    const int N = (T + CC - 1) / CC;
    const uint32_t QK = base_u32 + Ly.QK, KH = base_u32 + Ly.KH, VT = base_u32 + Ly.V;
    const uint32_t ST = base_u32 + Ly.S, LT = base_u32 + Ly.L, AB = base_u32 + Ly.AB;
    const uint32_t RT = base_u32 + Ly.RHS, ET = base_u32 + Ly.E;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)
            mbar_init(&bars[i], 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    // zero rows 64-127 of L and [Ab; 0] once (stacked MMA padding)
    for (int i = tid; i < 64 * 8; i += NT) {
        const int r = 64 + (i >> 3), c = (i & 7) * 8;
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        st_tile8(LT, 128, r, c, z);
        st_tile8(AB, 128, r, c, z);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int half = warp >> 2;
    const uint32_t gbytes = (uint32_t)(CC * G * 4);

    // phase parities
    uint32_t ph_qk = 0, ph_v = 0, ph_g = 0, ph_mma = 0;
    uint32_t pend = 0;     // bit per TMA barrier with a load in flight (thread 0's view)
    bool failed = false;
    auto wait_all = [&](int bar, uint32_t &ph) {
        const bool gave_up = !mbar_wait(&bars[bar], ph);
        if (!gave_up) {
            ph ^= 1u;
            if (bar != MMA)
                pend &= ~(1u << bar);
        }
        if (gave_up)
            atomicExch(&g_device_status, kTimeoutStatus);
        return __syncthreads_or(gave_up ? 1 : 0) != 0;
    };
    auto issue_qk = [&](int c) {
        pend |= 1u << TMA_QK;
        mbar_arrive_expect_tx(&bars[TMA_QK], 2u * CC * DK * 2u);
        for (int kb = 0; kb < DK / 64; ++kb) {
            tma_load_3d(base + Ly.QK + kb * 128 * 128, &tm_q, &bars[TMA_QK], 64 * kb, c * CC, (int)kh);
            tma_load_3d(base + Ly.QK + kb * 128 * 128 + 64 * 128, &tm_k, &bars[TMA_QK], 64 * kb, c * CC, (int)kh);
        }
    };
    auto issue_v = [&](int c) {
        pend |= 1u << TMA_V;
        mbar_arrive_expect_tx(&bars[TMA_V], CC * NVC * 2u);
        tma_load_3d(base + Ly.V, &tm_v, &bars[TMA_V], n0, c * CC, (int)vh);
    };
    auto issue_g = [&](int c) {
        pend |= 1u << TMA_G;
        mbar_arrive_expect_tx(&bars[TMA_G], gbytes);
        tma_load_3d(gts, &tm_g, &bars[TMA_G], 0, c * CC, (int)kh);
    };
    // beta (and the flattened gates when G < 4) of chunk c, one value per thread
    float pf_b = 0.f, pf_g = 0.f;
    auto prefetch_small = [&](int c) {
        const long cs = (long)c * CC;
        if (tid < CC)
            pf_b = (cs + tid < T) ? p.beta[kh * T + cs + tid] : 0.f;
        if (args.g_flat && tid < CC * G)
            pf_g = (cs + tid / G < T) ? p.g[(kh * T + cs) * G + tid] : 0.f;
    };
    auto mma_sync_wait = [&]() {   // called by all threads after tid 0 committed
        return wait_all(MMA, ph_mma);
    };

    // state: row i = 32 * (warp & 3) + lane (+128 for the second half), columns 32*half..+32
    constexpr int NH = DK / 128;
    float sreg[NH][32];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
        const int row = 128 * hh + 32 * (warp & 3) + lane;
#pragma unroll
        for (int n = 0; n < 32; ++n)
            sreg[hh][n] = 0.f;
        if (p.S0 != nullptr) {
            const float *src = p.S0 + (vh * DK + row) * p.dv + n0 + 32 * half;
#pragma unroll
            for (int n = 0; n < 32; n += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(src + n);
                sreg[hh][n] = v4.x; sreg[hh][n + 1] = v4.y; sreg[hh][n + 2] = v4.z; sreg[hh][n + 3] = v4.w;
            }
        }
#pragma unroll
        for (int n = 0; n < 32; n += 8)
            st_tile8(ST, DK, row, 32 * half + n, &sreg[hh][n]);
    }
    if (tid == 0 && N > 0) {
        prefetch_tensormap(&tm_q);
        issue_qk(0);
        issue_v(0);
        if (!args.g_flat)
            issue_g(0);
    }
    prefetch_small(0);
    fence_proxy_async_smem();
    __syncthreads();

    for (int c = 0; c < N && !failed; ++c) {
        const long c0 = (long)c * CC;
        const int Cl = (int)min((long)CC, T - c0);
        if (tid < CC)
            sbeta[tid] = pf_b;
        if (args.g_flat && tid < CC * G)
            gts[tid] = pf_g;
        if (args.g_flat) {
            __syncthreads();
        } else if (wait_all(TMA_G, ph_g)) {
            failed = true;
            break;
        }
        // ---- Lambda = cumsum over the chunk, one thread per decay group
        for (int gi = tid; gi < G; gi += NT) {
            float acc = 0.f;
            for (int t = 0; t < CC; ++t) {
                acc += gts[t * G + gi];
                gts[t * G + gi] = acc;
            }
        }
        __syncthreads();
        // per-channel Lambda_C, e^{Lambda_C}; growth guard
        bool strong = false;
        for (int i = tid; i < DK; i += NT) {
            const float lc = gts[(CC - 1) * G + i / width];
            lamc[i] = lc;
            fch[i] = __expf(lc);
            strong |= (-lc > kGrowthLimit);
        }
        if (G <= 8)
            for (int u = tid; u < CC * G; u += NT) {
                const int t = u / G, gi = u % G;
                const float d = gts[t * G + gi] - gts[(CC - 1) * G + gi];   // Lambda_t - Lambda_C >= 0
                fac[u] = __expf(-d);                                         // e^{Lambda_C - Lambda_t}
                fac[CC * 8 + u] = __expf(fminf(d, kGrowthLimit));            // e^{Lambda_t - Lambda_C}
            }
        strong = __syncthreads_or(strong ? 1 : 0) != 0;
        if (wait_all(TMA_QK, ph_qk)) {
            failed = true;
            break;
        }
        // ---- decayed operands: Khat (new tile), Qr / Kr in place (or raw for the exact Gram)
        for (int u = tid; u < CC * (DK / 8); u += NT) {
            const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
            float qv[8], kv[8], kh8[8];
            ld_tile8(QK, 128, t, i0, qv);
            ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int gi = (i0 + e) / width;
                float fd, fu;
                if (G <= 8) {
                    fd = fac[t * G + gi];
                    fu = fac[CC * 8 + t * G + gi];
                } else {
                    const float d = gts[t * G + gi] - lamc[i0 + e];
                    fd = __expf(-d);
                    fu = __expf(fminf(d, kGrowthLimit));
                }
                kh8[e] = kv[e] * fd;
                if (!strong) {
                    kv[e] *= fu;
                    qv[e] *= fu;
                }
            }
            st_tile8(KH, 64, t, i0, kh8);
            if (!strong) {
                st_tile8(QK, 128, t, i0, qv);
                st_tile8(QK, 128, 64 + t, i0, kv);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (!strong) {
            // ---- Gram: [Qr; Kr] Khat^T  (M = 128, N = 64, K = dk)
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, CC, false, false);
                for (int k0 = 0; k0 < DK; k0 += 16)
                    mma_bf16(tmem + T_G, desc_kmajor(QK, 128, 0, k0), desc_kmajor(KH, 64, 0, k0), id, k0 > 0);
                mma_commit(&bars[MMA]);
            }
            if (mma_sync_wait()) {
                failed = true;
                break;
            }
            tc_fence_after();
            {
                const int R = 32 * (warp & 3) + lane, j0 = 32 * half;
                float g0[16], g1[16];
                tmem_ld16(tq + T_G + j0, g0);
                tmem_ld16(tq + T_G + j0 + 16, g1);
                tmem_ld_wait();
                const bool qrow = R < CC;
                const int t = qrow ? R : R - CC;
                float out[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int j = j0 + u;
                    const float d = u < 16 ? g0[u] : g1[u - 16];
                    out[u] = qrow ? ((j <= t) ? d : 0.f) : ((j < t) ? sbeta[j] * d : 0.f);
                }
                if (qrow) {
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(LT, 128, t, j0 + u, &out[u]);
                } else {
#pragma unroll
                    for (int u = 0; u < 32; u += 4)
                        *reinterpret_cast<float4 *>(&Mf[t * LDM + j0 + u]) =
                            make_float4(out[u], out[u + 1], out[u + 2], out[u + 3]);
                }
            }
            tc_fence_before();
            // Kbar = Kr e^{Lambda_C}, Qbar = Qr e^{Lambda_C} (in place)
            for (int u = tid; u < CC * (DK / 8); u += NT) {
                const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
                float qv[8], kv[8];
                ld_tile8(QK, 128, t, i0, qv);
                ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    qv[e] *= fch[i0 + e];
                    kv[e] *= fch[i0 + e];
                }
                st_tile8(QK, 128, t, i0, qv);
                st_tile8(QK, 128, 64 + t, i0, kv);
            }
        } else {
            // ---- strong decay: the chunk's Gram exactly in fp32 from the raw tiles
            for (int u = tid; u < CC * CC; u += NT) {
                const int t = u / CC, j = u % CC;
                float m = 0.f, l = 0.f;
                if (j <= t) {
                    for (int i0 = 0; i0 < DK; i0 += 8) {
                        float qv[8], kt8[8], kj8[8];
                        ld_tile8(QK, 128, t, i0, qv);
                        ld_tile8(QK, 128, 64 + t, i0, kt8);
                        ld_tile8(QK, 128, 64 + j, i0, kj8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int gi = (i0 + e) / width;
                            const float d = __expf(gts[t * G + gi] - gts[j * G + gi]);
                            m += kt8[e] * kj8[e] * d;
                            l += qv[e] * kj8[e] * d;
                        }
                    }
                }
                Mf[t * LDM + j] = (j < t) ? sbeta[j] * m : 0.f;
                // one bf16 element of L, stored into its place in the swizzled tile
                const float lv = (j <= t) ? l : 0.f;
                const uint32_t addr = LT + sw128_off(128, t, j & ~7) + (j & 7) * 2;
                const uint32_t hi = __float_as_uint(lv);
                const uint16_t h = static_cast<uint16_t>((hi + 0x7FFFu + ((hi >> 16) & 1u)) >> 16);
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(h));
            }
            __syncthreads();
            // Kbar = k e^{Lambda_t}, Qbar = q e^{Lambda_t}
            for (int u = tid; u < CC * (DK / 8); u += NT) {
                const int t = u / (DK / 8), i0 = (u % (DK / 8)) * 8;
                float qv[8], kv[8];
                ld_tile8(QK, 128, t, i0, qv);
                ld_tile8(QK, 128, 64 + t, i0, kv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float f = __expf(gts[t * G + (i0 + e) / width]);
                    qv[e] *= f;
                    kv[e] *= f;
                }
                st_tile8(QK, 128, t, i0, qv);
                st_tile8(QK, 128, 64 + t, i0, kv);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // gates of this chunk are no longer needed except Lambda_C / e^{Lambda_C}: prefetch
        if (tid == 0 && c + 1 < N && !args.g_flat)
            issue_g(c + 1);
        // ---- chunk inverse -> Mf
        if (!p.neumann) {
            inverse64_inplace(Mf, Tf, tid);
        } else {
            // N (bf16, in the [Ab; 0] tile rows 0-63); X (bf16, in RHS tile); fp32 X in Mf
            for (int u = tid; u < CC * 8; u += NT) {
                const int t = u >> 3, j = (u & 7) * 8;
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v8[e] = Mf[t * LDM + j + e];
                st_tile8(AB, 128, t, j, v8);
                float x8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    x8[e] = (t == j + e) ? 1.f : 0.f;
                st_tile8(RT, 64, t, j, x8);
            }
            fence_proxy_async_smem();
            __syncthreads();
            const int rr = row64g(warp, lane);
            const int cb = 32 * half;
            // Horner: X <- I - N X, `order` times (from X = I)
            for (int pw = 1; pw <= p.neu_order; ++pw) {
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(64, 64, false, true);
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_N, desc_kmajor(AB, 128, 0, k0), desc_mnmajor(RT, 64, k0, 0), id, k0 > 0);
                    mma_commit(&bars[MMA]);
                }
                if (mma_sync_wait()) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float d0[16], d1[16];
                tmem_ld16(tq + T_N + cb, d0);
                tmem_ld16(tq + T_N + cb + 16, d1);
                tmem_ld_wait();
                if (rr >= 0) {
                    float x[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        x[u] = ((rr == cb + u) ? 1.f : 0.f) - (u < 16 ? d0[u] : d1[u - 16]);
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(RT, 64, rr, cb + u, &x[u]);
                    if (pw == p.neu_order)
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            Mf[rr * LDM + cb + u] = x[u];
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
            }
            if (failed)
                break;
            if (p.neu_order == 0) {
                for (int u = tid; u < CC * CC; u += NT)
                    Mf[(u / CC) * LDM + (u % CC)] = ((u / CC) == (u % CC)) ? 1.f : 0.f;
                __syncthreads();
            }
            // Newton residual steps: Rm = I - X - N X ; X <- X + X Rm
            for (int st = 0; st < p.neu_resid && !failed; ++st) {
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(64, 64, false, true);
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_N, desc_kmajor(AB, 128, 0, k0), desc_mnmajor(RT, 64, k0, 0), id, k0 > 0);
                    mma_commit(&bars[MMA]);
                }
                if (mma_sync_wait()) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float d0[16], d1[16];
                tmem_ld16(tq + T_N + cb, d0);
                tmem_ld16(tq + T_N + cb + 16, d1);
                tmem_ld_wait();
                if (rr >= 0) {
                    float rm[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        rm[u] = ((rr == cb + u) ? 1.f : 0.f) - Mf[rr * LDM + cb + u] - (u < 16 ? d0[u] : d1[u - 16]);
#pragma unroll
                    for (int u = 0; u < 32; u += 8)
                        st_tile8(ET, 64, rr, cb + u, &rm[u]);     // Rm as an MN-major B operand
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
                // X Rm with X (bf16, RHS tile) as a K-major A operand
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(64, 64, false, true);
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_N, desc_kmajor(RT, 64, 0, k0), desc_mnmajor(ET, 64, k0, 0), id, k0 > 0);
                    mma_commit(&bars[MMA]);
                }
                if (mma_sync_wait()) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                tmem_ld16(tq + T_N + cb, d0);
                tmem_ld16(tq + T_N + cb + 16, d1);
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
                        st_tile8(RT, 64, rr, cb + u, &x[u]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncthreads();
            }
            if (failed)
                break;
        }
        // ---- [Ab; 0] = diag(beta) A  (rows 0-63)
        for (int u = tid; u < CC * 8; u += NT) {
            const int t = u >> 3, j = (u & 7) * 8;
            const float bt = sbeta[t];
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                a[e] = bt * Mf[t * LDM + j + e];
            st_tile8(AB, 128, t, j, a);
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---- [Qbar; Kbar] S  (M = 128, N = 64, K = dk)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, NVC, false, true);
            for (int k0 = 0; k0 < DK; k0 += 16)
                mma_bf16(tmem + T_Y, desc_kmajor(QK, 128, 0, k0), desc_mnmajor(ST, DK, k0, 0), id, k0 > 0);
            mma_commit(&bars[MMA]);
        }
        if (mma_sync_wait()) {
            failed = true;
            break;
        }
        tc_fence_after();
        if (wait_all(TMA_V, ph_v)) {
            failed = true;
            break;
        }
        // q, k of this chunk are spent (Khat has its own tile): prefetch the next ones
        if (tid == 0 && c + 1 < N)
            issue_qk(c + 1);
        // ---- RHS = V - Kbar S  (rows 64-127 of T_Y)
        if ((warp & 3) >= 2) {
            const int t = 32 * (warp & 3) + lane - CC;
            float y0[16], y1[16];
            tmem_ld16(tq + T_Y + 32 * half, y0);
            tmem_ld16(tq + T_Y + 32 * half + 16, y1);
            tmem_ld_wait();
            float r[32];
#pragma unroll
            for (int u = 0; u < 32; u += 8) {
                float v8[8];
                ld_tile8(VT, 64, t, 32 * half + u, v8);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    r[u + e] = v8[e] - (u + e < 16 ? y0[u + e] : y1[u + e - 16]);
            }
#pragma unroll
            for (int u = 0; u < 32; u += 8)
                st_tile8(RT, 64, t, 32 * half + u, &r[u]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && c + 1 < N) {
            issue_v(c + 1);
        }
        // ---- E = [Ab; 0] RHS
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, NVC, false, true);
            for (int k0 = 0; k0 < CC; k0 += 16)
                mma_bf16(tmem + T_E, desc_kmajor(AB, 128, 0, k0), desc_mnmajor(RT, 64, k0, 0), id, k0 > 0);
            mma_commit(&bars[MMA]);
        }
        if (mma_sync_wait()) {
            failed = true;
            break;
        }
        tc_fence_after();
        if ((warp & 3) < 2) {
            const int t = 32 * (warp & 3) + lane;
            float e0[16], e1[16];
            tmem_ld16(tq + T_E + 32 * half, e0);
            tmem_ld16(tq + T_E + 32 * half + 16, e1);
            tmem_ld_wait();
            st_tile8(ET, 64, t, 32 * half, &e0[0]);
            st_tile8(ET, 64, t, 32 * half + 8, &e0[8]);
            st_tile8(ET, 64, t, 32 * half + 16, &e1[0]);
            st_tile8(ET, 64, t, 32 * half + 24, &e1[8]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (c + 1 < N)
            prefetch_small(c + 1);
        // ---- dS = Khat^T E  (M = 128 per half of dk),  O = QS + [L; 0] E
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_ds = idesc_bf16(128, NVC, true, true);
            const uint32_t id_o = idesc_bf16(128, NVC, false, true);
            for (int hh = 0; hh < NH; ++hh)
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_DS + 64 * hh, desc_mnmajor(KH, 64, k0, 128 * hh),
                             desc_mnmajor(ET, 64, k0, 0), id_ds, k0 > 0);
            for (int k0 = 0; k0 < CC; k0 += 16)
                mma_bf16(tmem + T_Y, desc_kmajor(LT, 128, 0, k0), desc_mnmajor(ET, 64, k0, 0), id_o, 1u);
            mma_commit(&bars[MMA]);
        }
        if (mma_sync_wait()) {
            failed = true;
            break;
        }
        tc_fence_after();
        // ---- S <- diag(e^{Lambda_C}) S + dS ; O (rows 0-63 of T_Y)
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            const int row = 128 * hh + 32 * (warp & 3) + lane;
            const float F = fch[row];
            float d0[16], d1[16];
            tmem_ld16(tq + T_DS + 64 * hh + 32 * half, d0);
            tmem_ld16(tq + T_DS + 64 * hh + 32 * half + 16, d1);
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 32; ++n)
                sreg[hh][n] = F * sreg[hh][n] + (n < 16 ? d0[n] : d1[n - 16]);
#pragma unroll
            for (int n = 0; n < 32; n += 8)
                st_tile8(ST, DK, row, 32 * half + n, &sreg[hh][n]);
        }
        if ((warp & 3) < 2) {
            const int t = 32 * (warp & 3) + lane;
            float o0[16], o1[16];
            tmem_ld16(tq + T_Y + 32 * half, o0);
            tmem_ld16(tq + T_Y + 32 * half + 16, o1);
            tmem_ld_wait();
            if (t < Cl) {
                const long orow = (vh * T + c0 + t) * p.dv + n0 + 32 * half;
                if constexpr (OUT_BF16) {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow);
                    dst[0] = make_uint4(pack_bf16(o0[0], o0[1]), pack_bf16(o0[2], o0[3]), pack_bf16(o0[4], o0[5]), pack_bf16(o0[6], o0[7]));
                    dst[1] = make_uint4(pack_bf16(o0[8], o0[9]), pack_bf16(o0[10], o0[11]), pack_bf16(o0[12], o0[13]), pack_bf16(o0[14], o0[15]));
                    dst[2] = make_uint4(pack_bf16(o1[0], o1[1]), pack_bf16(o1[2], o1[3]), pack_bf16(o1[4], o1[5]), pack_bf16(o1[6], o1[7]));
                    dst[3] = make_uint4(pack_bf16(o1[8], o1[9]), pack_bf16(o1[10], o1[11]), pack_bf16(o1[12], o1[13]), pack_bf16(o1[14], o1[15]));
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow);
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        dst[n] = make_float4(o0[4 * n], o0[4 * n + 1], o0[4 * n + 2], o0[4 * n + 3]);
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        dst[4 + n] = make_float4(o1[4 * n], o1[4 * n + 1], o1[4 * n + 2], o1[4 * n + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    if (!failed && p.S_final != nullptr) {
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            const int row = 128 * hh + 32 * (warp & 3) + lane;
            float *dst = p.S_final + (vh * DK + row) * p.dv + n0 + 32 * half;
#pragma unroll
            for (int n = 0; n < 32; n += 4)
                *reinterpret_cast<float4 *>(dst + n) =
                    make_float4(sreg[hh][n], sreg[hh][n + 1], sreg[hh][n + 2], sreg[hh][n + 3]);
        }
    }
    // drain: let every load and product this CTA started finish (bounded)
    if (tid == 0) {
        mma_commit(&bars[MMA]);
        mbar_wait(&bars[MMA], ph_mma, 200000000ull);
        if (pend & (1u << TMA_QK))
            mbar_wait(&bars[TMA_QK], ph_qk, 200000000ull);
        if (pend & (1u << TMA_V))
            mbar_wait(&bars[TMA_V], ph_v, 200000000ull);
        if (pend & (1u << TMA_G))
            mbar_wait(&bars[TMA_G], ph_g, 200000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// fp32 3-D map, no swizzle
inline bool make_map_f32(CUtensorMap *m, const void *ptr, const cuuint64_t (&dims)[3],
                         const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3])
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, bool OB>
int launch(const Params &p, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv, mg;
    const long sk = (long)p.B * p.Hk;
    GenArgs a;
    a.p = p;
    a.nvt = p.dv / NVC;
    a.g_flat = p.G < 4;
    bool ok = make_map(&mq, p.q, DK, p.T, sk, CC) && make_map(&mk, p.k, DK, p.T, sk, CC) &&
              make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CC);
    if (!a.g_flat) {
        const cuuint64_t dims[3] = {(cuuint64_t)p.G, (cuuint64_t)p.T, (cuuint64_t)sk};
        const cuuint64_t str[2] = {(cuuint64_t)p.G * 4, (cuuint64_t)p.G * 4 * p.T};
        const cuuint32_t box[3] = {(cuuint32_t)p.G, CC, 1};
        ok = ok && make_map_f32(&mg, p.g, dims, str, box);
    } else {
        mg = mq;   // unused
    }
    if (!ok)
        return 6;
    const Plan<DK> Ly = plan<DK>();
    auto kern = gen_kernel<DK, OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    dim3 grid(a.nvt * p.Hv, p.B);
    kern<<<grid, NT, Ly.total, stream>>>(mq, mk, mv, mg, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

inline bool supports(const Params &p)
{
    return p.in_bf16 && p.C == CC && (p.dk == 128 || p.dk == 256) && p.dv % NVC == 0 &&
           p.G >= 1 && p.G <= gmax(p.dk) && p.T >= 1 && p.B <= 65535;
}

}  // namespace gen
