// gdr_tc_split.cuh -- second pass of the two-pass tensor-core path: the
// inter-chunk state recurrence and the readout, for key width dk = 128, chunk
// C = 64, 64 value columns per CTA, any decay grouping.  The chunk-local
// factors T = diag(beta) (I + M)^{-1}, L and W = T Kbar come from the first
// pass (gdr_tc_prep.cuh), so the serial chain per chunk holds only the state
// products ("Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta
// Attention for TPUs", §2.1, §2.3 Table 2, §2.4.2):
//   U = T V                                  (off the chain, one chunk ahead)
//   P = W S,  E = U - P                      (chain)
//   S <- F S + Khat^T E,  O = Qbar S + L E   (chain; O leaves off the chain)
// with Kbar = k e^{Lambda_t}, Khat = k e^{Lambda_C - Lambda_t},
// Qbar = q e^{Lambda_t}, F = diag(e^{Lambda_C}) -- all factors <= 1.  For the
// scalar gate Khat^T E = K^T (diag(e^{Lambda_C - Lambda}) E) and
// Qbar S = diag(e^Lambda) (Q S) (the epilogue applies it), so q and k are used
// as loaded; for grouped / per-channel gates Qbar and Khat come decayed from
// the first pass.  Nothing here evaluates an exponential.
//
// Roles (warp-specialised, hand-offs through mbarriers; every wait bounded):
//   warps 0-1   epilogue: O = f (Q S) + L E from TMEM to global memory
//   warps 2, 12 producers: TMA / bulk copies into a 2-stage ring.  A thread's
//               bulk copies are accepted one after another (about 30 bytes a
//               cycle), so two threads share a stage: warp 2 issues W, Q and
//               the factors, warp 12 T and V, then group Y
//   warp 3      MMA issuer (one thread)
//   warps 4-11  state chain: S (fp32, TMEM) -> bf16 operand, E = U - P; two
//               warps per TMEM lane quarter, each lane on 32 of the 64 columns
// A stage is loaded in two groups with their own barriers, so that it can be
// refilled as soon as each group's last reader is done:
//   X = {W, Q, T, V, factors}: read by U, P and the state warps (which copy their
//       factors to registers early) -> free once P is done;
//   Y = {K, L}: read by the update and the readout -> free after them.
// MMA operands are stacked so that M = 128 and no product reads a tile that a
// load may be refilling:
//   [0; T] V -> U (rows 64-127),  [Q; W] S -> Q S (rows 0-63), P (rows 64-127),
//   Khat^T E onto F S,  [L; 0] E -> L E (rows 0-63).

namespace split {

constexpr int NWARP = 13;
constexpr int NTHR = NWARP * 32;   // 416
constexpr int CC = 64;
constexpr int KD = 128;             // key width of the segment-parallel form
constexpr int NVC = 64;
constexpr int W_EPI0 = 0, W_PROD = 2, W_MMA = 3, W_STATE0 = 4, W_PROD_Y = 12;
constexpr int N_STATE = 256, N_EPI = 64;
constexpr int NB_STATE = 1, NB_EPI = 2;   // named barriers

constexpr uint32_t T_U = 0;        // two buffers of 64 cols: [0; T] V (rows 64-127)
constexpr uint32_t T_PO = 128;     // two buffers of 64 cols: [Q; W] S
constexpr uint32_t T_S = 256;      // fp32 state, 64 cols per 128 key rows
// two buffers of 64 cols after the state: [L; 0] E (rows 0-63)
__host__ __device__ constexpr uint32_t t_le(int dk) { return T_S + dk / 2; }
// chunk-boundary momentum (dk = 128): the velocity Z, fp32, 64 cols after the LE buffers
constexpr uint32_t T_Z = 448;
constexpr uint32_t TMEM_COLS = 512;

enum Bar { FULLX0, FULLX1, FULLY0, FULLY1, FREEX0, FREEX1, FREEY0, FREEY1, S_READY, P_FULL, E_READY,
           UPD_DONE, OUT0, OUT1, OFREE0, OFREE1, DRAIN, VFREE, NBARS };

// The stage-s member of a two-stage plan array, selected rather than indexed, so that
// a plan whose arrays are indexed by a runtime stage stays in registers (an indexed
// array would live in local memory, one load on every use).
__host__ __device__ __forceinline__ uint32_t stage(const uint32_t (&a)[2], int s) { return s ? a[1] : a[0]; }

template <int DK>
struct Gates {                        // landed by bulk copies from the first pass's record
    float ea[CC], eb[CC];             // scalar gate: e^{Lambda_t}, e^{Lambda_C - Lambda_t}
    float F[DK];                      // e^{Lambda_C} per key channel (F[0] for the scalar gate)
};

struct Plan {
    uint32_t qwk[2], lz[2], v[2], ab[2], gates[2];
    uint32_t S, E, Eh, bar, misc, total;
};

// Stage: [Q | W | K] (rows 0-63 | 64-127 | 128-191, dk columns), [L | 0]
// (64 + 64 rows), V (64 rows) and [0 | T] (64 + 64 rows), 64 columns each.  At
// dk = 256 the [Q | W | K] tile (96 KB) has one buffer shared by both stages:
// the next chunk's W and Q land once P has read this chunk's, its K once the
// update has (the other parts keep two stages).
template <int DK>
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
        s.qwk[i] = (i == 0 || DK == 128) ? take((DK / 64) * 192 * 128) : s.qwk[0];
        s.lz[i] = take(128 * 128);
        s.v[i] = take(64 * 128);
        s.ab[i] = take(128 * 128);
        s.gates[i] = take(sizeof(Gates<DK>));
    }
    s.S = take(DK * NVC * 2);
    s.E = take(CC * NVC * 2);
    s.Eh = scalar ? take(CC * NVC * 2) : s.E;
    s.bar = take(NBARS * 8 + 16);
    s.misc = s.bar + NBARS * 8;
    s.total = o + 1024;
    return s;
}

// How a launch walks the chunks.  MODE_SEQ: every CTA walks its whole sequence.
// The segment-parallel form cuts each sequence into nseg segments of seg_len
// chunks (grid.z = segment) and composes the affine maps S -> A_c S + B_c of the
// chunks, A_c = F_c - Khat_c^T W_c and B_c = Khat_c^T U_c:
//   MODE_SEG_AB: value-tile CTAs run their segment from S = 0 and store its end
//     state Btil (no outputs); transition CTAs (grid.x past the value tiles, two
//     per key head) run it from the identity with no values and store
//     Atil = prod A_c, 64 of its columns each (the 128-column pass runs both
//     chains of a key head in one CTA, ab128_kernel);
//   seg_combine_kernel: S_start(0) = S0, S_start(g + 1) = Atil_g S_start(g) + Btil_g;
//   MODE_SEG_C: every segment runs from its S_start and writes o; the last one
//     writes S_final.
enum Mode { MODE_SEQ = 0, MODE_SEG_AB = 1, MODE_SEG_C = 2 };

struct SplitArgs {
    Params p;
    const uint8_t *factors;   // first-pass output, [B * Hk * nchunks][rec_bytes]
    uint32_t rec_bytes;       // prep::SC_BYTES (scalar gate) or prep::EXT_BYTES
    int nvt;
    int nchunks;
    int mode;                 // Mode
    int nseg, seg_len;        // segments per sequence and chunks per segment
    float *seg_end;           // [B][Hv][nseg][KD][dv]: Btil of each segment
    float *seg_trans;         // [B][Hk][nseg][KD][KD]: Atil of each segment
    float *seg_start;         // [B][Hv][nseg][KD][dv]: the state each segment starts from
    int pair;                 // chunks of 128 run as pairs of 64-token halves (Neumann inverse)
    uint32_t pair_y;          // byte offset of the pair correction Y in a record
};

// Segment count for the state pass of a request: cost model in chunk periods, one
// resident CTA per SM on kSMs SMs.  The segmented form does about three times the
// chain work (values from zero, the transition, values again), so it pays only
// when the sequential pass leaves most SMs idle.
constexpr int kSMs = 148;
constexpr int kMinSegChunks = 16;

struct SegPlan {
    int nseg, seg_len;
};

inline SegPlan seg_plan(const Params &p)
{
    const int N = prep::nchunks(p);
    if (p.dk != KD || p.momentum)   // built for dk = 128 and a state without velocity
        return SegPlan{1, N};
    const int even = p.pair ? 2 : 1;   // pairs never straddle a segment boundary
    const long nvh = (long)(p.dv / NVC) * p.Hv * p.B;
    const long ntr = (long)(KD / NVC) * p.Hk * p.B;
    auto waves = [](long ctas) { return (ctas + kSMs - 1) / kSMs; };
    const long seq_cost = waves(nvh) * (long)N;
    SegPlan best{1, N};
    long best_cost = seq_cost;
    for (int ns = 2; ns <= N / kMinSegChunks; ++ns) {
        const int L = ((N + ns - 1) / ns + even - 1) / even * even;
        const int nsg = (N + L - 1) / L;
        const long cost = (waves((nvh + ntr) * nsg) + waves(nvh * nsg)) * (long)L + nsg;
        if (cost < best_cost) {
            best_cost = cost;
            best = SegPlan{nsg, L};
        }
    }
    return (best.nseg > 1 && best_cost * 5 <= seq_cost * 4) ? best : SegPlan{1, N};
}

// Bytes past the records that the segmented form needs (256-byte aligned pieces).
inline size_t seg_bytes(const Params &p)
{
    const SegPlan sp = seg_plan(p);
    if (sp.nseg == 1)
        return 0;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t per_v = (size_t)p.B * p.Hv * sp.nseg * KD * p.dv * 4;
    return 2 * al(per_v) + al((size_t)p.B * p.Hk * sp.nseg * KD * KD * 4);
}

// Bounded wait without sleeping between probes: every hand-off in this kernel
// is on or next to the per-chunk critical chain, where a back-off sleep would
// add its length to the chunk period.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag)
{
    if (ptx::mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait(bar, parity))
            return true;
        if ((it & 255) == 0) {
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

template <int DK, bool OUT_BF16>
__global__ void __launch_bounds__(NTHR, 1)
split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const SplitArgs args)
{
    using namespace ptx;
    using ws::named_sync;
    using ws::named_vote_or;
    extern __shared__ uint8_t smem_raw[];
    const Params &p = args.p;
    const bool scalar = p.G == 1;
    const Plan Ly = plan<DK>(scalar);
    constexpr bool ONE = DK > 128;          // one [Q | W | K] buffer (see plan)
    constexpr int NKB = DK / 64;            // 64-column blocks of a key-side tile
    constexpr uint32_t T_LE = t_le(DK);
    const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_u32 - smem_u32(smem_raw));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nvh = args.nvt * p.Hv;   // value-tile CTAs per batch entry
    // a transition CTA of the segmented form: identity start, no values, no outputs
    const bool trans = args.mode == MODE_SEG_AB && (int)blockIdx.x >= nvh;
    const int xi = trans ? (int)blockIdx.x - nvh : (int)blockIdx.x;
    const int nt = trans ? xi % (DK / NVC) : xi % args.nvt;
    const int hv = trans ? 0 : xi / args.nvt;
    const int b = blockIdx.y;
    const int hk = trans ? xi / (DK / NVC) : hv / p.R;
    const int n0 = nt * NVC;
    const long kh = (long)b * p.Hk + hk;
    const long vh = (long)b * p.Hv + hv;
    const int T = p.T;
    const int N = args.nchunks;
    const bool outputs = args.mode != MODE_SEG_AB;   // o is written
    // this CTA's chunks: cbeg .. cbeg + nloc - 1 (local index i = c - cbeg drives the
    // ring stages and barrier phases)
    const int seg = blockIdx.z;
    const int cbeg = seg * args.seg_len;
    const int nloc = min(args.seg_len, N - cbeg);

    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 4);
    auto gates_of = [&](int s) { return reinterpret_cast<Gates<DK> *>(base + stage(Ly.gates, s)); };
    // Wait before loading chunk i into stage i & 1 until its previous contents are
    // released (FREEX0 / FREEY0 and the stage's offset): with two buffers, their use by
    // chunk i - 2; with one [Q | W | K] buffer, the previous chunk's release of the
    // other stage, which also implies chunk i - 2's (the releases come in chunk order)
    auto wait_free = [&](int bar0, int i) -> bool {
        if (ONE) {
            if (i < 1)
                return true;
            return wait_or_abort(&bars[bar0 + ((i - 1) & 1)], ((i - 1) >> 1) & 1, abort_flag);
        }
        if (i < 2)
            return true;
        return wait_or_abort(&bars[bar0 + (i & 1)], ((i >> 1) - 1) & 1, abort_flag);
    };
    const uint32_t S_T = base_u32 + Ly.S, E_T = base_u32 + Ly.E, EH_T = base_u32 + Ly.Eh;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)   // FREEX: the MMAs' commit and the state warps
            mbar_init(&bars[i], (i == FREEX0 || i == FREEX1) ? 2 : 1);
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
    // the zero halves of [L; 0] and [0; T] (never loaded)
    for (int i = tid; i < 2 * 64 * 8; i += NTHR) {
        const int st = i >> 9, r = (i >> 3) & 63, c = (i & 7) * 8;
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        st_tile8(base_u32 + stage(Ly.lz, st), 128, 64 + r, c, z);
        st_tile8(base_u32 + stage(Ly.ab, st), 128, r, c, z);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int R = 32 * (warp & 3) + lane;     // TMEM lane of this thread

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        int narmx = 0;     // group X loads armed per stage
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, s = i & 1;
            const long c0 = (long)c * CC;
            const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
            uint8_t *qwk = base + stage(Ly.qwk, s);
            // group X: W, Q (or Qbar), T, V, the decay factors.  Q only where o is
            // written; T and V not for a transition CTA.
            {
                const bool ok = wait_free(FREEX0, i);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            if (lane == 0) {
                uint64_t *full = &bars[FULLX0 + s];
                const uint32_t fac_bytes = scalar ? prep::SC_BYTES - prep::SC_EA : DK * 4;
                // W, Q: dk / 64 images each; T: one; V: 64 x 64 bf16
                mbar_arrive_expect_tx(full, NKB * prep::IMG + (outputs ? NKB * prep::IMG : 0u) +
                                                (trans ? 0u : prep::IMG + CC * NVC * 2) + fac_bytes);
                for (int kb = 0; kb < NKB; ++kb) {
                    uint8_t *blk = qwk + kb * 192 * 128;
                    bulk_load(blk + 64 * 128, fac + prep::REC_W + kb * prep::IMG, prep::IMG, full);
                    if (!outputs)
                        continue;
                    if (scalar)
                        tma_load_3d(blk, &tm_q, full, 64 * kb, (int)c0, (int)kh);
                    else
                        bulk_load(blk, fac + prep::ext_qb(DK) + kb * prep::IMG, prep::IMG, full);
                }
                if (scalar)
                    bulk_load(gates_of(s)->ea, fac + prep::SC_EA, fac_bytes, full);
                else
                    bulk_load(gates_of(s)->F, fac + prep::ext_f(DK), fac_bytes, full);
            }
            ++narmx;
        }
        // drain loads that may still be landing (bounded): the last armed phase of
        // each barrier, whether or not a consumer saw it
        if (lane == 0) {
            for (int s = 0; s < 2; ++s)
                if ((narmx + 1 - s) / 2 > 0)   // loads armed on stage s
                    mbar_wait(&bars[FULLX0 + s], ((narmx + 1 - s) / 2 - 1) & 1, 200000000ull);
        }
    } else if (warp == W_PROD_Y) {
        // ------------------------------------------------------------ second producer
        // T and V of group X (their bytes are part of what warp W_PROD expects on FULLX,
        // so the phase completes only when both threads' copies have landed), then
        // group Y.
        int narmy = 0;     // group Y loads armed per stage
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, s = i & 1;
            const long c0 = (long)c * CC;
            const uint8_t *fac = args.factors + (size_t)(kh * N + c) * args.rec_bytes;
            uint8_t *qwk = base + stage(Ly.qwk, s);
            // T and V of group X (counted in the FULLX bytes that warp W_PROD expects)
            if (!trans) {
                {
                    const bool ok = wait_free(FREEX0, i);
                    if (__any_sync(0xffffffffu, !ok))
                        break;
                }
                if (lane == 0) {
                    uint64_t *full = &bars[FULLX0 + s];
                    bulk_load(base + stage(Ly.ab, s) + 64 * 128, fac, prep::IMG, full);
                    tma_load_3d(base + stage(Ly.v, s), &tm_v, full, n0, (int)c0, (int)vh);
                }
            }
            // group Y: K (or Khat), L (L only where o is written)
            {
                const bool ok = wait_free(FREEY0, i);
                if (__any_sync(0xffffffffu, !ok))
                    break;
            }
            // pairs: the first half's Y goes under its L ([L; Y]); stage 0 holds first
            // halves, since every segment starts at an even chunk
            const bool with_y = args.pair && s == 0;
            if (lane == 0) {
                uint64_t *full = &bars[FULLY0 + s];
                mbar_arrive_expect_tx(full, (NKB + (outputs ? 1u : 0u)) * prep::IMG + (with_y ? prep::IMG : 0u));
                if (with_y)
                    bulk_load(base + stage(Ly.lz, s) + 64 * 128, fac + args.pair_y, prep::IMG, full);
                for (int kb = 0; kb < NKB; ++kb) {
                    uint8_t *blk = qwk + kb * 192 * 128 + 128 * 128;
                    if (scalar)
                        tma_load_3d(blk, &tm_k, full, 64 * kb, (int)c0, (int)kh);
                    else
                        bulk_load(blk, fac + prep::ext_kh(DK) + kb * prep::IMG, prep::IMG, full);
                }
                if (outputs)
                    bulk_load(base + stage(Ly.lz, s), fac + prep::IMG, prep::IMG, full);
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
            const uint32_t id_u = idesc_bf16(128, NVC, false, true);
            const uint32_t id_po = idesc_bf16(128, NVC, false, true);
            const uint32_t id_s = idesc_bf16(128, NVC, true, true);   // per 128 key rows
            // descriptors at k = 0 of stage 0; a K step adds its byte offset / 16 to the
            // start field, stage 1 a fixed distance
            const uint64_t d_ab0 = desc_kmajor(base_u32 + Ly.ab[0], 128, 0, 0);
            const uint64_t d_v0 = desc_mnmajor(base_u32 + Ly.v[0], 64, 0, 0);
            const uint64_t d_qw0 = desc_kmajor(base_u32 + Ly.qwk[0], 192, 0, 0);
            const uint64_t d_kt0 = desc_mnmajor(base_u32 + Ly.qwk[0], 192, 128, 0);
            const uint64_t d_lz0 = desc_kmajor(base_u32 + Ly.lz[0], 128, 0, 0);
            const uint64_t dab = (Ly.ab[1] - Ly.ab[0]) >> 4, dv = (Ly.v[1] - Ly.v[0]) >> 4;
            const uint64_t dqw = (Ly.qwk[1] - Ly.qwk[0]) >> 4, dlz = (Ly.lz[1] - Ly.lz[0]) >> 4;
            const uint64_t d_s = desc_mnmajor(S_T, DK, 0, 0);
            // K^T's rows 128-255 (dk = 256): two 64-column blocks further on
            const uint64_t dkt_hi = (uint64_t)((2 * 192 * 128) >> 4);
            const uint64_t d_e = desc_mnmajor(scalar ? EH_T : E_T, CC, 0, 0);
            const uint64_t d_eo = desc_mnmajor(E_T, CC, 0, 0);
            auto kstep = [](int k0, int rows) {
                return static_cast<uint64_t>(((k0 >> 6) * rows * 128 + (k0 & 63) * 2) >> 4);
            };
            auto mstep = [](int k0) { return static_cast<uint64_t>(k0 * 8); };
            auto issue_u = [&](int st) {   // U of the chunk in stage st -> T_U buffer st
                const uint64_t a0 = d_ab0 + st * dab, v0 = d_v0 + st * dv;
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_U + 64 * st, a0 + kstep(k0, 128), v0 + mstep(k0), id_u, k0 > 0);
            };
            // a transition CTA has no values: U = 0 and no U product (u_ready stays true)
            bool ok = true, u_ready = trans;
            for (int i = 0; i < nloc && ok; ++i) {
                const int s = i & 1;
                const uint32_t par = i & 1;
                if (!(ok = wait_or_abort(&bars[FULLX0 + s], (i >> 1) & 1, abort_flag)))
                    break;
                if (!u_ready) {
                    tc_fence_after();
                    issue_u(s);
                }
                if (!(ok = wait_or_abort(&bars[S_READY], par, abort_flag)))
                    break;
                if (i >= 2 && !(ok = wait_or_abort(&bars[OFREE0 + s], ((i >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint64_t qw = d_qw0 + s * dqw, kt = d_kt0 + s * dqw, lz = d_lz0 + s * dlz;
                for (int k0 = 0; k0 < DK; k0 += 16)
                    mma_bf16(tmem + T_PO + 64 * s, qw + kstep(k0, 192), d_s + mstep(k0), id_po, k0 > 0);
                mma_commit(&bars[P_FULL]);
                // U and P are the last tensor-core readers of group X (the state warps
                // hold their factors in registers by then and arrive themselves)
                mma_commit(&bars[FREEX0 + s]);
                // the next chunk's U overlaps this chunk's E step when its tiles are in
                u_ready = trans;
                if (!trans && i + 1 < nloc && mbar_test(&bars[FULLX0 + (s ^ 1)], ((i + 1) >> 1) & 1)) {
                    tc_fence_after();
                    issue_u(s ^ 1);
                    u_ready = true;
                }
                if (!(ok = wait_or_abort(&bars[E_READY], par, abort_flag)))
                    break;
                if (!(ok = wait_or_abort(&bars[FULLY0 + s], (i >> 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                for (int h = 0; h < DK / 128; ++h)
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_S + 64 * h, kt + h * dkt_hi + mstep(k0), d_e + mstep(k0), id_s, 1u);
                if (p.momentum)   // the same update into the velocity (dk = 128)
                    for (int k0 = 0; k0 < CC; k0 += 16)
                        mma_bf16(tmem + T_Z, kt + mstep(k0), d_e + mstep(k0), id_s, 1u);
                mma_commit(&bars[UPD_DONE]);
                for (int k0 = 0; k0 < CC; k0 += 16)
                    mma_bf16(tmem + T_LE + 64 * s, lz + kstep(k0, 128), d_eo + mstep(k0), id_po, k0 > 0);
                mma_commit(&bars[OUT0 + s]);
                mma_commit(&bars[FREEY0 + s]);
            }
            // whatever was issued must finish before tensor memory is released
            mma_commit(&bars[DRAIN]);
            mbar_wait(&bars[DRAIN], 0, 200000000ull);
        }
    } else if (warp >= W_STATE0) {
        // ------------------------------------------------------------ state chain
        const int stid = tid - W_STATE0 * 32;
        const int cs = 32 * ((warp - W_STATE0) >> 2);   // this lane's 32 of the 64 columns
        constexpr int NH = DK / 128;                     // key rows R + 128 h of this thread
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            // start state: S0 (or zero) for a whole sequence, zero for a segment's end
            // state, the identity's columns for a transition, S_start of the segment
            const int row = R + 128 * h;
            float s0[16], s1[16];
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                s0[n] = (trans && row == n0 + cs + n) ? 1.f : 0.f;
                s1[n] = (trans && row == n0 + cs + 16 + n) ? 1.f : 0.f;
            }
            const float *src = nullptr;
            if (args.mode == MODE_SEQ && p.S0 != nullptr)
                src = p.S0 + (vh * DK + row) * p.dv + n0 + cs;
            else if (args.mode == MODE_SEG_C)
                src = args.seg_start + (((size_t)vh * args.nseg + seg) * KD + row) * p.dv + n0 + cs;
            if (src != nullptr) {
#pragma unroll
                for (int n = 0; n < 16; n += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(src + n);
                    const float4 b4 = *reinterpret_cast<const float4 *>(src + 16 + n);
                    s0[n] = a4.x; s0[n + 1] = a4.y; s0[n + 2] = a4.z; s0[n + 3] = a4.w;
                    s1[n] = b4.x; s1[n + 1] = b4.y; s1[n + 2] = b4.z; s1[n + 3] = b4.w;
                }
            }
            tmem_st16(tq + T_S + 64 * h + cs, s0);
            tmem_st16(tq + T_S + 64 * h + cs + 16, s1);
        }
        if (p.momentum) {   // Z_0 = 0
            float z[16];
#pragma unroll
            for (int n = 0; n < 16; ++n)
                z[n] = 0.f;
            tmem_st16(tq + T_Z + cs, z);
            tmem_st16(tq + T_Z + cs + 16, z);
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
            // S_{c-1} -> bf16 operand of P; only then T_S <- F S_{c-1} (the update MMA
            // accumulates onto it), which nothing reads before E_READY
            float s0[NH][16], s1[NH][16];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                tmem_ld16(tq + T_S + 64 * h + cs, s0[h]);
                tmem_ld16(tq + T_S + 64 * h + cs + 16, s1[h]);
            }
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                st_tile8(S_T, DK, R + 128 * h, cs, &s0[h][0]);
                st_tile8(S_T, DK, R + 128 * h, cs + 8, &s0[h][8]);
                st_tile8(S_T, DK, R + 128 * h, cs + 16, &s1[h][0]);
                st_tile8(S_T, DK, R + 128 * h, cs + 24, &s1[h][8]);
            }
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
            const Gates<DK> *gt = gates_of(s);
            // this thread's factors of the stage, read now: group X is refilled as soon
            // as P is done
            const float f_eb = (scalar && R >= CC) ? gt->eb[R - CC] : 1.f;
            // chunk-boundary momentum: Z <- mu kappa_c Z, and S <- F S + that Z, so that the
            // update, added to both, leaves Z_c = mu kappa_c Z_{c-1} + Khat^T E and
            // S_c = F S_{c-1} + Z_c (dk = 128: one row per thread); 16 columns at a time
            const float zk = p.momentum ? p.mu * (p.kappa != nullptr ? (float)p.kappa[(long)b * N + cbeg + i]
                                                                     : 1.f)
                                        : 0.f;
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float F = scalar ? gt->F[0] : gt->F[R + 128 * h];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float *sv = part == 0 ? s0[h] : s1[h];
                    const uint32_t col = 64 * h + cs + 16 * part;
#pragma unroll
                    for (int n = 0; n < 16; ++n)
                        sv[n] *= F;
                    if (p.momentum) {
                        float z[16];
                        tmem_ld16(tq + T_Z + cs + 16 * part, z);
                        tmem_ld_wait();
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            z[n] *= zk;
                            sv[n] += z[n];
                        }
                        tmem_st16(tq + T_Z + cs + 16 * part, z);
                    }
                    tmem_st16(tq + T_S + col, *reinterpret_cast<const float(*)[16]>(sv));
                }
            }
            if (named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[P_FULL], par, abort_flag))) {
                ok = false;
                break;
            }
            if (stid == 0)   // every state thread has read its factors (the vote above)
                mbar_arrive(&bars[FREEX0 + s]);
            tc_fence_after();
            if (R >= CC) {   // warps of lane quarters 2 and 3: rows t of P, U and E
                const int t = R - CC;
                const float f = f_eb;
                float p0[16], p1[16], u0[16], u1[16];
                tmem_ld16(tq + T_PO + 64 * s + cs, p0);
                tmem_ld16(tq + T_PO + 64 * s + cs + 16, p1);
                if (trans) {
#pragma unroll
                    for (int n = 0; n < 16; ++n)
                        u0[n] = u1[n] = 0.f;
                } else {
                    tmem_ld16(tq + T_U + 64 * s + cs, u0);
                    tmem_ld16(tq + T_U + 64 * s + cs + 16, u1);
                }
                // second half of a pair: + Y E1, left by the first half's [L; Y] E product in
                // rows 64-127 of its LE buffer (complete: it was issued before this P)
                const bool corr = args.pair && (i & 1);
                float y0[16], y1[16];
                if (corr) {
                    tmem_ld16(tq + T_LE + cs, y0);
                    tmem_ld16(tq + T_LE + cs + 16, y1);
                }
                tmem_ld_wait();
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    u0[n] -= p0[n];
                    u1[n] -= p1[n];
                }
                if (corr)
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        u0[n] += y0[n];
                        u1[n] += y1[n];
                    }
                st_tile8(E_T, CC, t, cs, &u0[0]);
                st_tile8(E_T, CC, t, cs + 8, &u0[8]);
                st_tile8(E_T, CC, t, cs + 16, &u1[0]);
                st_tile8(E_T, CC, t, cs + 24, &u1[8]);
                if (scalar) {
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        u0[n] *= f;
                        u1[n] *= f;
                    }
                    st_tile8(EH_T, CC, t, cs, &u0[0]);
                    st_tile8(EH_T, CC, t, cs + 8, &u0[8]);
                    st_tile8(EH_T, CC, t, cs + 16, &u1[0]);
                    st_tile8(EH_T, CC, t, cs + 24, &u1[8]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_sync(NB_STATE, N_STATE);
            if (stid == 0)
                mbar_arrive(&bars[E_READY]);
        }
        tmem_st_wait();   // a chunk left early may still have its F S store in flight
        if (ok && nloc > 0 &&
            named_vote_or(NB_STATE, N_STATE, !wait_or_abort(&bars[UPD_DONE], (nloc - 1) & 1, abort_flag)))
            ok = false;
        // end state: S_final (whole sequence, or the last segment), Btil or Atil of a segment
        float *dst = nullptr;
        if (args.mode == MODE_SEG_AB)
            dst = trans ? args.seg_trans + (((size_t)kh * args.nseg + seg) * KD + R) * KD + n0 + cs
                        : args.seg_end + (((size_t)vh * args.nseg + seg) * KD + R) * p.dv + n0 + cs;
        else if (p.S_final != nullptr && seg == args.nseg - 1)
            dst = p.S_final + (vh * DK + R) * p.dv + n0 + cs;
        if (ok && dst != nullptr) {
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < NH; ++h) {   // rows R + 128 h (the segment buffers: dk = 128)
                float s0[16], s1[16];
                tmem_ld16(tq + T_S + 64 * h + cs, s0);
                tmem_ld16(tq + T_S + 64 * h + cs + 16, s1);
                tmem_ld_wait();
                float *d = dst + (size_t)128 * h * p.dv;
#pragma unroll
                for (int n = 0; n < 16; n += 4) {
                    *reinterpret_cast<float4 *>(d + n) = make_float4(s0[n], s0[n + 1], s0[n + 2], s0[n + 3]);
                    *reinterpret_cast<float4 *>(d + 16 + n) =
                        make_float4(s1[n], s1[n + 1], s1[n + 2], s1[n + 3]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (rows t in lanes 0-63)
        const int etid = tid - W_EPI0 * 32;
        const int t = R;
        for (int i = 0; i < nloc; ++i) {
            const int c = cbeg + i, ob = i & 1;
            const long c0 = (long)c * CC;
            const int Cl = (int)min((long)CC, T - c0);
            // Qbar S = e^{Lambda_t} (Q S) for the scalar gate (factor from the record)
            const float f = scalar ? reinterpret_cast<const float *>(
                                         args.factors + (size_t)(kh * N + c) * args.rec_bytes +
                                         prep::SC_EA)[t]
                                   : 1.f;
            if (named_vote_or(NB_EPI, N_EPI, !wait_or_abort(&bars[OUT0 + ob], (i >> 1) & 1, abort_flag)))
                break;
            tc_fence_after();
            const bool live = outputs && t < Cl;
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

// Start state of every segment: S_start(0) = S0 (or zero), S_start(g + 1) =
// Atil_g S_start(g) + Btil_g, in fp32 on the CUDA cores.  One CTA per (batch, value
// head, 16 value columns), 128 threads; thread (rb, cb) keeps rows rb, rb + 32,
// rb + 64, rb + 96 at columns 4 cb .. 4 cb + 3 of S, so that each step of the inner
// index is four float4 loads of Atil's rows and one of S's for sixteen products (the
// rows 32 apart fall in distinct bank groups).  Each output sums Btil, then the inner
// index in ascending order.  The steps are sequential, so Atil_{g+1} is copied in
// (cp.async, second buffer) and Btil_{g+1} loaded into registers while step g
// computes.
constexpr int CMB_COLS = 16, CMB_LDA = KD + 4;   // rows 16-byte aligned, 4-bank row offset
constexpr int CMB_THREADS = 128;
constexpr uint32_t CMB_SMEM = (2 * KD * CMB_LDA + KD * CMB_COLS) * 4;

__global__ void __launch_bounds__(CMB_THREADS) seg_combine_kernel(const SplitArgs a)
{
    using namespace ptx;
    extern __shared__ __align__(16) float cmb[];
    float *Ss = cmb + 2 * KD * CMB_LDA;   // S_start(g), 16 columns
    const Params &p = a.p;
    const int ncg = p.dv / CMB_COLS;
    const int cg = blockIdx.x % ncg, hv = blockIdx.x / ncg, b = blockIdx.y;
    const long vh = (long)b * p.Hv + hv, kh = (long)b * p.Hk + hv / p.R;
    const int tid = threadIdx.x, rb = tid >> 2, c4 = (tid & 3) * 4, col = cg * CMB_COLS + c4;
    auto fetch = [&](int g) {   // Atil_g into buffer g % 2
        const float *At = a.seg_trans + ((size_t)kh * a.nseg + g) * KD * KD;
        float *As = cmb + (g & 1) * KD * CMB_LDA;
        for (int u = tid; u < KD * KD / 4; u += CMB_THREADS)
            cp_async16(smem_u32(As + (u / (KD / 4)) * CMB_LDA + (u % (KD / 4)) * 4), At + 4 * u, 16u);
        cp_async_commit();
    };
    float sv[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)   // (S0 is the caller's: no alignment assumed)
            sv[i][j] = p.S0 != nullptr ? p.S0[(vh * KD + rb + 32 * i) * p.dv + col + j] : 0.f;
    // Btil_g, loaded one step ahead (its latency hides behind the step before)
    float bn[4][4];
    auto load_b = [&](int g) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 bt = *reinterpret_cast<const float4 *>(
                a.seg_end + (((size_t)vh * a.nseg + g) * KD + rb + 32 * i) * p.dv + col);
            bn[i][0] = bt.x; bn[i][1] = bt.y; bn[i][2] = bt.z; bn[i][3] = bt.w;
        }
    };
    if (a.nseg > 1) {
        fetch(0);
        load_b(0);
    }
    for (int g = 0; g < a.nseg; ++g) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float *st = a.seg_start + (((size_t)vh * a.nseg + g) * KD + rb + 32 * i) * p.dv + col;
            *reinterpret_cast<float4 *>(st) = make_float4(sv[i][0], sv[i][1], sv[i][2], sv[i][3]);
        }
        if (g + 1 == a.nseg)
            break;
        cp_async_wait_all();   // Atil_g has landed (this thread's share)
        __syncthreads();       // ... everyone's; the previous step's readers are done
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(&Ss[(rb + 32 * i) * CMB_COLS + c4]) =
                make_float4(sv[i][0], sv[i][1], sv[i][2], sv[i][3]);
        __syncthreads();
        if (g + 2 < a.nseg)
            fetch(g + 1);
        const float *As = cmb + (g & 1) * KD * CMB_LDA;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] = bn[i][j];
        if (g + 2 < a.nseg)
            load_b(g + 1);
        for (int l = 0; l < KD; l += 4) {
            float av[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 a4 = *reinterpret_cast<const float4 *>(&As[(rb + 32 * i) * CMB_LDA + l]);
                av[i][0] = a4.x; av[i][1] = a4.y; av[i][2] = a4.z; av[i][3] = a4.w;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 s4 = *reinterpret_cast<const float4 *>(&Ss[(l + u) * CMB_COLS + c4]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[i][0] += av[i][u] * s4.x;
                    acc[i][1] += av[i][u] * s4.y;
                    acc[i][2] += av[i][u] * s4.z;
                    acc[i][3] += av[i][u] * s4.w;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                sv[i][j] = acc[i][j];
    }
    cp_async_wait_all();
}

// dk = 128 with any gate grouping; dk = 256 with grouped gates (records of the
// grouped / per-channel kind: the scalar gate's record is built for dk = 128)
inline bool supports(const Params &p)
{
    return prep::supports(p) && (p.dk == KD || (p.dk == 256 && p.G > 1)) && p.dv % NVC == 0 &&
           p.G <= p.dk && p.T >= 1 && (!p.momentum || (p.dk == KD && !p.pair));
}

template <int DK, bool OB>
int launch(const Params &p, const void *factors, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, DK, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mk, p.k, DK, p.T, (long)p.B * p.Hk, CC) ||
        !make_map(&mv, p.v, p.dv, p.T, (long)p.B * p.Hv, CC))
        return 6;
    const Plan Ly = plan<DK>(p.G == 1);
    auto kern = split_kernel<DK, OB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total) !=
        cudaSuccess)
        return 6;
    SplitArgs a;
    a.p = p;
    a.factors = static_cast<const uint8_t *>(factors);
    a.rec_bytes = prep::rec_bytes(p);
    a.nvt = p.dv / NVC;
    a.nchunks = prep::nchunks(p);
    const SegPlan sp = seg_plan(p);
    a.nseg = sp.nseg;
    a.seg_len = sp.seg_len;
    a.seg_end = a.seg_trans = a.seg_start = nullptr;
    a.pair = p.pair;
    a.pair_y = prep::kind_bytes(prep::record_kind(p), p.dk) + prep::PAIR_Y;
    if (sp.nseg == 1) {
        a.mode = MODE_SEQ;
        kern<<<dim3(a.nvt * p.Hv, p.B, 1), NTHR, Ly.total, stream>>>(mq, mk, mv, a);
        return cudaGetLastError() == cudaSuccess ? 0 : 6;
    }
    // segmented: buffers past the records (sizes as seg_bytes)
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    uint8_t *w = static_cast<uint8_t *>(const_cast<void *>(factors)) + al(prep::ws_bytes(p));
    const size_t per_v = al((size_t)p.B * p.Hv * sp.nseg * KD * p.dv * 4);
    a.seg_end = reinterpret_cast<float *>(w);
    a.seg_start = reinterpret_cast<float *>(w + per_v);
    a.seg_trans = reinterpret_cast<float *>(w + 2 * per_v);
    if (cudaFuncSetAttribute(seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)CMB_SMEM) != cudaSuccess)
        return 6;
    a.mode = MODE_SEG_AB;
    kern<<<dim3(a.nvt * p.Hv + (KD / NVC) * p.Hk, p.B, sp.nseg), NTHR, Ly.total, stream>>>(mq, mk, mv, a);
    seg_combine_kernel<<<dim3((p.dv / CMB_COLS) * p.Hv, p.B), CMB_THREADS, CMB_SMEM, stream>>>(a);
    a.mode = MODE_SEG_C;
    kern<<<dim3(a.nvt * p.Hv, p.B, sp.nseg), NTHR, Ly.total, stream>>>(mq, mk, mv, a);
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

}  // namespace split
