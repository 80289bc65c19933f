// q1_gemv_tc.cu -- Q1_0_g128 matrix-vector products at M = 1 on the
// 5th-generation tensor cores (tcgen05.mma kind::i8, A operand in tensor
// memory), for one weight matrix or a group of R matrices that multiply the
// same activation vector.  Used when K is a multiple of 1024.
//
// What is computed ("Bonsai-27B-gguf technical white paper digest",
// "technical architecture highlights": one sign bit per weight, one FP16
// scale per 128 weights), for every matrix r of the group:
//     y_r[n] = sum_g d_r[n][g] * sum_{k in g} s(b_r[n][k]) * x[k],
//     s(1) = +1, s(0) = -1.
//
// Operands.  A 128-row tile of weights is the MMA's A (M = 128); each
// thread of the four expander warps owns one row, which is also its lane
// of tensor memory.  For a 128-k group it reads the row's 16 bytes of sign
// bits and, for each of the four 32-bit words q and each bit position i,
// keeps bit i of the word's four bytes with one LOP3: four u8 values
// b * 2^i.  The 32 registers (4 words x 8 positions = 128 weights) go to
// 32 tensor-memory columns with one tcgen05.st, and one 32-k MMA per word
// multiplies them.  B (N = 8) holds x as exact integers: per group x is
// scaled to 24-bit fixed point X_k = round(x_k 2^(23-E_g)), multiplied by
// 2^(7-i) to cancel the bit weight of its A slot, and split into four
// signed 8-bit limbs, one per B row; B rows 4-7 are never read back.  Each
// group accumulates into its own 8 tensor-memory columns, so
//     sum_l 256^l D_l = 2^7 sum_{k in g} b_k X_k     (exact, int32 limbs)
// and, with sum s x = 2 sum b x - sum x,
//     y += d * (2^(E_g - 29) sum_l 256^l D_l - S_g),  S_g = 2^(E_g-23) sum X_k.
//
// Pipeline (one CTA: 4 expander warps, 1 copy warp, 1 MMA warp; two CTAs
// per SM):
//   copy warp  per stage of 1024 k: the 128 rows' sign bits (16-byte
//              cp.async, into rows 144 bytes apart so that the expanders'
//              16-byte reads are free of bank conflicts), their 8 scales, and
//              (bulk copies) the stage's prepared B limbs and group constants;
//   expanders  bits -> tensor memory (A buffer ring), and the epilogue of the
//              group four steps back (tcgen05.ld of its four limb sums);
//   MMA warp   four MMAs per group, each committed to the A buffer's and the
//              accumulator slot's barriers.
// Work split: persistent CTAs take equal contiguous runs of (matrix, 128-row
// tile) over all of K; when that leaves SMs idle, K is cut into S slices,
// the S CTAs of a tile form a thread-block cluster, and their partial sums
// are added in rank order through distributed shared memory (deterministic,
// no global scratch).  Every wait is bounded (tc_common.cuh).
#include <algorithm>

#include "q1_common.cuh"
#include "tc_common.cuh"

namespace lowbit {

constexpr int kQtRows = 128;                                // rows per tile (MMA M)
constexpr int kQtGroups = 8;                                // 128-k groups per stage
constexpr int kQtStageK = kQtGroups * 128;                  // 1024
constexpr int kQtStages = 4;
constexpr int kQtRowStride = 144;                           // bytes per row of bits in a stage
constexpr int kQtOffB = kQtRows * kQtRowStride;             // prepared B limbs
constexpr int kQtBBytes = kQtStageK / 16 * 64;              // 64 chunks of 16 k x 4 limbs
constexpr int kQtOffScales = kQtOffB + kQtBBytes;           // also absorbs B's unread rows 4-7
constexpr int kQtScaleBytes = kQtRows * 16;
constexpr int kQtOffInfo = kQtOffScales + kQtScaleBytes;
constexpr int kQtInfoBytes = kQtGroups * 8;
constexpr int kQtStageBytes = (kQtOffInfo + kQtInfoBytes + 127) & ~127;
constexpr int kQtRoundGroups = 2;                           // groups per round (one A buffer, one sync)
constexpr int kQtRounds = kQtGroups / kQtRoundGroups;      // rounds per stage
constexpr int kQtNA = 3;                                    // A buffers (64 columns each)
constexpr int kQtND = 4;                                    // accumulator slots (16 columns each)
constexpr int kQtLag = 3;                                   // epilogue runs this many rounds behind
constexpr int kQtACols = kQtRoundGroups * 32;
constexpr int kQtDCols = kQtRoundGroups * 8;
constexpr int kQtColD = kQtNA * kQtACols;
constexpr int kQtTmemCols = 256;
constexpr int kQtExpWarps = 4;
constexpr int kQtCopyWarp = 4;
constexpr int kQtMmaWarp = 5;
constexpr int kQtThreads = 6 * 32;
constexpr int kQtMaxCluster = 8;
constexpr int kQtMinExp = -96;                              // activations below 2^-96 round to 0
constexpr int kQtNumBars = 2 * kQtStages + 2 * kQtNA + 2 * kQtND + 1;
constexpr int kQtOffBars = kQtStages * kQtStageBytes;
constexpr int kQtOffPart = kQtOffBars + ((kQtNumBars * 8 + 4 + 15) & ~15);
constexpr int kQtSmemBytes = kQtOffPart + kQtRows * 4;      // > 1/3 of an SM: at most two CTAs per SM

static_assert(kQtLag < kQtRounds + 1 && kQtLag < kQtND + 1, "lagged epilogue slots are static, D slots suffice");
static_assert(kQtColD + kQtND * kQtDCols <= kQtTmemCols, "tensor memory budget");
static_assert(3 * kQtSmemBytes > 228 * 1024, "two CTAs per SM at most (tensor memory is split in two)");

__device__ unsigned g_q1tc_fault;  // set when a bounded wait ran out

struct Q1TcParams {
    const uint8_t *bsrc;   // prepared B: [K/16 chunks][4 limbs][16 bytes]
    const float2 *info;    // [K/128] (2^(E-29), S)
    int N, K, blocksN, nstages, tiles;
    int S, L;              // slices per tile (cluster size) and stages per slice
};

// ---------------------------------------------------------------------------
// activation prepare: x (bf16) -> B limbs + per-group constants + bf16 copy
// ---------------------------------------------------------------------------

// One CTA of 128 threads per 128-k group; thread t is k = 128 g + t, i.e.
// bit i = t % 8 of byte jj = (t / 8) % 4 of word q = t / 32 of the group's
// 16 bytes of signs.  Its limbs go to B chunk 2 (4g + q) + i / 4, row l,
// byte 4 (i % 4) + jj: the K position of the A byte that holds its sign.
__global__ void __launch_bounds__(128) k_q1_prep_tc(const uint16_t *__restrict__ x, uint8_t *__restrict__ act,
                                                    size_t info_off, size_t xcopy_off)
{
    __shared__ float smax[4];
    __shared__ int ssum[4];
    pdl_launch_dependents();
    const int g = blockIdx.x, t = threadIdx.x, k = g * 128 + t;
    const int warp = t >> 5, lane = t & 31;
    pdl_wait_primary();  // x is produced, and act last read, by earlier kernels

    const uint16_t xb = x[k];
    reinterpret_cast<uint16_t *>(act + xcopy_off)[k] = xb;
    const float xv = bf16_bits_to_float(xb);
    const float wm = warp_max(fabsf(xv));
    if (lane == 0) smax[warp] = wm;
    __syncthreads();
    const float m = fmaxf(fmaxf(smax[0], smax[1]), fmaxf(smax[2], smax[3]));
    // E = smallest integer with m < 2^E (m normal: exponent field - 126)
    const int e8 = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    const int E = max(e8 == 0 ? kQtMinExp : e8 - 126, kQtMinExp);
    const int X = __float2int_rn(ldexpf(xv, 23 - E));  // |X| <= 2^23
    const int q = t >> 5, jj = (t >> 3) & 3, i = t & 7;
    const int V = X * (1 << (7 - i));                   // cancels the A slot weight 2^i; |V| <= 2^30
    const int l0 = (int)(int8_t)(V & 0xFF);
    int r = (V - l0) >> 8;
    const int l1 = (int)(int8_t)(r & 0xFF);
    r = (r - l1) >> 8;
    const int l2 = (int)(int8_t)(r & 0xFF);
    const int l3 = (r - l2) >> 8;                       // in [-64, 64]
    uint8_t *bdst = act + (size_t)(2 * (4 * g + q) + (i >> 2)) * 64 + 4 * (i & 3) + jj;
    bdst[0] = (uint8_t)l0;
    bdst[16] = (uint8_t)l1;
    bdst[32] = (uint8_t)l2;
    bdst[48] = (uint8_t)l3;

    const int ws = warp_sum_int(X);
    if (lane == 0) ssum[warp] = ws;
    __syncthreads();
    if (t == 0) {
        const int T = ssum[0] + ssum[1] + ssum[2] + ssum[3];  // |T| <= 2^30
        reinterpret_cast<float2 *>(act + info_off)[g] = make_float2(ldexpf(1.0f, E - 29), ldexpf((float)T, E - 23));
    }
}

// ---------------------------------------------------------------------------
// product kernel
// ---------------------------------------------------------------------------

// D (+)= A x B with A in tensor memory.  ACC (accumulate into D) is an
// immediate: a predicate computed from a register slows every MMA issue by
// tens of cycles.
template <bool ACC>
__device__ __forceinline__ void umma_i8_tmem_a(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "n"(ACC ? 1 : 0));
}

// B operand in shared memory: K-major, no swizzle; the 8-row core matrix of
// 16-byte rows starts at `addr`, the second 16-k chunk 64 bytes further on.
__device__ __forceinline__ uint64_t bdesc_noswz(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (4ull << 16) /*LBO 64 B*/ | (8ull << 32) /*SBO 128 B*/ |
           (1ull << 46) /*version*/;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 16-byte global -> shared copy; with `valid` false it writes zeros and
// reads nothing.
__device__ __forceinline__ void cp_async16_zfill(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed
// (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, unsigned parity)
{
    return mbar_wait_warp(bar, parity, &g_q1tc_fault);
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_peer_f32(const float *local, unsigned rank)
{
    unsigned ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

struct QtWork {
    int t0, t1, s_lo, ns, J;  // tiles [t0, t1), stages [s_lo, s_lo + ns) of each; J stages in all
};

__device__ __forceinline__ QtWork qt_work(const Q1TcParams &p)
{
    QtWork w;
    if (p.S == 1) {
        const long long G = gridDim.x, b = blockIdx.x;
        w.t0 = (int)(b * p.tiles / G);
        w.t1 = (int)((b + 1) * p.tiles / G);
        w.s_lo = 0;
        w.ns = p.nstages;
    } else {
        const int slice = blockIdx.x % p.S;
        w.t0 = blockIdx.x / p.S;
        w.t1 = w.t0 + 1;
        w.s_lo = slice * p.L;
        w.ns = min(p.nstages, w.s_lo + p.L) - w.s_lo;
    }
    w.J = (w.t1 - w.t0) * w.ns;
    return w;
}

__global__ void __launch_bounds__(kQtThreads, 2) k_q1_tc(const __grid_constant__ Q1Group grp, const Q1TcParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQtOffBars);
    uint64_t *empty = full + kQtStages;
    uint64_t *afull = empty + kQtStages;
    uint64_t *aempty = afull + kQtNA;
    uint64_t *dfull = aempty + kQtNA;
    uint64_t *dempty = dfull + kQtND;
    uint64_t *done = dempty + kQtND;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    float *part = reinterpret_cast<float *>(smem + kQtOffPart);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQtStages; ++s) {
            mbar_init(full + s, 32 + 1);  // 32 copy lanes' cp.async arrivals + the bulk copies' expect_tx
            mbar_init(empty + s, kQtExpWarps + 1);
        }
        for (int a = 0; a < kQtNA; ++a) {
            mbar_init(afull + a, kQtExpWarps);
            mbar_init(aempty + a, 1);
        }
        for (int d = 0; d < kQtND; ++d) {
            mbar_init(dfull + d, 1);
            mbar_init(dempty + d, kQtExpWarps);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == kQtMmaWarp) tmem_alloc(tmem_slot, kQtTmemCols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const QtWork w = qt_work(p);
    const int rowbytes = p.K >> 3, G = p.K >> 7;

    if (warp == kQtCopyWarp) {
        // ---- copies: sign bits and scales of 128 rows, prepared B, group constants ----
        // weights: 16-byte cp.async per lane, eight lanes per 128-byte row
        // (coalesced), completion signalled by each lane's noinc arrive
        auto issue_weights = [&](int j) {
            const int slot = j % kQtStages;
            const unsigned sb = smem_u32(smem + slot * kQtStageBytes);
            const int tile = w.t0 + j / w.ns, st = w.s_lo + j % w.ns;
            const int r = tile / p.blocksN, row0 = (tile - r * p.blocksN) * kQtRows;
            const int nrows = min(kQtRows, p.N - row0);
            const uint8_t *bsrc = grp.bits[r] + (size_t)row0 * rowbytes + (size_t)st * 128;
            const uint8_t *ssrc =
                reinterpret_cast<const uint8_t *>(grp.scales[r] + (size_t)row0 * G + (size_t)st * kQtGroups);
#pragma unroll 8
            for (int u = 0; u < kQtRows * 8 / 32; ++u) {
                const int c = lane + 32 * u, row = c >> 3, col = c & 7;
                const bool v = row < nrows;
                cp_async16_zfill(sb + row * kQtRowStride + col * 16, v ? bsrc + (size_t)row * rowbytes + col * 16 : bsrc,
                                 v);
            }
#pragma unroll
            for (int u = 0; u < kQtRows / 32; ++u) {
                const int row = lane + 32 * u;
                const bool v = row < nrows;
                cp_async16_zfill(sb + kQtOffScales + row * 16, v ? ssrc + (size_t)row * G * 2 : ssrc, v);
            }
            cp_async_arrive_noinc(full + slot);
        };
        // prepared activation: two bulk copies counted in transaction bytes
        auto issue_act = [&](int j) {
            const int slot = j % kQtStages;
            uint8_t *stage = smem + slot * kQtStageBytes;
            const int st = w.s_lo + j % w.ns;
            if (lane == 0) {
                mbar_arrive_expect_tx(full + slot, (unsigned)(kQtBBytes + kQtInfoBytes));
                bulk_g2s(stage + kQtOffB, p.bsrc + (size_t)st * kQtBBytes, kQtBBytes, full + slot);
                bulk_g2s(stage + kQtOffInfo, p.info + (size_t)st * kQtGroups, kQtInfoBytes, full + slot);
            }
        };
        const int pre = min(w.J, kQtStages);
        for (int j = 0; j < pre; ++j) issue_weights(j);  // weights do not depend on earlier kernels
        pdl_wait_primary();                                // the prepared activation does
        for (int j = 0; j < pre; ++j) issue_act(j);
        int issued = pre;
        for (int j = pre; j < w.J; ++j) {
            if (!warp_wait(empty + j % kQtStages, ((j / kQtStages) - 1) & 1)) break;
            issue_weights(j);
            issue_act(j);
            issued = j + 1;
        }
        // copies still in flight must land before the CTA exits (only an
        // early exit of the consumers leaves any)
        for (int j = max(0, issued - kQtStages); j < issued; ++j) warp_wait(full + j % kQtStages, (j / kQtStages) & 1);
    } else if (warp == kQtMmaWarp) {
        // ---- MMA issue: four 32-k MMAs per group into the group's accumulator slot ----
        constexpr uint32_t idesc = (2u << 4) /*s32 D*/ | (0u << 7) /*u8 A*/ | (1u << 10) /*s8 B*/ |
                                   (uint32_t)(8 >> 3) << 17 /*N = 8*/ | (uint32_t)(kQtRows >> 4) << 24 /*M*/;
        bool ok = true;
        for (int j = 0; j < w.J && ok; ++j) {
            const int slot = j % kQtStages;
            if (!warp_wait(full + slot, (j / kQtStages) & 1)) break;
            const uint32_t bbase = smem_u32(smem + slot * kQtStageBytes + kQtOffB);
#pragma unroll 1
            for (int rr = 0; rr < kQtRounds; ++rr) {
                const int r = j * kQtRounds + rr;
                const int ab = r % kQtNA, ds = r % kQtND;
                if (!warp_wait(afull + ab, (r / kQtNA) & 1) ||
                    (r >= kQtND && !warp_wait(dempty + ds, ((r / kQtND) - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int gg = 0; gg < kQtRoundGroups; ++gg) {
                        const uint32_t dcol = tmem + kQtColD + ds * kQtDCols + gg * 8;
                        const uint32_t acol = tmem + ab * kQtACols + gg * 32;
                        const uint32_t bq = bbase + 64 * 8 * (kQtRoundGroups * rr + gg);
                        umma_i8_tmem_a<false>(dcol, acol, bdesc_noswz(bq), idesc);
                        umma_i8_tmem_a<true>(dcol, acol + 8, bdesc_noswz(bq + 128), idesc);
                        umma_i8_tmem_a<true>(dcol, acol + 16, bdesc_noswz(bq + 256), idesc);
                        umma_i8_tmem_a<true>(dcol, acol + 24, bdesc_noswz(bq + 384), idesc);
                    }
                    umma_commit(aempty + ab);
                    umma_commit(dfull + ds);
                    if (rr == kQtRounds - 1) umma_commit(empty + slot);
                }
                __syncwarp();
            }
        }
        // every MMA issued has completed before tensor memory is released
        if (elect_one()) umma_commit(done);
        __syncwarp();
        warp_wait(done, 0);
    } else {
        // ---- expanders: thread t owns row t of the tile and tensor-memory lane t ----
        // A round is two groups (256 k): one A buffer, one accumulator slot.
        // Round r's accumulators are loaded before round r + kQtLag's LOP3s
        // and used after them; round r's A buffer is handed to the MMA warp
        // in round r + 1, after that round's LOP3s, so that neither the
        // tensor-memory load nor the store completion is waited for idle.
        const int t = threadIdx.x;
        const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);
        float yacc = 0.f;
        // d * 2^(E-29) and d * S per stage slot (group), for the lagged epilogue
        float qc[kQtGroups] = {}, qs[kQtGroups] = {};
        bool ok = true;
        bool waited = false;

        auto flush = [&](int tile) {
            if (!waited) {
                pdl_wait_primary();  // y may still be read by an earlier kernel
                waited = true;
            }
            if (p.S == 1) {
                const int r = tile / p.blocksN, row = (tile - r * p.blocksN) * kQtRows + t;
                if (row < p.N) grp.y[r][row] = yacc;
            } else {
                part[t] = yacc;
            }
            yacc = 0.f;
        };
        // add the limb sums of round e's groups (stage slots 2 rr_e, 2 rr_e + 1)
        auto accumulate = [&](const uint32_t (&v)[kQtDCols], int rr_e) {
#pragma unroll
            for (int gg = 0; gg < kQtRoundGroups; ++gg) {
                const int tlo = (int)v[8 * gg] + 256 * (int)v[8 * gg + 1];  // |D_l| < 2^21: both fit in int32
                const int thi = (int)v[8 * gg + 2] + 256 * (int)v[8 * gg + 3];
                const float u = fmaf((float)thi, 65536.f, (float)tlo);
                const int qsl = kQtRoundGroups * rr_e + gg;
                yacc = fmaf(qc[qsl], u, yacc - qs[qsl]);
            }
        };
        auto load_acc = [&](int e, uint32_t (&v)[kQtDCols]) -> bool {
            const int ds = e % kQtND;
            if (!warp_wait(dfull + ds, (e / kQtND) & 1)) return false;
            tc_fence_after();
            tmem_ld16(tlane + kQtColD + ds * kQtDCols, v);
            return true;
        };
        auto release_acc = [&](int e) {
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty + e % kQtND);
        };
        auto hand_over = [&](int r) {  // round r's A buffer is written: hand it to the MMA warp
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull + r % kQtNA);
        };

        for (int j = 0; j < w.J && ok; ++j) {
            const int slot = j % kQtStages;
            if (!warp_wait(full + slot, (j / kQtStages) & 1)) {
                ok = false;
                break;
            }
            const uint8_t *stage = smem + slot * kQtStageBytes;
            const uint4 sc = *reinterpret_cast<const uint4 *>(stage + kQtOffScales + t * 16);
            const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
            const bool prev_tile_end = j > 0 && (j - 1) % w.ns == w.ns - 1;
#pragma unroll
            for (int rr = 0; rr < kQtRounds; ++rr) {
                const int r = j * kQtRounds + rr;
                uint4 wb[kQtRoundGroups];
#pragma unroll
                for (int gg = 0; gg < kQtRoundGroups; ++gg)
                    wb[gg] = *reinterpret_cast<const uint4 *>(stage + t * kQtRowStride + (2 * rr + gg) * 16);
                const float4 inf = *reinterpret_cast<const float4 *>(stage + kQtOffInfo + rr * 16);
                // the epilogue's accumulator load goes out before this round's LOP3s
                uint32_t dv[kQtDCols];
                const int e = r - kQtLag;
                if (e >= 0 && !load_acc(e, dv)) {
                    ok = false;
                    break;
                }
                uint32_t a[kQtRoundGroups * 32];
#pragma unroll
                for (int gg = 0; gg < kQtRoundGroups; ++gg) {
                    const uint32_t wq[4] = {wb[gg].x, wb[gg].y, wb[gg].z, wb[gg].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int i = 0; i < 8; ++i) a[32 * gg + 8 * q + i] = wq[q] & (0x01010101u << i);
                }
                if (e >= 0) {
                    release_acc(e);
                    accumulate(dv, (rr + kQtRounds - kQtLag) % kQtRounds);
                }
                // this round's constants (after the lagged epilogue read the old ones)
#pragma unroll
                for (int gg = 0; gg < kQtRoundGroups; ++gg) {
                    const int g = 2 * rr + gg;
                    const float d = f16_bits_to_float((uint16_t)(scw[g >> 1] >> (16 * (g & 1))));
                    qc[g] = d * (gg ? inf.z : inf.x);
                    qs[g] = d * (gg ? inf.w : inf.y);
                }
                if (r >= 1) hand_over(r - 1);
                if (rr == kQtLag - 1 && prev_tile_end) flush(w.t0 + (j - 1) / w.ns);
                const int ab = r % kQtNA;
                if (r >= kQtNA && !warp_wait(aempty + ab, ((r / kQtNA) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st32(tlane + ab * kQtACols, *reinterpret_cast<const uint32_t(*)[32]>(a));
                tmem_st32(tlane + ab * kQtACols + 32, *reinterpret_cast<const uint32_t(*)[32]>(a + 32));
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // this stage's bits, scales and constants are read
        }
        if (ok && w.J > 0) {
            const int R = w.J * kQtRounds;
            hand_over(R - 1);
            // the last kQtLag rounds' epilogues, then the last tile
#pragma unroll
            for (int rr = kQtRounds - kQtLag; rr < kQtRounds; ++rr) {
                uint32_t dv[kQtDCols];
                if (ok) ok = load_acc(R - kQtRounds + rr, dv);
                if (ok) {
                    release_acc(R - kQtRounds + rr);
                    accumulate(dv, rr);
                }
            }
            if (ok) flush(w.t1 - 1);
        }
    }

    if (p.S > 1) {
        // partial sums of the S slices of this tile, added in rank order
        cluster_sync_all();
        if (warp < kQtExpWarps) {
            const int t = threadIdx.x, rank = blockIdx.x % p.S;
            if (t % p.S == rank) {
                float s = 0.f;
                for (int q = 0; q < p.S; ++q) s += ld_peer_f32(part + t, (unsigned)q);
                const int tile = blockIdx.x / p.S;
                const int r = tile / p.blocksN, row = (tile - r * p.blocksN) * kQtRows + t;
                if (row < p.N) grp.y[r][row] = s;
            }
        }
        cluster_sync_all();  // peers keep their shared memory until every rank has read it
    }
    __syncthreads();
    tc_fence_after();
    if (warp == kQtMmaWarp) tmem_dealloc(tmem, kQtTmemCols);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static int qt_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// prepared activation: B limbs (4 K bytes), group constants (8 bytes per
// 128 k), bf16 copy of x (for the CUDA-core kernels)
static size_t qt_info_off(int K) { return align256((size_t)K * 4); }
size_t q1tc_xcopy_off(int K) { return align256(qt_info_off(K) + (size_t)(K / 128) * 8); }
size_t q1tc_act_bytes(int K) { return align256(q1tc_xcopy_off(K) + (size_t)K * 2); }

bool q1tc_supported(int R, int N, int K)
{
    return R >= 1 && R <= kQ1MaxGroup && N >= 1 && K >= kQtStageK && K % kQtStageK == 0;
}

lowbit_status q1tc_prepare_launch(const uint16_t *x, int K, void *act, cudaStream_t st)
{
    cudaError_t e = launch_pdl(k_q1_prep_tc, dim3(K / 128), dim3(128), 0, st, x, static_cast<uint8_t *>(act),
                               qt_info_off(K), q1tc_xcopy_off(K));
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q1tc_gemv_launch(const uint8_t *const *bits, const uint16_t *const *scales, const void *act,
                               float *const *y, int R, int N, int K, cudaStream_t st)
{
    Q1Group grp;
    for (int r = 0; r < R; ++r) {
        grp.bits[r] = bits[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    const int sms = qt_num_sms(), slots = 2 * sms;
    Q1TcParams p = {};
    p.bsrc = static_cast<const uint8_t *>(act);
    p.info = reinterpret_cast<const float2 *>(static_cast<const uint8_t *>(act) + qt_info_off(K));
    p.N = N;
    p.K = K;
    p.blocksN = (N + kQtRows - 1) / kQtRows;
    p.nstages = K / kQtStageK;
    const long long tiles = (long long)R * p.blocksN;
    if (tiles >= (1LL << 30)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    p.tiles = (int)tiles;
    // K slices: as many as keep every (tile, slice) CTA resident at once
    int S = (int)std::min<long long>(std::min(kQtMaxCluster, p.nstages), std::max<long long>(1, slots / tiles));
    p.L = (p.nstages + S - 1) / S;
    p.S = (p.nstages + p.L - 1) / p.L;
    const long long grid = p.S > 1 ? tiles * p.S : std::min<long long>(tiles, slots);
    if (grid >= (1LL << 31)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;

    if (cudaFuncSetAttribute(k_q1_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kQtSmemBytes) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kQtThreads);
    cfg.dynamicSmemBytes = kQtSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int na = 1;
    if (p.S > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = p.S;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_q1_tc, grp, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

int q1tc_fault_flag()
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_q1tc_fault, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_q1tc_fault, &zero, sizeof(zero));
    return (int)v;
}

}  // namespace lowbit
