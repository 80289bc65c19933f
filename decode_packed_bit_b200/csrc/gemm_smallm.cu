// gemm_smallm.cu -- products at small batch on the bf16 tensor cores
// (mma.sync m16n8k16, fp32 accumulate): Q1_0_g128 for 2 <= M <= 16 and
// INT4_G64 for 2 <= M <= 32.  Both formats share the work split, the
// staging of x and the split-K reduction; they differ in how a thread turns
// its packed weights into exact bf16 A operands.
//
// What is computed ("Bonsai-27B-gguf technical white paper digest",
// "technical architecture highlights": one sign bit per weight, one FP16
// scale per 128 weights):
//     y[m][n] = sum_g d[n][g] * sum_{k in g} s(b[n][k]) * x[m][k],  s(1) = +1, s(0) = -1.
//
// Operands.  A is the weight tile with every sign as an exact bf16 +-1; B is
// x (bf16, exact); the tensor core sums the exact products in fp32, one
// accumulator per 128-k group, and the group's scale is applied once per
// (row, group, vector) with an FMA.  Inside each 16-k step the MMA's k order
// is permuted so that the four k slots a thread holds for one row (slots 2t,
// 2t+1, 2t+8, 2t+9) are the four consecutive sign bits 4t..4t+3 of the step,
// i.e. one nibble: a 16-entry shared table maps a nibble to the two bf16x2
// registers, and the matching B registers are simply x[m][k..k+3], one
// 8-byte word.
//
// Work split of one product (as for the M = 1 kernels): a warp owns 32 rows
// (two 16-row tiles); a CTA of four warps 128 rows of one K-slice; the S
// slices of a row block form a thread-block cluster and add their partial
// sums in rank order through distributed shared memory.  The CTA stages x in
// shared memory in fragment order; every warp streams its rows' packed
// weights and scales through a cp.async ring, one step (256 k for Q1_0_g128,
// 128 k for INT4_G64) at a time.  A group of products that read one x runs in
// one persistent launch instead (k_smallm_grp, at the end of this file).
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc_common.cuh"

namespace lowbit {

constexpr int kSmWarps = 4;
constexpr int kSmRows = kSmWarps * 32;     // rows per CTA
constexpr int kSmStepK = 256;              // k per pipeline step (two groups)
constexpr int kSmRowStride = 48;           // 32 bytes of signs per row, padded: conflict-free 16-byte reads
constexpr int kSmStageW = 32 * kSmRowStride;
constexpr int kSmStageBytes = kSmStageW + 32 * 4;  // + two fp16 scales per row
constexpr int kSmStages = 3;  // weight and x rings (three CTAs fit on an SM)
static_assert(kSmStages == 3, "the per-step wait depth below assumes a lookahead of two steps");
constexpr int kSmMaxM = 16;
constexpr int kSmMaxCluster = 8;
constexpr int kSmMaxSmem = 220 * 1024;

struct SmParams {
    const uint8_t *bits;
    const uint16_t *scales;
    const uint16_t *x;
    float *y;
    int M, N, K;
    int nsteps;  // K / 256
    int L;       // steps per K-slice
    int NT;      // n8 tiles of the batch (8 vectors each)
};

__device__ __forceinline__ void sm_cp16(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void sm_cp4(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void sm_cp8(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(valid ? 8 : 0) : "memory");
}
__device__ __forceinline__ void sm_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void sm_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copy step `st` (256 k) of rows blk*32..+32: lane L copies 16-byte half L%2
// of rows L/2 and L/2 + 16, and the scale pair of row L.
__device__ __forceinline__ void sm_issue(unsigned stage, const SmParams &p, int blk, int st, int lane)
{
    const int rowbytes = p.K >> 3, G = p.K >> 7;
    const int half = lane & 1, r0 = blk * 32 + (lane >> 1);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int row = r0 + 16 * u;
        const bool ok = row < p.N;
        sm_cp16(stage + ((lane >> 1) + 16 * u) * kSmRowStride + half * 16,
                ok ? p.bits + (size_t)row * rowbytes + st * 32 + half * 16 : p.bits, ok);
    }
    const int srow = blk * 32 + lane;
    const bool sok = srow < p.N;
    sm_cp4(stage + kSmStageW + lane * 4, sok ? p.scales + (size_t)srow * G + 2 * st : p.scales, sok);
}

__device__ __forceinline__ void hmma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                     uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void sm_cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float sm_ld_peer(const float *local, unsigned rank)
{
    unsigned ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"((unsigned)__cvta_generic_to_shared(local)),
                 "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

// Consume one staged step of a warp: two groups of 8 k16 steps each.
template <int NT>
__device__ __forceinline__ void sm_consume(const uint8_t *stage, const uint2 *xf, const uint2 *lut, int lane,
                                           float (&yacc)[2][NT][4])
{
    const int g = lane >> 2, t = lane & 3;
    // the signs of this lane's rows g, g+8, g+16, g+24 (32 bytes each)
    uint4 w[2][2][2];  // [tile][row g / g+8][16-byte half]
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                w[tt][r][h] = *reinterpret_cast<const uint4 *>(stage + (16 * tt + 8 * r + g) * kSmRowStride + 16 * h);
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[tt][nt][0] = acc[tt][nt][1] = acc[tt][nt][2] = acc[tt][nt][3] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const int ks = 8 * grp + s;  // k16 step within the 256-k stage: halfword ks of a row's 32 bytes
            uint2 b[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) b[nt] = xf[(ks * NT + nt) * 32 + lane];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint2 a[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint4 &q = w[tt][r][ks >> 3];
                    const uint32_t word = ((ks >> 1) & 3) == 0 ? q.x : ((ks >> 1) & 3) == 1 ? q.y
                                        : ((ks >> 1) & 3) == 2 ? q.z : q.w;
                    const uint32_t nib = (word >> (16 * (ks & 1) + 4 * t)) & 0xFu;
                    a[r] = lut[nib];
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) hmma(acc[tt][nt], a[0].x, a[1].x, a[0].y, a[1].y, b[nt].x, b[nt].y);
            }
        }
        // scale: rows g and g+8 of each tile
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const float d0 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kSmStageW + (16 * tt + g) * 4 + 2 * grp));
            const float d1 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kSmStageW + (16 * tt + 8 + g) * 4 + 2 * grp));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                yacc[tt][nt][0] = fmaf(d0, acc[tt][nt][0], yacc[tt][nt][0]);
                yacc[tt][nt][1] = fmaf(d0, acc[tt][nt][1], yacc[tt][nt][1]);
                yacc[tt][nt][2] = fmaf(d1, acc[tt][nt][2], yacc[tt][nt][2]);
                yacc[tt][nt][3] = fmaf(d1, acc[tt][nt][3], yacc[tt][nt][3]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// INT4_G64 ("acorn-llm 0.11.4", "int4 quantisation quality: group
// quantisation"): y[m][n] = sum_g d[n][g] sum_{k in g} q[n][k] x[m][k].
// A is q as an exact bf16: a thread's four k slots of a 16-k step are the two
// packed bytes 2t, 2t+1 of the row's 8 bytes (k 4t..4t+3, low nibble first),
// so B is again x[m][k..k+3].  A byte b becomes the bf16 pair {q_lo, q_hi}:
// prmt isolates b, b * 0x1001 puts its nibbles at bits 0 and 16, and with the
// sign bit of each nibble flipped (n ^ 8 = q + 8) and 0x4300 (128.0) or-ed in,
// each half reads 136 + q exactly; a bf16 subtraction of 136 leaves q.
// ---------------------------------------------------------------------------

constexpr int kI4sStepK = 128;                // k per pipeline step (two groups of 64)
constexpr int kI4sRowStride = 80;             // 64 bytes per row, padded: conflict-free 8-byte reads
constexpr int kI4sStageW = 32 * kI4sRowStride;
constexpr int kI4sStageBytes = kI4sStageW + 32 * 4;  // + two fp16 scales per row
constexpr int kI4sMaxM = 32;

// Copy step `st` (128 k) of rows blk*32..+32: lane L copies 16-byte column L%4
// of rows L/4 + {0, 8, 16, 24}, and the scale pair of row L.
__device__ __forceinline__ void i4s_issue(unsigned stage, const SmParams &p, int blk, int st, int lane)
{
    const int rowbytes = p.K >> 1, G = p.K >> 6;
    const int col = lane & 3, r0 = blk * 32 + (lane >> 2);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int row = r0 + 8 * u;
        const bool ok = row < p.N;
        sm_cp16(stage + ((lane >> 2) + 8 * u) * kI4sRowStride + col * 16,
                ok ? p.bits + (size_t)row * rowbytes + st * 64 + col * 16 : p.bits, ok);
    }
    const int srow = blk * 32 + lane;
    const bool sok = srow < p.N;
    sm_cp4(stage + kI4sStageW + lane * 4, sok ? p.scales + (size_t)srow * G + 2 * st : p.scales, sok);
}

// bf16 pair {q(low nibble), q(high nibble)} of byte `sel` (0..3) of w, exact
__device__ __forceinline__ uint32_t i4_pair_bf16(uint32_t w, uint32_t sel)
{
    const uint32_t b = __byte_perm(w, 0u, sel | 0x4440u);       // the byte alone
    const uint32_t v = ((b * 0x1001u) & 0x000F000Fu) ^ 0x43084308u;  // 136 + q in each half
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x43084308u));  // - 136
    return r;
}

template <int NT>
__device__ __forceinline__ void i4s_consume(const uint8_t *stage, const uint2 *xf, int lane, float (&yacc)[2][NT][4])
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[tt][nt][0] = acc[tt][nt][1] = acc[tt][nt][2] = acc[tt][nt][3] = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int ks = 4 * grp + s;  // k16 step within the 128-k stage: bytes 8 ks .. 8 ks + 7 of a row
            uint2 b[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) b[nt] = xf[(ks * NT + nt) * 32 + lane];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t a[2][2];  // [row g / g+8][k 4t..4t+1 / 4t+2..4t+3]
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    // this lane's two bytes: 2t, 2t+1 of the step's 8
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(
                        stage + (16 * tt + 8 * r + g) * kI4sRowStride + 8 * ks + 4 * (t >> 1));
                    const uint32_t s0 = 2u * (t & 1);
                    a[r][0] = i4_pair_bf16(w, s0);
                    a[r][1] = i4_pair_bf16(w, s0 + 1u);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    hmma(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
            }
        }
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const float d0 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kI4sStageW + (16 * tt + g) * 4 + 2 * grp));
            const float d1 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kI4sStageW + (16 * tt + 8 + g) * 4 + 2 * grp));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                yacc[tt][nt][0] = fmaf(d0, acc[tt][nt][0], yacc[tt][nt][0]);
                yacc[tt][nt][1] = fmaf(d0, acc[tt][nt][1], yacc[tt][nt][1]);
                yacc[tt][nt][2] = fmaf(d1, acc[tt][nt][2], yacc[tt][nt][2]);
                yacc[tt][nt][3] = fmaf(d1, acc[tt][nt][3], yacc[tt][nt][3]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// the kernel (both formats)
// ---------------------------------------------------------------------------
//
// grid: x = K-slice (cluster rank), y = 128-row block.  Per pipeline step the
// CTA's four warps each copy their 32 rows' packed weights into their own
// ring slot, and all 128 threads copy a share of the step's x fragments
// (k16 step ks, batch tile nt, lane (g, t) -> x[8 nt + g][k .. k+3], k = 16 ks
// + 4 t; zeros past the batch) into a CTA-wide ring.  A step is consumed
// after every thread's copies of it have landed (its own wait, then a CTA
// barrier), and that barrier also frees the slot of the previous step.

template <int FMT>
struct SmFmt;
template <>
struct SmFmt<1> {
    static constexpr int kStepK = kSmStepK, kStageBytes = kSmStageBytes;
};
template <>
struct SmFmt<3> {
    static constexpr int kStepK = kI4sStepK, kStageBytes = kI4sStageBytes;
};

template <int FMT, int NT>
__global__ void __launch_bounds__(kSmWarps * 32) k_smallm(const SmParams p)
{
    constexpr int kK16 = SmFmt<FMT>::kStepK / 16;
    constexpr int kSB = SmFmt<FMT>::kStageBytes;
    constexpr int kXFrags = kK16 * NT * 32;  // uint2 per step
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint2 lut[16];
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = blockIdx.x, nsl = gridDim.x, rb = blockIdx.y;
    const int blk = rb * kSmWarps + warp;
    const int s_lo = slice * p.L, s_hi = min(p.nsteps, s_lo + p.L);
    const int ns = max(0, s_hi - s_lo);      // steps of this CTA (the same for all its warps)
    const bool rows = blk * 32 < p.N;        // this warp has rows
    uint2 *xr = reinterpret_cast<uint2 *>(smem);                          // x ring: kSmStages x kXFrags
    uint8_t *wring = smem + (size_t)kSmStages * kXFrags * 8 + warp * kSmStages * kSB;
    float *part = reinterpret_cast<float *>(smem + (size_t)kSmStages * kXFrags * 8 + kSmWarps * kSmStages * kSB);
    const unsigned xr_s = (unsigned)__cvta_generic_to_shared(xr);
    const unsigned wr_s = (unsigned)__cvta_generic_to_shared(wring);

    auto issue_w = [&](int s) {
        if (s < ns && rows) {
            if (FMT == 1)
                sm_issue(wr_s + (s % kSmStages) * kSB, p, blk, s_lo + s, lane);
            else
                i4s_issue(wr_s + (s % kSmStages) * kSB, p, blk, s_lo + s, lane);
        }
    };
    auto issue_x = [&](int s) {
        if (s >= ns) return;
        const unsigned dst = xr_s + (unsigned)((s % kSmStages) * kXFrags) * 8u;
        for (int i = threadIdx.x; i < kXFrags; i += kSmWarps * 32) {
            const int ln = i & 31, nt = (i >> 5) % NT, ks = (i >> 5) / NT;
            const int m = 8 * nt + (ln >> 2);
            const int k = (s_lo + s) * SmFmt<FMT>::kStepK + 16 * ks + 4 * (ln & 3);
            sm_cp8(dst + 8u * i, m < p.M ? p.x + (size_t)m * p.K + k : p.x, m < p.M);
        }
    };
    // weights of the first steps go out before the previous kernel ends; x after it
#pragma unroll
    for (int t = 0; t < kSmStages - 1; ++t) {
        issue_w(t);
        sm_commit();
    }
    if (FMT == 1 && threadIdx.x < 16) {
        // nibble -> two bf16x2: bit j of the nibble is the sign of k slot 4t + j
        const uint32_t v = threadIdx.x;
        auto sg = [&](int j) -> uint32_t { return ((v >> j) & 1u) ? 0x3F80u : 0xBF80u; };
        lut[threadIdx.x] = make_uint2(sg(0) | (sg(1) << 16), sg(2) | (sg(3) << 16));
    }
    pdl_wait_primary();  // x is produced by earlier kernels
#pragma unroll
    for (int t = 0; t < kSmStages - 1; ++t) issue_x(t);
    sm_commit();

    float yacc[2][NT][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
    for (int s = 0; s < ns; ++s) {
        // this thread's copies of step s are done once at most the one group
        // committed after them is pending (at s = 0 the prologue's x group,
        // which holds step 0's x, is the newest)
        if (s == 0)
            sm_wait<0>();
        else
            sm_wait<kSmStages - 2>();
        __syncthreads();  // every thread's copies of step s landed; step s-1's slots are free
        issue_w(s + kSmStages - 1);
        issue_x(s + kSmStages - 1);
        sm_commit();
        if (rows) {
            const uint8_t *st = wring + (s % kSmStages) * kSB;
            const uint2 *xf = xr + (s % kSmStages) * kXFrags;
            if (FMT == 1)
                sm_consume<NT>(st, xf, lut, lane, yacc);
            else
                i4s_consume<NT>(st, xf, lane, yacc);
        }
    }
    sm_wait<0>();

    // partial sums of this CTA: part[m][row]; lane (g, t) holds rows 16 tt + g (+8), vectors 8 nt + 2t (+1)
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int m = 8 * nt + 2 * t + (j & 1);
                const int row = warp * 32 + 16 * tt + g + 8 * (j >> 1);
                if (m < p.M) part[m * kSmRows + row] = yacc[tt][nt][j];
            }
    if (nsl == 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < p.M * kSmRows; i += blockDim.x) {
            const int m = i / kSmRows, row = rb * kSmRows + (i - m * kSmRows);
            if (row < p.N) p.y[(size_t)m * p.N + row] = part[i];
        }
        return;
    }
    sm_cluster_sync();  // every slice's partial sums are in its CTA's shared memory
    // rank q adds up entries [q*per, (q+1)*per) over all ranks, in rank order
    const int tot = p.M * kSmRows, per = (tot + nsl - 1) / nsl;
    for (int i = slice * per + threadIdx.x; i < min(tot, (slice + 1) * per); i += blockDim.x) {
        float v[kSmMaxCluster];
#pragma unroll
        for (int q = 0; q < kSmMaxCluster; ++q) v[q] = q < nsl ? sm_ld_peer(part + i, (unsigned)q) : 0.f;
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < kSmMaxCluster; ++q) sum += v[q];
        const int m = i / kSmRows, row = rb * kSmRows + (i - m * kSmRows);
        if (row < p.N) p.y[(size_t)m * p.N + row] = sum;
    }
    sm_cluster_sync();  // peers keep their shared memory until every rank has read it
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct SmPlan {
    int nsteps, L, S, blocks, NT;
    size_t smem;
    bool ok;
};

// fmt: 1 = Q1_0_g128 (256 k per step), 3 = INT4_G64 (128 k per step)
static SmPlan sm_plan(int fmt, int M, int N, int K, int sms)
{
    SmPlan P = {};
    const int stepk = fmt == 1 ? kSmStepK : kI4sStepK, maxm = fmt == 1 ? kSmMaxM : kI4sMaxM;
    const int k16 = stepk / 16;
    P.NT = (M + 7) / 8;
    P.nsteps = K / stepk;
    P.blocks = (N + kSmRows - 1) / kSmRows;
    if (M < 2 || M > maxm || N < 1 || K % stepk != 0 || P.nsteps < 1) return P;  // ok = false
    const size_t ring = (size_t)kSmWarps * kSmStages * (fmt == 1 ? kSmStageBytes : kI4sStageBytes);
    const size_t xring = (size_t)kSmStages * k16 * P.NT * 32 * 8, part = (size_t)M * kSmRows * 4;
    // K slices: as many as keep every CTA resident in one wave (three per SM)
    P.S = (int)std::min<long long>(std::min(kSmMaxCluster, P.nsteps), std::max<long long>(1, 3LL * sms / P.blocks));
    P.L = (P.nsteps + P.S - 1) / P.S;
    P.S = (P.nsteps + P.L - 1) / P.L;
    P.smem = xring + ring + part;
    P.ok = P.smem <= (size_t)kSmMaxSmem && P.blocks < 65536;
    return P;
}

static int sm_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

bool q1sm_supported(int M, int N, int K) { return sm_plan(1, M, N, K, sm_num_sms()).ok; }
bool i4sm_supported(int M, int N, int K) { return sm_plan(3, M, N, K, sm_num_sms()).ok; }

static lowbit_status sm_launch(int fmt, const uint8_t *bits, const uint16_t *scales, const uint16_t *x, float *y,
                               int M, int N, int K, cudaStream_t st)
{
    const SmPlan P = sm_plan(fmt, M, N, K, sm_num_sms());
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    SmParams p = {};
    p.bits = bits;
    p.scales = scales;
    p.x = x;
    p.y = y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.nsteps = P.nsteps;
    p.L = P.L;
    p.NT = P.NT;
    void (*kern)(const SmParams);
    if (fmt == 1)
        kern = P.NT == 1 ? k_smallm<1, 1> : k_smallm<1, 2>;
    else
        kern = P.NT == 1 ? k_smallm<3, 1> : P.NT == 2 ? k_smallm<3, 2> : P.NT == 3 ? k_smallm<3, 3> : k_smallm<3, 4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmMaxSmem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.S, P.blocks);
    cfg.blockDim = dim3(kSmWarps * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = P.S;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q1sm_launch(const uint8_t *bits, const uint16_t *scales, const uint16_t *x, float *y, int M, int N,
                          int K, cudaStream_t st)
{
    return sm_launch(1, bits, scales, x, y, M, N, K, st);
}

lowbit_status i4sm_launch(const uint8_t *q, const uint16_t *scales, const uint16_t *x, float *y, int M, int N, int K,
                          cudaStream_t st)
{
    return sm_launch(3, q, scales, x, y, M, N, K, st);
}

// ---------------------------------------------------------------------------
// grouped persistent form: R matrices of one shape that read one x (M >= 2)
// ---------------------------------------------------------------------------
//
// One CTA per SM: nw consumer warps and one producer warp.  Every consumer
// warp owns one 32-row block of one matrix over all of K per round, and the
// rounds walk the (matrix, block) list: block (j * gridDim + blockIdx) * nw +
// warp in round j.  Weights stream through a cp.async ring per warp, so a
// warp waits only for its own copies.  x is shared through two rings:
//   raw ring (kSgRaw slots, Q1_0_g128 only): one thread of the producer
//     warp loads each step's slice of x (M rows x one step of k, one 2-D
//     tensor copy) several steps ahead;
//   x ring (kSgSlots slots): the producer warp rewrites each raw slice once,
//     in the k order the A operands below want (INT4_G64: the tensor copy
//     itself fills the slot), and signals the slot's `full` mbarrier; each
//     consumer warp signals `empty` once it has read it.
// Warps may drift apart by up to kSgSlots steps without waiting for one
// another.
//
// A operands are built in registers:
//   Q1_0_g128, no table: for a 32-bit word w of a row's signs (bits j <->
//     k0 + j), w * 2^(15-j) has bit j at bit 15 and bit j+16 at bit 31, so
//     one LOP3 (~v & 0x80008000 | 0x3F803F80) gives the bf16 pair
//     {s(j), s(j+16)}.  In MMA step sigma of a 32-k unit, lane t's slots
//     2t, 2t+1 take j = 4t + 2 sigma (and j + 16), slots 2t+8, 2t+9 take
//     j + 1 (and j + 17); x is stored as pairs P[i] = {x[k0+i], x[k0+i+16]},
//     so the B registers of both steps are one 16-byte load, P[4t .. 4t+3].
//     The multipliers come from shared memory, which keeps the products on
//     the integer multiply-add pipe and the ALU pipe free for the LOP3s.
//   INT4_G64: as in the single-matrix kernel (i4_pair_bf16), lane t's slots
//     are k 4t .. 4t+3 of a 16-k step and B is x[m][k .. k+3], so x needs no
//     rewrite: the producer's tensor copy lands it in the x ring directly,
//     each row one step of k plus 16 more (read past the step, or zero fill
//     past K), which puts rows 288 bytes (32 mod 128) apart and keeps a half
//     warp's 8-byte reads of four rows free of bank conflicts.  No raw ring.
// The sums are exact products accumulated in fp32, one accumulator per
// group (the group's first MMA starts from zero); the group's scale is
// applied once per (row, group, vector).

constexpr int kSgMaxGroup = 256;
constexpr int kSgMaxWarps = 15;  // consumer warps (16 warps with the producer: 128 registers each)
constexpr int kSgMinWarps = 8;
// Ring depths (compile-time knobs; the defaults are the measured best).
#ifndef LOWBIT_SG_SLOTS
#define LOWBIT_SG_SLOTS 6
#endif
#ifndef LOWBIT_SG_RAW
#define LOWBIT_SG_RAW 3
#endif
#ifndef LOWBIT_SG_WSTAGES
#define LOWBIT_SG_WSTAGES 3
#endif
constexpr int kSgSlots = LOWBIT_SG_SLOTS;      // x ring depth, in steps
constexpr int kSgRaw = LOWBIT_SG_RAW;          // raw ring depth, in steps
constexpr int kSgWStages = LOWBIT_SG_WSTAGES;  // weight ring depth per warp, in steps
constexpr int kSgThreadsMax = (kSgMaxWarps + 1) * 32;

__device__ unsigned g_sg_fault;  // set when a bounded wait ran out

struct SmGroup {
    const uint8_t *bits[kSgMaxGroup];
    const uint16_t *scales[kSgMaxGroup];
    float *y[kSgMaxGroup];
};

struct SmGParams {
    int M, N, K, nsteps, blocksN, nblocks, rounds;
};

// Bytes of one row of an x slot.  Q1_0_g128 (rewritten order): 64 per 32-k
// unit plus 64, so that rows sit 64 bytes (mod 128) apart and a quarter
// warp's 16-byte reads of two rows are free of bank conflicts.  INT4_G64
// (natural order, filled by the tensor copy): the step's k plus 16 more.
__host__ __device__ constexpr int sg_xrow(int fmt, int stepk) { return fmt == 1 ? stepk * 2 + 64 : (stepk + 16) * 2; }

template <int FMT>
struct SgFmt;
template <>
struct SgFmt<1> {
    static constexpr int kStepK = kSmStepK, kStageBytes = kSmStageBytes, kRowStride = kSmRowStride,
                         kStageW = kSmStageW;
};
template <>
struct SgFmt<3> {
    static constexpr int kStepK = kI4sStepK, kStageBytes = kI4sStageBytes, kRowStride = kI4sRowStride,
                         kStageW = kI4sStageW;
};

// Shared memory of the grouped kernel, in order: raw ring, x ring (both
// written by tensor copies, which want 128-byte aligned destinations: every
// slot size below is a multiple of 128), the warps' weight rings.
__host__ __device__ constexpr size_t sg_raw_bytes(int fmt, int stepk, int M)
{
    return fmt == 1 ? (size_t)kSgRaw * M * stepk * 2 : 0;
}
__host__ __device__ constexpr size_t sg_xring_bytes(int fmt, int stepk, int NT)
{
    return (size_t)kSgSlots * 8 * NT * sg_xrow(fmt, stepk);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Wait until the phase with parity `parity` of `bar` has completed; false
// (and the fault word set) after kTcWaitNs.  The clock is read once per 16
// tests.
__device__ __forceinline__ bool sg_wait(uint64_t *bar, unsigned parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kTcWaitNs) {
            atomicExch(&g_sg_fault, 1u);
            return false;
        }
    }
}

// bf16 pair {s(j), s(j+16)} of sign word w, m = 2^(15-j): one LOP3 computing
// (~(w m) & 0x80008000) | 0x3F803F80
__device__ __forceinline__ uint32_t sg_sign_pair(uint32_t w, uint32_t m)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xAE;" : "=r"(r) : "r"(w * m), "r"(0x80008000u), "r"(0x3F803F80u));
    return r;
}

// the MMA of hmma() with a zero accumulator input
__device__ __forceinline__ void hmma0(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%10,%10,%10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

template <int NT>
__device__ __forceinline__ void sg_mma(bool first, float (&acc)[NT][4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, const uint4 (&bx)[NT], int sg)
{
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = sg ? bx[nt].z : bx[nt].x, b1 = sg ? bx[nt].w : bx[nt].y;
        if (first)
            hmma0(acc[nt], a0, a1, a2, a3, b0, b1);
        else
            hmma(acc[nt], a0, a1, a2, a3, b0, b1);
    }
}

// One staged Q1_0_g128 step of a warp (two groups), x slot `xs`.
// mul[i] = 2^(15 - 4t - i).
template <int NT>
__device__ __forceinline__ void sg_consume_q1(const uint8_t *stage, const uint8_t *xs, int lane, const uint32_t (&mul)[4],
                                           float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(1, kSmStepK);
    constexpr int kRS = kSmRowStride;
    constexpr int kSW = kSmStageW;
    constexpr int kUnits = kSmStepK / 64;  // 32-k units per group
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 16 * t;
    // both groups' scales of rows 16 tt + g (+8): one 32-bit word per row
    uint32_t dw[2][2];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int r = 0; r < 2; ++r) dw[tt][r] = *reinterpret_cast<const uint32_t *>(stage + kSW + (16 * tt + 8 * r + g) * 4);
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
        uint4 w4[2][2];  // the group's 16 bytes of signs of rows 16 tt + g (+8)
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int r = 0; r < 2; ++r)
                w4[tt][r] = *reinterpret_cast<const uint4 *>(stage + (16 * tt + 8 * r + g) * kRS + 16 * grp);
#pragma unroll
        for (int cu = 0; cu < kUnits; ++cu) {
            const int c = kUnits * grp + cu;  // 32-k unit within the step
            uint4 bx[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                bx[nt] = *reinterpret_cast<const uint4 *>(xl + 8 * nt * kXR + 64 * c);
#pragma unroll
                for (int sg = 0; sg < 2; ++sg) {
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const uint32_t w0 = cu == 0 ? w4[tt][0].x : cu == 1 ? w4[tt][0].y : cu == 2 ? w4[tt][0].z : w4[tt][0].w;
                        const uint32_t w1 = cu == 0 ? w4[tt][1].x : cu == 1 ? w4[tt][1].y : cu == 2 ? w4[tt][1].z : w4[tt][1].w;
                        const uint32_t a0 = sg_sign_pair(w0, mul[2 * sg]), a2 = sg_sign_pair(w0, mul[2 * sg + 1]);
                        const uint32_t a1 = sg_sign_pair(w1, mul[2 * sg]), a3 = sg_sign_pair(w1, mul[2 * sg + 1]);
                        sg_mma<NT>(cu == 0 && sg == 0, acc[tt], a0, a1, a2, a3, bx, sg);
                    }
                }
        }
        // scale: rows g and g+8 of each tile
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const float d0 = f16_bits_to_float((uint16_t)(dw[tt][0] >> (16 * grp)));
            const float d1 = f16_bits_to_float((uint16_t)(dw[tt][1] >> (16 * grp)));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                yacc[tt][nt][0] = fmaf(d0, acc[tt][nt][0], yacc[tt][nt][0]);
                yacc[tt][nt][1] = fmaf(d0, acc[tt][nt][1], yacc[tt][nt][1]);
                yacc[tt][nt][2] = fmaf(d1, acc[tt][nt][2], yacc[tt][nt][2]);
                yacc[tt][nt][3] = fmaf(d1, acc[tt][nt][3], yacc[tt][nt][3]);
            }
        }
    }
}

// One staged INT4_G64 step of a warp (two groups), x slot `xs` in natural
// order (rows sg_xrow apart): the body of i4s_consume with the B fragments
// read straight from the slot.
template <int NT>
__device__ __forceinline__ void sg_consume_i4(const uint8_t *stage, const uint8_t *xs, int lane, float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(3, kI4sStepK);
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 8 * t;
    const uint32_t s0 = 2u * (t & 1);
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int ks = 4 * grp + s;  // 16-k step within the stage: bytes 8 ks .. 8 ks + 7 of a row
            uint2 b[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) b[nt] = *reinterpret_cast<const uint2 *>(xl + 8 * nt * kXR + 32 * ks);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t a[2][2];  // [row g / g+8][k 4t..4t+1 / 4t+2..4t+3]
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    // this lane's two bytes: 2t, 2t+1 of the step's 8
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(
                        stage + (16 * tt + 8 * r + g) * kI4sRowStride + 8 * ks + 4 * (t >> 1));
                    a[r][0] = i4_pair_bf16(w, s0);
                    a[r][1] = i4_pair_bf16(w, s0 + 1u);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (s == 0)
                        hmma0(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                    else
                        hmma(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const float d0 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kI4sStageW + (16 * tt + g) * 4 + 2 * grp));
            const float d1 = f16_bits_to_float(
                *reinterpret_cast<const uint16_t *>(stage + kI4sStageW + (16 * tt + 8 + g) * 4 + 2 * grp));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                yacc[tt][nt][0] = fmaf(d0, acc[tt][nt][0], yacc[tt][nt][0]);
                yacc[tt][nt][1] = fmaf(d0, acc[tt][nt][1], yacc[tt][nt][1]);
                yacc[tt][nt][2] = fmaf(d1, acc[tt][nt][2], yacc[tt][nt][2]);
                yacc[tt][nt][3] = fmaf(d1, acc[tt][nt][3], yacc[tt][nt][3]);
            }
        }
    }
}

// Producer task (Q1_0_g128): output chunk q (0..3) of a 32-k unit, from
// the unit's 64 raw bytes at `src` (natural order), to `dst`.  Chunk q =
// P[4q .. 4q+3], P[i] = {x[i], x[i+16]}: words 2q, 2q+1 of the low half and
// the same words 8 later, i.e. 16-byte chunks q/2 and q/2 + 2 of the unit.
__device__ __forceinline__ void sg_rewrite(const uint8_t *src, uint8_t *dst, int q)
{
    const uint4 L = *reinterpret_cast<const uint4 *>(src + 16 * (q >> 1));
    const uint4 H = *reinterpret_cast<const uint4 *>(src + 16 * (q >> 1) + 32);
    const uint32_t l0 = (q & 1) ? L.z : L.x, l1 = (q & 1) ? L.w : L.y;
    const uint32_t h0 = (q & 1) ? H.z : H.x, h1 = (q & 1) ? H.w : H.y;
    *reinterpret_cast<uint4 *>(dst) =
        make_uint4(prmt(l0, h0, 0x5410u), prmt(l0, h0, 0x7632u), prmt(l1, h1, 0x5410u), prmt(l1, h1, 0x7632u));
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kSgThreadsMax, 1) k_smallm_grp(const __grid_constant__ SmGroup grp,
                                                                 const __grid_constant__ CUtensorMap xmap,
                                                                 const SmGParams q)
{
    constexpr int kStepK = SgFmt<FMT>::kStepK;
    constexpr int kSB = SgFmt<FMT>::kStageBytes;
    constexpr int kXR = sg_xrow(FMT, kStepK);
    constexpr int kXSlot = 8 * NT * kXR;
    constexpr int kUnitsStep = kStepK / 32;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // the tensor copies into the raw ring want a 128-byte aligned destination
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bars[2 * kSgSlots + kSgRaw];  // full[s], empty[s], raw[s]
    __shared__ uint32_t multab[4][4];
    uint64_t *full = bars, *empty = bars + kSgSlots, *rawbar = bars + 2 * kSgSlots;
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x >> 5) - 1;
    const int total = q.rounds * q.nsteps;  // (round, step) sequence of every warp
    const int rawslot = q.M * kStepK * 2;
    uint8_t *raw = smem;
    uint8_t *xring = smem + sg_raw_bytes(FMT, kStepK, q.M);

    // rows M .. 8 NT - 1 of every x slot stay zero; barriers; multipliers
    {
        const int zrows = 8 * NT - q.M;
        for (int i = threadIdx.x; i < kSgSlots * zrows * (kXR / 16); i += blockDim.x) {
            const int sl = i / (zrows * (kXR / 16)), rem = i - sl * zrows * (kXR / 16);
            const int row = q.M + rem / (kXR / 16), col = rem % (kXR / 16);
            *reinterpret_cast<uint4 *>(xring + sl * kXSlot + row * kXR + 16 * col) = make_uint4(0, 0, 0, 0);
        }
        if (threadIdx.x < 16) multab[threadIdx.x >> 2][threadIdx.x & 3] = 1u << (15 - 4 * (threadIdx.x >> 2) - (threadIdx.x & 3));
        if (threadIdx.x == 0) {
            for (int s = 0; s < kSgSlots; ++s) {
                mbar_init(full + s, FMT == 1 ? 32 : 1);  // the rewriting lanes, or the copying thread
                mbar_init(empty + s, (unsigned)nw);
            }
            for (int s = 0; s < kSgRaw; ++s) mbar_init(rawbar + s, 1);
            mbar_fence_init();
        }
        __syncthreads();
    }

    if (warp == nw) {
        pdl_wait_primary();  // x is produced by earlier kernels
        if (FMT == 3) {
            // ---- producer (INT4_G64): one tensor copy per step straight into the x ring
            if (lane == 0) {
                const unsigned bytes = (unsigned)(q.M * kXR);
                for (int u = 0; u < total; ++u) {
                    const int sl = u % kSgSlots;
                    if (u >= kSgSlots && !sg_wait(empty + sl, ((u / kSgSlots) - 1) & 1)) break;
                    mbar_arrive_expect_tx(full + sl, bytes);
                    tma_load_2d(xring + sl * kXSlot, &xmap, (u % q.nsteps) * kStepK, 0, full + sl);
                }
            }
            return;
        }
        // ---- producer (Q1_0_g128): raw slices by tensor copy, rewritten once into the x ring
        auto copy_raw = [&](int v) {  // lane 0: step v of the sequence into raw slot v % kSgRaw
            if (v >= total) return;
            uint64_t *bar = rawbar + v % kSgRaw;
            mbar_arrive_expect_tx(bar, (unsigned)rawslot);
            tma_load_2d(raw + (v % kSgRaw) * rawslot, &xmap, (v % q.nsteps) * kStepK, 0, bar);
        };
        if (lane == 0)
            for (int v = 0; v < kSgRaw; ++v) copy_raw(v);
        // task T = (unit item T/4 = (row n, unit c), output chunk T%4); a
        // quarter warp covers two adjacent units: 128 contiguous bytes each way
        const int tasks = q.M * kUnitsStep * 4;
        constexpr int kUn = 4;
        for (int u = 0; u < total; ++u) {
            const int sl = u % kSgSlots, rs = u % kSgRaw;
            bool ok = u < kSgSlots || sg_wait(empty + sl, ((u / kSgSlots) - 1) & 1);
            ok = ok && sg_wait(rawbar + rs, (u / kSgRaw) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            const uint8_t *rsrc = raw + rs * rawslot;
            uint8_t *xdst = xring + sl * kXSlot;
            for (int base = 0; base < tasks; base += 32 * kUn) {
#pragma unroll
                for (int i = 0; i < kUn; ++i) {
                    const int T = base + 32 * i + lane;
                    if (T < tasks) {
                        const int item = T >> 2, n = item / kUnitsStep, c = item - n * kUnitsStep;
                        sg_rewrite(rsrc + n * kStepK * 2 + 64 * c, xdst + n * kXR + 64 * c + 16 * (T & 3), T & 3);
                    }
                }
            }
            mbar_arrive(full + sl);
            // the raw slot's reads are done: it may be refilled (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) copy_raw(u + kSgRaw);
        }
        return;
    }

    // ---- consumers
    uint8_t *wring = xring + sg_xring_bytes(FMT, kStepK, NT) + (size_t)warp * kSgWStages * kSB;
    const unsigned wr_s = (unsigned)__cvta_generic_to_shared(wring);
    uint32_t mul[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mul[i] = multab[lane & 3][i];

    // Copy cursor: the (round, step) whose weights go out next and this
    // lane's sources for it.  Q1_0_g128: 16-byte half L%2 of rows L/2 and
    // L/2 + 16; INT4_G64: 16-byte column L%4 of rows L/4 + {0, 8, 16, 24};
    // both: the scale pair of row L.  Rows past N copy nothing (zero fill).
    constexpr int kCopies = FMT == 1 ? 2 : 4;
    constexpr int kStepBytes = kStepK / (FMT == 1 ? 8 : 2);  // packed bytes of a row per step
    const int rowbytes = q.K / (FMT == 1 ? 8 : 2), G = q.K / (FMT == 1 ? 128 : 64);
    // copy c lands kDstStride * c bytes after copy 0 within a stage
    constexpr unsigned kDstStride = FMT == 1 ? 16 * kSmRowStride : 8 * kI4sRowStride;
    const unsigned wdst0 = FMT == 1 ? (unsigned)((lane >> 1) * kSmRowStride + (lane & 1) * 16)
                                    : (unsigned)((lane >> 2) * kI4sRowStride + (lane & 3) * 16);
    const unsigned sdst = (unsigned)(SgFmt<FMT>::kStageW + lane * 4);
    int cj = 0, cs = 0, cstage = 0;  // copy cursor: round, step, ring stage
    bool clive = false;
    const uint8_t *csrc = nullptr;  // copy 0's row; copy c reads c * cstride bytes further
    const uint16_t *cscale = nullptr;
    const unsigned cstride = (unsigned)((FMT == 1 ? 16 : 8) * rowbytes);
    unsigned cok = 0;  // bit c: copy c reads a row < N; bit kCopies: the scale row
    auto set_round = [&](int j) {
        cj = j;
        cs = 0;
        const int b = (j * (int)gridDim.x + (int)blockIdx.x) * nw + warp;
        clive = j < q.rounds && b < q.nblocks;
        if (!clive) return;
        const int r = b / q.blocksN, blk = b - r * q.blocksN;
        const int r0 = blk * 32 + (FMT == 1 ? (lane >> 1) : (lane >> 2));
        cok = 0;
#pragma unroll
        for (int c = 0; c < kCopies; ++c) cok |= (r0 + (FMT == 1 ? 16 : 8) * c < q.N ? 1u : 0u) << c;
        csrc = grp.bits[r] + (size_t)r0 * rowbytes + (lane & (FMT == 1 ? 1 : 3)) * 16;
        const int srow = blk * 32 + lane;
        cok |= (srow < q.N ? 1u : 0u) << kCopies;
        cscale = grp.scales[r] + (srow < q.N ? (size_t)srow * G : 0);
    };
    auto issue_next = [&]() {  // one commit group per call, empty past the end
        if (clive) {
            const unsigned st = wr_s + cstage * kSB;
#pragma unroll
            for (int c = 0; c < kCopies; ++c) {
                const bool ok = (cok >> c) & 1u;
                sm_cp16(st + wdst0 + kDstStride * c, ok ? csrc + c * cstride + cs * kStepBytes : grp.bits[0], ok);
            }
            const bool sok = (cok >> kCopies) & 1u;
            sm_cp4(st + sdst, sok ? cscale + 2 * cs : cscale, sok);
        }
        sm_commit();
        cstage = cstage + 1 == kSgWStages ? 0 : cstage + 1;
        if (++cs == q.nsteps) set_round(cj + 1);
    };
    set_round(0);
#pragma unroll
    for (int t = 0; t < kSgWStages - 1; ++t) issue_next();
    pdl_wait_primary();  // y was last read by earlier kernels

    float yacc[2][NT][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
    const int g = lane >> 2, t4 = lane & 3;
    int sl = 0, stage = 0, s = 0, j = 0;
    unsigned phase = 0;
    int b = blockIdx.x * nw + warp;  // block of round j
    for (int u = 0; u < total; ++u) {
        issue_next();
        if (!__all_sync(0xffffffffu, sg_wait(full + sl, phase))) break;
        sm_wait<kSgWStages - 1>();  // this lane's copies of step u landed
        __syncwarp();               // ... and every lane's
        if (b < q.nblocks) {
            if (FMT == 1)
                sg_consume_q1<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, mul, yacc);
            else
                sg_consume_i4<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, yacc);
        }
        __syncwarp();  // every lane has read the slot and the stage
        if (lane == 0) mbar_arrive(empty + sl);
        if (++sl == kSgSlots) {
            sl = 0;
            phase ^= 1u;
        }
        stage = stage + 1 == kSgWStages ? 0 : stage + 1;
        if (++s == q.nsteps) {
            if (b < q.nblocks) {
                const int r = b / q.blocksN, blk = b - r * q.blocksN;
                float *y = grp.y[r];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int m = 8 * nt + 2 * t4 + (e & 1);
                            const int row = blk * 32 + 16 * tt + g + 8 * (e >> 1);
                            if (m < q.M && row < q.N) y[(size_t)m * q.N + row] = yacc[tt][nt][e];
                        }
            }
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
            s = 0;
            ++j;
            b += (int)gridDim.x * nw;
        }
    }
    sm_wait<0>();
}

struct SgPlan {
    int nsteps, blocksN, nblocks, warps, rounds, NT;
    size_t smem;
    bool ok;
};

// Consumer warps per CTA: as many as fit (<= kSgMaxWarps), then the count in
// [kSgMinWarps, max] whose rounds come out fullest (ties: more warps).
static SgPlan sg_plan(int fmt, int R, int M, int N, int K, int sms)
{
    SgPlan P = {};
    const int stepk = fmt == 1 ? kSmStepK : kI4sStepK, maxm = fmt == 1 ? kSmMaxM : kI4sMaxM;
    if (R < 1 || R > kSgMaxGroup || M < 2 || M > maxm || N < 1 || K % stepk != 0 || K < stepk) return P;
    P.NT = (M + 7) / 8;
    P.nsteps = K / stepk;
    P.blocksN = (N + 31) / 32;
    P.nblocks = R * P.blocksN;
    const size_t xring = sg_raw_bytes(fmt, stepk, M) + sg_xring_bytes(fmt, stepk, P.NT);
    const size_t per_warp = (size_t)kSgWStages * (fmt == 1 ? kSmStageBytes : kI4sStageBytes);
    if (128 + xring + kSgMinWarps * per_warp > (size_t)kSmMaxSmem) return P;
    const int fit = (int)std::min<size_t>(kSgMaxWarps, ((size_t)kSmMaxSmem - 128 - xring) / per_warp);
    double best = -1.0;
    for (int w = fit; w >= kSgMinWarps; --w) {
        if ((long long)P.nblocks < (long long)sms * w) continue;  // at least one full round
        const int rounds = (int)((P.nblocks + (long long)sms * w - 1) / ((long long)sms * w));
        const double eff = (double)P.nblocks / ((double)rounds * sms * w);
        if (eff > best + 1e-9) {
            best = eff;
            P.warps = w;
            P.rounds = rounds;
        }
    }
    P.smem = 128 /*alignment*/ + xring + (size_t)P.warps * per_warp;
    P.ok = P.warps >= kSgMinWarps;
    return P;
}

bool smg_supported(int fmt, int R, int M, int N, int K) { return sg_plan(fmt, R, M, N, K, sm_num_sms()).ok; }

lowbit_status smg_launch(int fmt, const uint8_t *const *bits, const uint16_t *const *scales, const uint16_t *x,
                         float *const *y, int R, int M, int N, int K, cudaStream_t st)
{
    const int sms = sm_num_sms();
    const SgPlan P = sg_plan(fmt, R, M, N, K, sms);
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    static SmGroup grp;  // large: kept off the stack
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int r = 0; r < R; ++r) {
        grp.bits[r] = bits[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return LOWBIT_ERR_CUDA;
    // x [M][K] bf16; one box = the M rows of one step of k (Q1_0_g128, into
    // the raw ring) or of one step plus 16 (INT4_G64, the x ring's row
    // stride), rows dense in shared memory; k past K reads as zero
    CUtensorMap xmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)(fmt == 1 ? kSmStepK : sg_xrow(3, kI4sStepK) / 2), (cuuint32_t)M};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LOWBIT_ERR_CUDA;
    SmGParams q = {};
    q.M = M;
    q.N = N;
    q.K = K;
    q.nsteps = P.nsteps;
    q.blocksN = P.blocksN;
    q.nblocks = P.nblocks;
    q.rounds = P.rounds;
    void (*kern)(const SmGroup, const CUtensorMap, const SmGParams);
    if (fmt == 1)
        kern = P.NT == 1 ? k_smallm_grp<1, 1> : k_smallm_grp<1, 2>;
    else
        kern = P.NT == 1 ? k_smallm_grp<3, 1>
             : P.NT == 2 ? k_smallm_grp<3, 2>
             : P.NT == 3 ? k_smallm_grp<3, 3>
                         : k_smallm_grp<3, 4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3((P.warps + 1) * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, grp, xmap, q);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// Read and clear the fault flag of the current device.
int smg_fault_flag()
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_sg_fault, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_sg_fault, &zero, sizeof(zero));
    return v != 0;
}

}  // namespace lowbit
