// q1_gemv_m1.cu -- Q1_0_g128 products at M = 1 (and, in the persistent
// kernel, M = 2..4) on the integer tensor cores (mma.sync m16n8k32, u8 x s8
// -> s32), for one weight matrix or a group of R matrices that multiply the
// same activation; and the one-launch decode step through a stack of them.
//
// What is computed ("Bonsai-27B-gguf technical white paper digest",
// "technical architecture highlights": one sign bit per weight, one FP16
// scale per 128 weights), for every matrix r of the group:
//     y_r[n] = sum_g d_r[n][g] * sum_{k in g} s(b_r[n][k]) * x[k],
//     s(1) = +1, s(0) = -1.
//
// Why tensor cores for a matrix-vector product: at 0.140625 bytes per weight
// HBM delivers more weights per second than the SM's 32-bit lanes can each
// touch once, so the inner loop must consume several weights per
// instruction.  The kernels feed raw sign bits to the integer tensor cores:
//
//   A operand: for bit position i (1..7) one lop3 keeps bit i of each of the
//     four bytes of a 32-bit word of packed signs, giving four u8 values
//     b_i*2^i -- four weights per instruction, no shifts, no table.  Plane 0
//     takes the packed bytes themselves, w = sum_i b_i 2^i, with no
//     instruction: seven masks per eight bit planes.
//   B operand: x rewritten exactly as integers.  Per 128-group, x is scaled
//     to 24-bit fixed point X_k = round(x_k * 2^(23-E_g)) (E_g = the group's
//     binary exponent ceiling).  For a byte whose bit i is weight k_i, plane
//     0 carries Y_0 = 2^7 X_{k_0} and plane i >= 1 carries
//     Y_i = 2^(7-i) X_{k_i} - 2^7 X_{k_0}, so that
//         w Y_0 + sum_{i>=1} (b_i 2^i) Y_i = 2^7 sum_i b_i X_{k_i}
//     (the bits of w in plane 0 are taken back out by the -2^7 X_{k_0} of
//     the other planes).  |Y| < 2^30 + 2^29; each Y is split into four
//     signed 8-bit limbs, one limb per B column, and each D column holds its
//     limb's share exactly in int32 (|D| < 16 * 509 * 128 < 2^20).
//   Two groups share one accumulator: B columns 0-3 carry the four limbs of
//     the first group of a 256-k chunk, columns 4-7 those of the second.  A
//     lane's B registers are zero whenever its column group differs from the
//     group of its k slots, so only 16 of the 32 lanes' fragments are stored
//     (1 KB per chunk); the other lanes read a zero block.
//   Epilogue per (row, group): 2^7 sum_k b X = sum_l D_l 2^(8l); the signed
//     sum is sum s x = 2 sum b x - sum x.  Lane quarter tq holds the limb
//     pair 2(tq&1), 2(tq&1)+1 of group tq>>1; it forms v = D_lo + 256 D_hi in
//     int32 (|v| < 2^29), converts it once, and adds d * (c_tq v + n_tq),
//     with c_tq = 2^(E-29) (times 2^16 for the high pair) and n_tq = -2^(E-23)
//     sum_k X_k for the low pair (0 for the high pair).  Integer-exact up to
//     the 24-bit rounding of x and the fp32 epilogue.
//
// Weight streaming: each warp owns a ring of shared-memory stages filled by
// cp.async, so the stages after the one being consumed are always in flight,
// and each B fragment read from shared memory feeds two 16-row mma tiles.
// The first stages are issued before griddepcontrol.wait, which lets the
// weight stream of a launch overlap the tail of the previous kernel.
//
// Work splits:
//   persistent kernel (k_q1_m1_lean; groups with at least 8 32-row blocks
//     per SM, K % 1024 == 0): one CTA per SM takes an equal range of (matrix,
//     32-row block) cells over all of K, cut into equal per-warp ranges of
//     1024-k steps; the activation of MV = 1, 2 or 4 vectors sits in shared
//     memory, built from x by every CTA or staged from a prepared copy.
//   stream kernel (other groups with many 32-row blocks): the older
//     persistent form with 512-k steps and whole cells per warp.
//   split kernel (too few tiles to fill the GPU, e.g. one matrix): K is cut
//     into S <= 8 slices, the S CTAs of one 128-row block form a thread-block
//     cluster, and their partial sums are added in fixed rank order through
//     distributed shared memory (deterministic, no global scratch).
#include <algorithm>
#include <mutex>

#include "q1_common.cuh"

namespace lowbit {

constexpr int kQ1ChunkK = 256;
constexpr int kQ1FragBytesPerChunk = 1024;  // 8 mma x 16 live lanes x 8 bytes
constexpr int kQ1InfoBytesPerChunk = 32;    // four lane quarters x (c, n) floats
constexpr int kQ1ZeroBytes = 4096;          // zero block read by the dead lanes (covers a 4-chunk step)
// Inside a chunk's fragments, the live entries e = 0..15 of the mmas 2j and
// 2j+1 sit side by side (16 bytes per entry), so one 16-byte load fetches a
// lane's B registers for two bit planes.
#ifndef LOWBIT_Q1_BPAIR
#define LOWBIT_Q1_BPAIR 1
#endif
constexpr int kQ1FragLaneStride = LOWBIT_Q1_BPAIR ? 16 : 8;  // bytes between live entries
// offset of mma i's fragment from a lane's base (entry e at e * kQ1FragLaneStride)
__host__ __device__ constexpr int q1_frag_plane(int i) { return LOWBIT_Q1_BPAIR ? (i >> 1) * 256 + (i & 1) * 8 : i * 128; }
// Tuning knobs (compile-time; the defaults are the measured best).
#ifndef LOWBIT_Q1_WARPS
#define LOWBIT_Q1_WARPS 8
#endif
#ifndef LOWBIT_Q1_STAGES
#define LOWBIT_Q1_STAGES 3
#endif
constexpr int kQ1Warps = LOWBIT_Q1_WARPS;
constexpr int kQ1MinExp = -96;              // activations below 2^-96 round to 0
constexpr int kQ1MaxSmem = 226 * 1024;     // dynamic part; leaves room for static smem
constexpr int kQ1MaxCluster = 8;




// ---------------------------------------------------------------------------
// activation prepare: x (bf16) -> limb fragments + per-lane epilogue constants
// ---------------------------------------------------------------------------

// The two epilogue constant pairs of one group (lane quarters 2h, 2h+1).
__device__ __forceinline__ void q1_write_info(float2 *dst, bool exists, int E, int T)
{
    float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
    if (exists) {
        lo = make_float2(ldexpf(1.0f, E - 29), -ldexpf((float)T, E - 23));
        hi = make_float2(ldexpf(1.0f, E - 13), 0.f);
    }
    dst[0] = lo;
    dst[1] = hi;
}

// B fragment of live entry e (0..15) of mma i, from a chunk's limbs
// lb[limb][k - 256 ch].  Entry e is the lane with k quarter t = e & 3 and
// column 4 (t >> 1) + (e >> 2), i.e. limb e >> 2 of the group of its k slots.
// Register j, byte c holds B[k-slot 16j + 4t + c]; k-slot 16j + 4t + c of mma
// i carries bit i of packed byte 8t + 4j + c of the row's 32-byte chunk, i.e.
// k = 64t + 32j + 8c + i.
__device__ __forceinline__ uint2 q1_fragment(const int8_t (*lb)[256], int i, int e)
{
    const int t = e & 3;
    const int8_t *l = lb[e >> 2];
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) w[j] |= (uint32_t)(uint8_t)l[64 * t + 32 * j + 8 * c + i] << (8 * c);
    return make_uint2(w[0], w[1]);
}

// The B value of weight k in bit plane i = k & 7, from its fixed-point x X
// and X0, that of the byte's plane-0 weight k & ~7: 2^7 X0 for i = 0, else
// 2^(7-i) X - 2^7 X0.  |X|, |X0| <= 2^23 give |result| <= 2^30 + 2^29.
__device__ __forceinline__ int q1_plane_value(int X, int X0, int i)
{
    return i == 0 ? X * 128 : X * (1 << (7 - i)) - X0 * 128;
}

// One CTA of 256 threads per 256-k chunk.  Thread kk first turns x[k] into
// four limbs; then thread t < 128 writes the 8-byte B fragment of live entry
// t%16 for mma t/16.  A plain bf16 copy of x is kept after the fragments for
// shapes the tensor kernels do not take (K/128 odd), which the SIMT kernel
// reads.
__global__ void __launch_bounds__(256) k_q1_prep_m1(const uint16_t *__restrict__ x, int K,
                                                    uint8_t *__restrict__ act, size_t info_off,
                                                    size_t xcopy_off)
{
    __shared__ float smax[8];
    __shared__ int ssum[8];
    __shared__ int8_t limb[4][256];
    pdl_launch_dependents();
    const int ch = blockIdx.x;
    const int kk = threadIdx.x;
    const int k = ch * kQ1ChunkK + kk;
    const int warp = kk >> 5, lane = kk & 31;
    const int h = kk >> 7;  // group of this k within the chunk
    pdl_wait_primary();     // x is produced, and act last read, by earlier kernels

    const uint16_t xb = k < K ? x[k] : (uint16_t)0;
    if (k < K) reinterpret_cast<uint16_t *>(act + xcopy_off)[k] = xb;
    const float xv = bf16_bits_to_float(xb);
    const float wm = warp_max_nonneg(fmaxf(0.f, fabsf(xv)));
    if (lane == 0) smax[warp] = wm;
    __syncthreads();
    const float m = fmaxf(fmaxf(smax[4 * h], smax[4 * h + 1]), fmaxf(smax[4 * h + 2], smax[4 * h + 3]));
    // E = smallest integer with m < 2^E (m normal: exponent field - 126)
    const int e8 = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    const int E = max(e8 == 0 ? kQ1MinExp : e8 - 126, kQ1MinExp);
    const int X = __float2int_rn(ldexpf(xv, 23 - E));       // |X| <= 2^23
    // k & 7 == lane & 7: the byte's plane-0 weight is in lane (lane & ~7)
    const int B = q1_plane_value(X, __shfl_sync(0xffffffffu, X, lane & ~7), k & 7);
    int l0 = (int)(int8_t)(B & 0xFF);
    int r = (B - l0) >> 8;
    int l1 = (int)(int8_t)(r & 0xFF);
    r = (r - l1) >> 8;
    int l2 = (int)(int8_t)(r & 0xFF);
    const int l3 = (r - l2) >> 8;                           // |B| <= 2^30 + 2^29 keeps it in [-97, 97]
    limb[0][kk] = (int8_t)l0;
    limb[1][kk] = (int8_t)l1;
    limb[2][kk] = (int8_t)l2;
    limb[3][kk] = (int8_t)l3;

    const int ws = warp_sum_int(X);
    if (lane == 0) ssum[warp] = ws;
    __syncthreads();
    if ((kk & 127) == 0) {
        const int T = ssum[4 * h] + ssum[4 * h + 1] + ssum[4 * h + 2] + ssum[4 * h + 3];  // |T| < 2^30
        q1_write_info(reinterpret_cast<float2 *>(act + info_off) + 4 * ch + 2 * h, (2 * ch + h) * 128 < K, E, T);
    }
    if (kk < 128) {
        const uint2 f = q1_fragment(limb, kk >> 4, kk & 15);
        const int i = kk >> 4, e = kk & 15;
        *reinterpret_cast<uint2 *>(act + (size_t)ch * kQ1FragBytesPerChunk + e * kQ1FragLaneStride + q1_frag_plane(i)) = f;
    }
}

// ---------------------------------------------------------------------------
// shared pieces of the product kernels
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the same with a zero accumulator input
__device__ __forceinline__ void mma_u8s8_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%10,%10,%10};"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// Asynchronous global -> shared copies (shared address given as a 32-bit
// shared-window address); a copy with `valid` false writes zeros and reads
// nothing.
__device__ __forceinline__ void cp_async16(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A step is 32 rows (two 16-row mma tiles) x 2 chunks: 64 bytes of each row.
// In a stage the rows sit 96 bytes apart, which keeps the consumers' 8-byte
// reads free of bank conflicts; the 32 x 2 fp16 scale pairs follow.
constexpr int kQ1StepRows = 32;
constexpr int kQ1StepChunks = 2;
constexpr int kQ1Stages = LOWBIT_Q1_STAGES;
constexpr int kQ1RowStride = 96;
constexpr int kQ1StageW = kQ1StepRows * kQ1RowStride;
constexpr int kQ1StageBytes = kQ1StageW + kQ1StepRows * 8;
constexpr int kQ1WarpRing = kQ1Stages * kQ1StageBytes;
constexpr int kQ1SplitWarps = 4;

struct Q1Params {
    const uint8_t *act;
    const uint16_t *x;  // split kernel: build the activation from x itself (act unused)
    size_t info_off;
    int R, N, K, nchunks;
    int M;              // lean kernel: vectors of x (<= its MV)
    int L;              // chunks per K-slice (split kernel) or nchunks (stream kernel)
    int blocksN;        // 32-row blocks per matrix
    int cells;          // stream kernel: R * blocksN
    int act_smem;       // bytes reserved for staged activation chunks
};

// Issue the copies of one step into the stage at shared address `stage`:
// rows blk*32..+32 of matrix r, chunks ch0, ch0+1 (only those < chend).
// Lane L copies the 16-byte column L%4 of rows L/4 + {0,8,16,24} and the fp16
// scale pair of chunk L%2 of rows L/2 + {0,16}.  FULL: no bounds tests.
template <bool FULL>
__device__ __forceinline__ void issue_step(unsigned stage, const Q1Group &grp, const Q1Params &p, int r, int blk,
                                           int ch0, int chend, int lane)
{
    const int rowbytes = p.K >> 3, G = p.K >> 7;
    const int col = lane & 3, c = col >> 1;
    const int row0 = blk * kQ1StepRows + (lane >> 2);
    const uint8_t *bsrc = grp.bits[r] + (size_t)row0 * rowbytes + ch0 * 32 + col * 16;
    const unsigned bdst = stage + (lane >> 2) * kQ1RowStride + col * 16;
    const bool cok = FULL || (ch0 + c < chend && ch0 * 32 + col * 16 + 16 <= rowbytes);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const bool ok = FULL || (cok && row0 + 8 * u < p.N);
        cp_async16(bdst + 8 * u * kQ1RowStride, ok ? bsrc + (size_t)(8 * u) * rowbytes : grp.bits[r], ok);
    }
    const int sc = lane & 1;
    const int srow0 = blk * kQ1StepRows + (lane >> 1);
    const uint16_t *ssrc = grp.scales[r] + (size_t)srow0 * G + 2 * (ch0 + sc);
    const unsigned sdst = stage + kQ1StageW + (lane >> 1) * 8 + sc * 4;
    const bool sok = FULL || (ch0 + sc < chend && 2 * (ch0 + sc) < G);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const bool ok = FULL || (sok && srow0 + 16 * u < p.N);
        cp_async4(sdst + 16 * u * 8, ok ? ssrc + (size_t)(16 * u) * G : grp.scales[r], ok);
    }
}

__device__ __forceinline__ void issue_any(unsigned stage, const Q1Group &grp, const Q1Params &p, int r, int blk,
                                          int ch0, int chend, int lane)
{
    const bool full = ch0 + kQ1StepChunks <= chend && blk * kQ1StepRows + kQ1StepRows <= p.N &&
                      (ch0 + kQ1StepChunks) * 256 <= p.K;
    if (full)
        issue_step<true>(stage, grp, p, r, blk, ch0, chend, lane);
    else
        issue_step<false>(stage, grp, p, r, blk, ch0, chend, lane);
}

struct LaneConst {
    int woff, soff;     // offsets inside a stage (row g of tile 0, chunk 0)
    int tq, h;
    int e;              // fragment entry this lane reads (lane & 15)
    bool live;          // its column group is the group of its k slots
};

__device__ __forceinline__ LaneConst lane_const(int lane)
{
    LaneConst lc;
    const int g = lane >> 2;
    lc.tq = lane & 3;
    lc.h = lc.tq >> 1;
    lc.woff = g * kQ1RowStride + lc.tq * 8;
    lc.soff = kQ1StageW + g * 8 + lc.h * 2;
    lc.e = lane & 15;
    lc.live = (lane >> 4) == lc.h;
    return lc;
}

// The B fragment base of a step: a live lane reads its entry of the step's
// first chunk, a dead lane the zero block.
__device__ __forceinline__ const uint8_t *bfrag_base(const uint8_t *frags, const uint8_t *zero, int chunk,
                                                     const LaneConst &lc)
{
    return lc.live ? frags + (size_t)chunk * kQ1FragBytesPerChunk + lc.e * kQ1FragLaneStride
                   : zero + lc.e * kQ1FragLaneStride;
}

// A register of bit plane i from a word of packed signs: the word itself
// for plane 0 (its B values take the other planes' bits back out), bit i of
// each byte for the others.
__device__ __forceinline__ uint32_t q1_plane(uint32_t w, int i) { return i == 0 ? w : w & (0x01010101u << i); }

// D_lo + 256 D_hi of one limb pair, as a float (one rounding; |v| < 2^29).
__device__ __forceinline__ float limb_pair(int lo, int hi) { return (float)(lo + (hi << 8)); }

// Multiply-accumulate one staged step of nch (1 or 2) chunks.  bf: this
// lane's B fragment base for the step (bfrag_base); inf: this lane's (c, n)
// pair of the step's first chunk (stride 4 per chunk).  yacc[t][r]: row
// g + 8r of tile t.
__device__ __forceinline__ void consume_step(const uint8_t *st, const uint8_t *bf, const float2 *inf, int nch,
                                             const LaneConst &lc, float (&yacc)[2][2])
{
    uint2 w[2][2][kQ1StepChunks];  // [tile][row g / g+8][chunk]
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < kQ1StepChunks; ++c)
                w[t][r][c] = *reinterpret_cast<const uint2 *>(st + lc.woff + (16 * t + 8 * r) * kQ1RowStride + c * 32);
    int d[2][kQ1StepChunks][4];
    if (nch == kQ1StepChunks) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int c = 0; c < kQ1StepChunks; ++c) {
                const uint2 b = *reinterpret_cast<const uint2 *>(bf + c * kQ1FragBytesPerChunk + q1_frag_plane(i));
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint32_t a0 = q1_plane(w[t][0][c].x, i), a1 = q1_plane(w[t][1][c].x, i);
                    const uint32_t a2 = q1_plane(w[t][0][c].y, i), a3 = q1_plane(w[t][1][c].y, i);
                    if (i == 0)
                        mma_u8s8_z(d[t][c], a0, a1, a2, a3, b.x, b.y);
                    else
                        mma_u8s8(d[t][c], a0, a1, a2, a3, b.x, b.y);
                }
            }
        }
    } else {  // one chunk left
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint2 b = *reinterpret_cast<const uint2 *>(bf + q1_frag_plane(i));
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const uint32_t a0 = q1_plane(w[t][0][0].x, i), a1 = q1_plane(w[t][1][0].x, i);
                const uint32_t a2 = q1_plane(w[t][0][0].y, i), a3 = q1_plane(w[t][1][0].y, i);
                if (i == 0)
                    mma_u8s8_z(d[t][0], a0, a1, a2, a3, b.x, b.y);
                else
                    mma_u8s8(d[t][0], a0, a1, a2, a3, b.x, b.y);
            }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) d[t][1][0] = d[t][1][1] = d[t][1][2] = d[t][1][3] = 0;
    }
#pragma unroll
    for (int c = 0; c < kQ1StepChunks; ++c) {
        // a chunk past the end holds zero weights and contributes nothing
        const float2 ci = c < nch ? inf[4 * c] : make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint16_t sc =
                    *reinterpret_cast<const uint16_t *>(st + lc.soff + (16 * t + 8 * r) * 8 + c * 4);
                const float v = limb_pair(d[t][c][2 * r], d[t][c][2 * r + 1]);
                yacc[t][r] = fmaf(f16_bits_to_float(sc), fmaf(ci.x, v, ci.y), yacc[t][r]);
            }
    }
}

// Copy prepared chunks [ch_lo, ch_lo+n) (fragments, then the per-lane
// constants) to smem, and clear the zero block that follows them.
__device__ __forceinline__ void stage_act(uint8_t *smem, const Q1Params &p, int ch_lo, int n)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(p.act + (size_t)ch_lo * kQ1FragBytesPerChunk);
    uint4 *dst = reinterpret_cast<uint4 *>(smem);
    for (int i = threadIdx.x; i < n * (kQ1FragBytesPerChunk / 16); i += blockDim.x) dst[i] = __ldg(src + i);
    const uint4 *isrc = reinterpret_cast<const uint4 *>(p.act + p.info_off + (size_t)ch_lo * kQ1InfoBytesPerChunk);
    uint4 *idst = reinterpret_cast<uint4 *>(smem + (size_t)n * kQ1FragBytesPerChunk);
    for (int i = threadIdx.x; i < n * (kQ1InfoBytesPerChunk / 16); i += blockDim.x) idst[i] = __ldg(isrc + i);
}

// Zero block of kQ1ZeroBytes at `z` (16-byte aligned).
__device__ __forceinline__ void clear_zero_block(uint8_t *z)
{
    for (int i = threadIdx.x; i < kQ1ZeroBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(z)[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Limb scratch of one warp's build: four limbs, each 256 bytes plus 4 of
// padding (the fragment reads of the 16 live entries then fall in distinct
// banks).  The limb of k = 32 j + 8 c + i sits at byte 32 j + 4 i + c of its
// limb row, so the four k = 8c + i (c = 0..3) of a fragment word are one
// aligned 32-bit word.
constexpr int kQ1LimbStride = 260;
constexpr int kQ1LimbScratch = 4 * kQ1LimbStride + 16;  // per warp, 16-byte multiple
constexpr int kQ1BuildScratch = kQ1SplitWarps * kQ1LimbScratch;  // limb scratch of the fused split kernel

// 2^e for -126 <= e <= 127, exactly.
__device__ __forceinline__ float q1_pow2(int e) { return __int_as_float((e + 127) << 23); }

// The work of k_q1_prep_m1 for one 256-k chunk, done by one warp: lane l
// takes k = 256 ch + 32 j + l (j = 0..7; j < 4 is the chunk's first group),
// so every per-group reduction is a warp shuffle.  lw: this warp's limb
// scratch (kQ1LimbScratch bytes); info: the chunk's four (c, n) pairs.
// Writes the same bytes as k_q1_prep_m1: the scaling by 2^(23-E) and the
// constants are exact powers of two (23 - E, E - 29, E - 13 and E - 23 stay
// within the normal exponent range for kQ1MinExp <= E <= 128).
__device__ __forceinline__ void q1_build_chunk_warp(const uint16_t *__restrict__ x, int K, int ch, uint8_t *frag,
                                                    float2 *info, uint8_t *lw, int lane)
{
    float xv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int k = ch * kQ1ChunkK + 32 * j + lane;
        xv[j] = k < K ? bf16_bits_to_float(x[k]) : 0.f;
    }
    float m[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j >> 2] = fmaxf(m[j >> 2], fabsf(xv[j]));
    int E[2], T[2] = {0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float mh = warp_max_nonneg(m[h]);
        const int e8 = (int)((__float_as_uint(mh) >> 23) & 0xFFu);
        E[h] = max(e8 == 0 ? kQ1MinExp : e8 - 126, kQ1MinExp);  // smallest E with max|x| < 2^E
    }
    const int wpos = 4 * (lane & 7) + (lane >> 3);  // this lane's byte in each 32-k row of the scratch
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int X = __float2int_rn(xv[j] * q1_pow2(23 - E[j >> 2]));  // |X| <= 2^23
        T[j >> 2] += X;
        // k & 7 == lane & 7: the byte's plane-0 weight is in lane (lane & ~7)
        const int B = q1_plane_value(X, __shfl_sync(0xffffffffu, X, lane & ~7), lane & 7);
        const int l0 = (int)(int8_t)(B & 0xFF);
        int r = (B - l0) >> 8;
        const int l1 = (int)(int8_t)(r & 0xFF);
        r = (r - l1) >> 8;
        const int l2 = (int)(int8_t)(r & 0xFF);
        lw[0 * kQ1LimbStride + 32 * j + wpos] = (uint8_t)l0;
        lw[1 * kQ1LimbStride + 32 * j + wpos] = (uint8_t)l1;
        lw[2 * kQ1LimbStride + 32 * j + wpos] = (uint8_t)l2;
        lw[3 * kQ1LimbStride + 32 * j + wpos] = (uint8_t)((r - l2) >> 8);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int Th = warp_sum_int(T[h]);  // |T| <= 2^30
        if (lane == 0) {
            float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
            if ((2 * ch + h) * 128 < K) {
                lo = make_float2(q1_pow2(E[h] - 29), -((float)Th * q1_pow2(E[h] - 23)));
                hi = make_float2(q1_pow2(E[h] - 13), 0.f);
            }
            info[2 * h] = lo;
            info[2 * h + 1] = hi;
        }
    }
    __syncwarp();
    // fragment words: the same layout as k_q1_prep_m1 writes; lane l takes
    // entry e = l & 15 (k quarter t = e & 3, limb e >> 2) of mmas
    // 4 (l >> 4) .. 4 (l >> 4) + 3; register j of mma i holds k = 64 t + 32 j
    // + 8 c + i, c = 0..3: one scratch word
    const int e = lane & 15, t = e & 3;
    const uint8_t *lrow = lw + (e >> 2) * kQ1LimbStride;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int i = 4 * (lane >> 4) + q;
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(lrow + 32 * (2 * t) + 4 * i);
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(lrow + 32 * (2 * t + 1) + 4 * i);
        *reinterpret_cast<uint2 *>(frag + e * kQ1FragLaneStride + q1_frag_plane(i)) = make_uint2(w0, w1);
    }
    __syncwarp();  // the scratch is reused for the warp's next chunk
}

// Half h of q1_build_chunk_warp's work: group h (k = 256 ch + 128 h ..
// +127) of the chunk, i.e. its constants info[2h], info[2h+1] and the eight
// fragment entries whose k quarter t = e & 3 is 2h or 2h + 1 (each entry
// reads only its group's limbs).  Two warps building the two halves of a
// chunk write disjoint bytes, each with a limb scratch of its own; a warp's
// chain of loads, reductions and stores is half as long.  xat(k): x[k], a
// bf16 number, as a float (k < K).
template <typename XAt>
__device__ __forceinline__ void q1_build_half_warp(XAt xat, int K, int ch, int h, uint8_t *frag, float2 *info,
                                                   uint8_t *lw, int lane)
{
    float xv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = ch * kQ1ChunkK + 128 * h + 32 * j + lane;
        xv[j] = k < K ? xat(k) : 0.f;
    }
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(xv[j]));
    const float mh = warp_max_nonneg(m);
    const int e8 = (int)((__float_as_uint(mh) >> 23) & 0xFFu);
    const int E = max(e8 == 0 ? kQ1MinExp : e8 - 126, kQ1MinExp);  // smallest E with max|x| < 2^E
    const int wpos = 4 * (lane & 7) + (lane >> 3);  // this lane's byte in each 32-k row of the scratch
    int T = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int X = __float2int_rn(xv[j] * q1_pow2(23 - E));  // |X| <= 2^23
        T += X;
        // k & 7 == lane & 7: the byte's plane-0 weight is in lane (lane & ~7)
        const int B = q1_plane_value(X, __shfl_sync(0xffffffffu, X, lane & ~7), lane & 7);
        const int l0 = (int)(int8_t)(B & 0xFF);
        int r = (B - l0) >> 8;
        const int l1 = (int)(int8_t)(r & 0xFF);
        r = (r - l1) >> 8;
        const int l2 = (int)(int8_t)(r & 0xFF);
        const int row = 32 * (4 * h + j);  // the chunk's 32-k row of these k
        lw[0 * kQ1LimbStride + row + wpos] = (uint8_t)l0;
        lw[1 * kQ1LimbStride + row + wpos] = (uint8_t)l1;
        lw[2 * kQ1LimbStride + row + wpos] = (uint8_t)l2;
        lw[3 * kQ1LimbStride + row + wpos] = (uint8_t)((r - l2) >> 8);
    }
    const int Th = warp_sum_int(T);  // |T| <= 2^30
    if (lane == 0) {
        float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
        if ((2 * ch + h) * 128 < K) {
            lo = make_float2(q1_pow2(E - 29), -((float)Th * q1_pow2(E - 23)));
            hi = make_float2(q1_pow2(E - 13), 0.f);
        }
        info[2 * h] = lo;
        info[2 * h + 1] = hi;
    }
    __syncwarp();
    // lane l takes entry e = 4 (l' >> 1) + 2h + (l' & 1), l' = l & 7 (limb
    // l' >> 1, k quarter t = 2h + (l' & 1)), of mmas 2 (l >> 3) and
    // 2 (l >> 3) + 1
    const int el = lane & 7, e = 4 * (el >> 1) + 2 * h + (el & 1), t = e & 3;
    const uint8_t *lrow = lw + (e >> 2) * kQ1LimbStride;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int i = 2 * (lane >> 3) + q;
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(lrow + 32 * (2 * t) + 4 * i);
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(lrow + 32 * (2 * t + 1) + 4 * i);
        *reinterpret_cast<uint2 *>(frag + e * kQ1FragLaneStride + q1_frag_plane(i)) = make_uint2(w0, w1);
    }
    __syncwarp();  // the scratch is reused for the warp's next task
}

__device__ __forceinline__ unsigned long long globaltimer_ns_q1()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Final per-cell reduction: lanes tq = 0..3 of a row group hold the two
// groups' low/high limb partials; lane tq writes row g + 8*(tq&1) of tile
// tq>>1 into out(tile, row).
template <typename Out>
__device__ __forceinline__ void finish_cell(float (&yacc)[2][2], int lane, Out out)
{
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            yacc[t][r] += __shfl_xor_sync(0xffffffffu, yacc[t][r], 1);
            yacc[t][r] += __shfl_xor_sync(0xffffffffu, yacc[t][r], 2);
        }
    const int tq = lane & 3, g = lane >> 2;
    const int t = tq >> 1, r = tq & 1;
    const float v = t ? (r ? yacc[1][1] : yacc[1][0]) : (r ? yacc[0][1] : yacc[0][0]);
    out(16 * t + g + 8 * r, v);
    yacc[0][0] = yacc[0][1] = yacc[1][0] = yacc[1][1] = 0.f;
}

// ---------------------------------------------------------------------------
// stream kernel: persistent CTAs, cells = (matrix, 32-row block), all of K
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kQ1Warps * 32, (kQ1Warps <= 8 ? 2 : 1)) k_q1_m1_stream(const __grid_constant__ Q1Group grp,
                                                                   const Q1Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = (int)((long long)blockIdx.x * p.cells / gridDim.x);
    const int c1 = (int)((long long)(blockIdx.x + 1) * p.cells / gridDim.x);
    uint8_t *ring = smem + p.act_smem + warp * kQ1WarpRing;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);
    const int spc = (p.nchunks + kQ1StepChunks - 1) / kQ1StepChunks;  // steps per cell

    // issue iterator: cell -> (matrix ir, block iblk), step within the cell
    int icell = c0 + warp, ir = icell / p.blocksN, iblk = icell - ir * p.blocksN, istep = 0, islot = 0;
    auto issue_next = [&]() {
        if (icell < c1) {
            issue_any(ring_s + islot * kQ1StageBytes, grp, p, ir, iblk, istep * kQ1StepChunks, p.nchunks, lane);
            if (++istep == spc) {
                istep = 0;
                icell += kQ1Warps;
                iblk += kQ1Warps;
                while (iblk >= p.blocksN) {
                    iblk -= p.blocksN;
                    ++ir;
                }
            }
        }
        cp_async_commit();
        islot = islot + 1 == kQ1Stages ? 0 : islot + 1;
    };

#pragma unroll
    for (int t = 0; t < kQ1Stages - 1; ++t) issue_next();

    pdl_wait_primary();  // the activation and the outputs follow stream order from here
    uint8_t *zero = smem + p.act_smem - kQ1ZeroBytes;
    if (c1 > c0) stage_act(smem, p, 0, p.nchunks);
    clear_zero_block(zero);
    __syncthreads();

    const LaneConst lc = lane_const(lane);
    const float2 *sinfo = reinterpret_cast<const float2 *>(smem + (size_t)p.nchunks * kQ1FragBytesPerChunk) + lc.tq;

    int cell = c0 + warp, r = cell / p.blocksN, blk = cell - r * p.blocksN;
    int slot = 0;
    float yacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    while (cell < c1) {
        for (int s = 0; s < spc; ++s) {
            issue_next();
            cp_async_wait<kQ1Stages - 1>();
            __syncwarp();
            const int chs = s * kQ1StepChunks;
            consume_step(ring + slot * kQ1StageBytes, bfrag_base(smem, zero, chs, lc), sinfo + 4 * chs,
                         min(kQ1StepChunks, p.nchunks - chs), lc, yacc);
            __syncwarp();  // every lane is done with this stage before it is refilled
            slot = slot + 1 == kQ1Stages ? 0 : slot + 1;
        }
        float *yr = grp.y[r];
        const int row0 = blk * kQ1StepRows, N = p.N;
        finish_cell(yacc, lane, [&](int row, float v) {
            if ((lane & 3) < 4 && row0 + row < N) yr[row0 + row] = v;
        });
        cell += kQ1Warps;
        blk += kQ1Warps;
        while (blk >= p.blocksN) {
            blk -= p.blocksN;
            ++r;
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// lean stream kernel: the stream kernel's cells with 1024 k per step, for
// K % 1024 == 0, N % 32 == 0 and 16-byte aligned operands (no bounds tests)
// ---------------------------------------------------------------------------
//
// A stage holds 32 rows x 128 bytes of signs and, after them, each row's
// 16-byte run of eight fp16 scales.  Row q's 16-byte piece p sits at piece
// p ^ 2(q & 3): the 8-byte fragment reads of a warp then cover all 32 banks
// once per 128 bytes.  A lane copies piece (lane & 7) of rows (lane >> 3) +
// 4u, u = 0..7 (four whole rows per instruction), and the scale run of row
// `lane`.  One CTA per SM; every warp has its own ring of S stages.

constexpr int kQ1LChunks = 4;                                  // chunks per step
constexpr int kQ1LRowBytes = kQ1LChunks * 32;
constexpr int kQ1LStageW = kQ1StepRows * kQ1LRowBytes;
constexpr int kQ1LStageBytes = kQ1LStageW + kQ1StepRows * 16;
#ifndef LOWBIT_Q1_LEAN_STAGES
#define LOWBIT_Q1_LEAN_STAGES 2
#endif
#ifndef LOWBIT_Q1_LEAN_WARPS
#define LOWBIT_Q1_LEAN_WARPS 16
#endif

constexpr int kQ1LStages = LOWBIT_Q1_LEAN_STAGES;
constexpr int kQ1LMaxWarps = LOWBIT_Q1_LEAN_WARPS;
constexpr int kQ1LMinWarps = 8;

__device__ __forceinline__ void cp_async16_full(unsigned dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// One staged step.  woff[c]: this lane's byte offset of chunk c in row g of
// a stage; soff: its scale offset (row g, group h of chunk 0); bf: its B
// fragment base (bfrag_base); inf: its (c, n) pair of the step's first chunk.
// The chunks go in groups of kQ1LInter: inside a group the bit planes are the
// outer loop, so 2 kQ1LInter accumulator chains are in flight at once.
#ifndef LOWBIT_Q1_LEAN_INTER
#define LOWBIT_Q1_LEAN_INTER 2
#endif
constexpr int kQ1LInter = LOWBIT_Q1_LEAN_INTER;
static_assert(kQ1LChunks % kQ1LInter == 0, "chunk groups must tile the step");

// MV vectors: vector v's fragments at bf + v * bstride (bstride = 0 for the
// dead lanes, which read the zero block) and its constants at inf + v *
// istride.  A bit plane's masked weights feed one mma per vector.  With one
// vector two chunks are interleaved (kQ1LInter); with more, one chunk at a
// time keeps the accumulators in registers.
template <int MV>
__device__ __forceinline__ void lean_consume(const uint8_t *st, const uint8_t *bf, int bstride, const float2 *inf,
                                             int istride, const int (&woff)[kQ1LChunks], int soff,
                                             float (&yacc)[2][2][MV])
{
    constexpr int kInter = MV == 1 ? kQ1LInter : 1;
#pragma unroll
    for (int c0 = 0; c0 < kQ1LChunks; c0 += kInter) {
        uint2 w[kInter][2][2];  // [chunk][tile][row g / g+8]
#pragma unroll
        for (int q = 0; q < kInter; ++q)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    w[q][t][r] = *reinterpret_cast<const uint2 *>(st + woff[c0 + q] + (16 * t + 8 * r) * kQ1LRowBytes);
        int d[kInter][2][MV][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // bit planes 2j, 2j+1
#pragma unroll
            for (int q = 0; q < kInter; ++q) {
                uint2 bb[MV][2];
#pragma unroll
                for (int v = 0; v < MV; ++v) {
#if LOWBIT_Q1_BPAIR
                    const uint4 b4 = *reinterpret_cast<const uint4 *>(bf + v * bstride + (c0 + q) * kQ1FragBytesPerChunk +
                                                                      j * 256);
                    bb[v][0] = make_uint2(b4.x, b4.y);
                    bb[v][1] = make_uint2(b4.z, b4.w);
#else
                    bb[v][0] = *reinterpret_cast<const uint2 *>(bf + v * bstride + (c0 + q) * kQ1FragBytesPerChunk +
                                                                q1_frag_plane(2 * j));
                    bb[v][1] = *reinterpret_cast<const uint2 *>(bf + v * bstride + (c0 + q) * kQ1FragBytesPerChunk +
                                                                q1_frag_plane(2 * j + 1));
#endif
                }
#pragma unroll
                for (int o = 0; o < 2; ++o) {
                    const int i = 2 * j + o;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const uint2 w0 = w[q][t][0], w1 = w[q][t][1];
                        const uint32_t a0 = q1_plane(w0.x, i), a1 = q1_plane(w1.x, i);
                        const uint32_t a2 = q1_plane(w0.y, i), a3 = q1_plane(w1.y, i);
#pragma unroll
                        for (int v = 0; v < MV; ++v) {
                            if (i == 0)
                                mma_u8s8_z(d[q][t][v], a0, a1, a2, a3, bb[v][o].x, bb[v][o].y);
                            else
                                mma_u8s8(d[q][t][v], a0, a1, a2, a3, bb[v][o].x, bb[v][o].y);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kInter; ++q) {
            const int c = c0 + q;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float sc = f16_bits_to_float(
                        *reinterpret_cast<const uint16_t *>(st + soff + (16 * t + 8 * r) * 16 + c * 4));
#pragma unroll
                    for (int v = 0; v < MV; ++v) {
                        const float2 ci = inf[v * istride + 4 * c];
                        yacc[t][r][v] = fmaf(sc, fmaf(ci.x, limb_pair(d[q][t][v][2 * r], d[q][t][v][2 * r + 1]), ci.y),
                                             yacc[t][r][v]);
                    }
                }
        }
    }
}

// Work split: CTA b takes the cells [c0, c1) (equal shares of R * N/32);
// its T = (c1 - c0) * K/1024 steps are cut into equal contiguous ranges, one
// per warp.  A cell cut between warps w and w+1 is finished through shared
// memory, tail of w + head of w+1, in that order.  The planner gives every
// warp at least one cell's worth of steps, so no cell has a third part.
// With p.x set, every CTA builds the activation fragments from x itself (one
// chunk per warp at a time, in a limb scratch of its own after the rings, so
// that every ring slot is already streaming weights during the build).
// MV > 1: the product of MV vectors (rows of x; those at or past p.M read as
// zero and are not written), each with its own fragments and constants:
// vector v's fragments at v * nchunks KB, then all constants, vector-major.
// Warps per CTA at most: the several-vector forms keep more accumulators, so
// they run at most 12 warps (168 registers a thread).
__host__ __device__ constexpr int q1l_max_warps(int mv) { return mv == 1 ? kQ1LMaxWarps : 12; }

template <int MV, int KF>
__global__ void __launch_bounds__(q1l_max_warps(MV) * 32, 1) k_q1_m1_lean(const __grid_constant__ Q1Group grp,
                                                                          const Q1Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float part[2][q1l_max_warps(MV)][MV][kQ1StepRows];  // [head / tail][warp][vector][row] of cut cells
    pdl_launch_dependents();
    // KF > 0: K known at compile time, so the copy addresses of a step are
    // one register plus immediate offsets and the per-cell counts constants
    const int K = KF > 0 ? KF : p.K;
    const int nchunks = KF > 0 ? KF / kQ1ChunkK : p.nchunks;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int c0 = (int)((long long)blockIdx.x * p.cells / gridDim.x);
    const int c1 = (int)((long long)(blockIdx.x + 1) * p.cells / gridDim.x);
    const int spc = nchunks / kQ1LChunks;  // steps per cell
    const int T = (c1 - c0) * spc;
    const int s0 = (int)((long long)warp * T / nw), s1 = (int)((long long)(warp + 1) * T / nw);
    const size_t rowbytes = (size_t)(K >> 3);
    const int G = K >> 7;
    uint8_t *ring = smem + p.act_smem + warp * (kQ1LStages * kQ1LStageBytes);
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);

    // issue side: step is of this warp's range = cell c0 + is / spc, step is % spc
    const int rq = lane >> 3;
    const unsigned wdst = (unsigned)(rq * kQ1LRowBytes + (((lane & 7) ^ (rq << 1)) << 4));
    const unsigned sdst = (unsigned)(kQ1LStageW + lane * 16);
    int is = s0, islot = 0;
    int ir = 0, iblk = 0, ist = 0;  // matrix, 32-row block and step in cell of `is`
    const uint8_t *wsrc = nullptr;
    const uint16_t *ssrc = nullptr;
    auto cell_src = [&]() {
        wsrc = grp.bits[ir] + (size_t)(iblk * kQ1StepRows + rq) * rowbytes + (lane & 7) * 16 + ist * kQ1LRowBytes;
        ssrc = grp.scales[ir] + (size_t)(iblk * kQ1StepRows + lane) * G + ist * 2 * kQ1LChunks;
    };
    if (s0 < s1) {
        const int cell = c0 + s0 / spc;
        ir = cell / p.blocksN;
        iblk = cell - ir * p.blocksN;
        ist = s0 % spc;
        cell_src();
    }
    auto issue_next = [&]() {
        if (is < s1) {
            const unsigned st = ring_s + islot * kQ1LStageBytes;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                cp_async16_full(st + wdst + u * 4 * kQ1LRowBytes, wsrc + (size_t)(4 * u) * rowbytes);
            cp_async16_full(st + sdst, ssrc);
            wsrc += kQ1LRowBytes;
            ssrc += 2 * kQ1LChunks;
            ++is;
            if (++ist == spc) {
                ist = 0;
                if (++iblk == p.blocksN) {
                    iblk = 0;
                    ++ir;
                }
                if (is < s1) cell_src();
            }
        }
        cp_async_commit();
        islot = islot + 1 == kQ1LStages ? 0 : islot + 1;
    };
    // every ring slot starts filling before the wait: while the activation is
    // built, all of this warp's stages are in flight
#pragma unroll
    for (int t = 0; t < kQ1LStages; ++t) issue_next();

    pdl_wait_primary();  // x or the activation, and the outputs, follow stream order from here
    const int vfrag = nchunks * kQ1FragBytesPerChunk;  // bytes of one vector's fragments
    uint8_t *zero = smem + p.act_smem - kQ1ZeroBytes;
    float2 *info = reinterpret_cast<float2 *>(smem + (size_t)MV * vfrag);
    if (p.x != nullptr) {
        // this warp's limb scratch, after every warp's ring
        uint8_t *lw = smem + p.act_smem + (size_t)nw * (kQ1LStages * kQ1LStageBytes) + (size_t)warp * kQ1LimbScratch;
        for (int idx = warp; idx < MV * nchunks; idx += nw) {
            const int v = idx / nchunks, ch = idx - v * nchunks;
            uint8_t *frag = smem + (size_t)v * vfrag + (size_t)ch * kQ1FragBytesPerChunk;
            float2 *inf = info + 4 * (v * nchunks + ch);
            if (v < p.M) {
                q1_build_chunk_warp(p.x + (size_t)v * K, K, ch, frag, inf, lw, lane);
            } else {
                for (int i = lane; i < kQ1FragBytesPerChunk / 16; i += 32)
                    reinterpret_cast<uint4 *>(frag)[i] = make_uint4(0u, 0u, 0u, 0u);
                if (lane < 4) inf[lane] = make_float2(0.f, 0.f);
            }
        }
    } else if (c1 > c0) {
        stage_act(smem, p, 0, nchunks);  // one vector
    }
    clear_zero_block(zero);
    __syncthreads();

    const int g = lane >> 2, tq = lane & 3;
    int woff[kQ1LChunks];
#pragma unroll
    for (int c = 0; c < kQ1LChunks; ++c)
        woff[c] = g * kQ1LRowBytes + (((2 * c + (tq >> 1)) ^ ((g & 3) << 1)) << 4) + (tq & 1) * 8;
    const int soff = kQ1LStageW + g * 16 + (tq >> 1) * 2;
    const bool live = (lane >> 4) == (tq >> 1);
    const uint8_t *bf_live = smem + (lane & 15) * kQ1FragLaneStride, *bf_dead = zero + (lane & 15) * kQ1FragLaneStride;
    const int bstride = live ? vfrag : 0;
    const float2 *inf0 = info + tq;

    int s = s0, slot = 0;
    while (s < s1) {
        // one cell (or the part of it in [s0, s1))
        const int cell = c0 + s / spc, st0 = s % spc;
        const int st1 = min(spc, st0 + (s1 - s));
        float yacc[2][2][MV];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int v = 0; v < MV; ++v) yacc[t][r][v] = 0.f;
        for (int t = st0; t < st1; ++t) {
            cp_async_wait<kQ1LStages - 1>();  // the oldest of the kQ1LStages stages in flight has landed
            __syncwarp();
            lean_consume<MV>(ring + slot * kQ1LStageBytes,
                             live ? bf_live + t * (kQ1LChunks * kQ1FragBytesPerChunk) : bf_dead, bstride,
                             inf0 + 4 * kQ1LChunks * t, 4 * nchunks, woff, soff, yacc);
            __syncwarp();  // every lane is done with this stage before it is refilled
            issue_next();  // refill the slot just consumed
            slot = slot + 1 == kQ1LStages ? 0 : slot + 1;
        }
        s += st1 - st0;
        const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
        const int cut = st0 > 0 ? 0 : (st1 < spc ? 1 : -1);
#pragma unroll
        for (int v = 0; v < MV; ++v) {
            float yv[2][2] = {{yacc[0][0][v], yacc[0][1][v]}, {yacc[1][0][v], yacc[1][1][v]}};
            float *yr = grp.y[r] + (size_t)v * p.N + blk * kQ1StepRows;
            finish_cell(yv, lane, [&](int row, float val) {
                if (cut >= 0)
                    part[cut][warp][v][row] = val;
                else if (v < p.M)
                    yr[row] = val;
            });
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // cells cut between warps w and w + 1: one warp per cut, one row per lane
    if (warp + 1 < nw && s1 % spc != 0 && s1 > s0) {
        const int cell = c0 + s1 / spc;
        const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
#pragma unroll
        for (int v = 0; v < MV; ++v)
            if (v < p.M)
                grp.y[r][(size_t)v * p.N + blk * kQ1StepRows + lane] = part[1][warp][v][lane] + part[0][warp + 1][v][lane];
    }
}

// ---------------------------------------------------------------------------
// split kernel: a cluster of S CTAs = S K-slices of one 128-row block
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store a float into rank `rank`'s shared memory, at the address `local`
// has in this CTA.
__device__ __forceinline__ void st_cluster_f32(float *local, unsigned rank, float v)
{
    const unsigned a = (unsigned)__cvta_generic_to_shared(local);
    unsigned ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

#ifndef LOWBIT_Q1_SPLIT_STAGES
#define LOWBIT_Q1_SPLIT_STAGES 3
#endif
#ifndef LOWBIT_Q1_SPLIT_CTAS_PER_SM
#define LOWBIT_Q1_SPLIT_CTAS_PER_SM 2
#endif
#ifndef LOWBIT_Q1_SPLIT_FILL
#define LOWBIT_Q1_SPLIT_FILL 0
#endif
constexpr int kQ1SplitStages = LOWBIT_Q1_SPLIT_STAGES;  // steps of a split warp in flight
constexpr int kQ1SplitRing = kQ1SplitStages * kQ1StageBytes;

constexpr int kQ1SplitRows = kQ1SplitWarps * kQ1StepRows;  // rows of one CTA
// dynamic shared memory of the split kernel at most: its static partial-sum
// and receive buffers take the rest of the 227 KB
constexpr int kQ1SplitSmemCap = kQ1MaxSmem - (kQ1SplitRows + kQ1MaxCluster) * 4;

// grid: x = slice (= cluster rank), y = r * blocks_per_matrix + row block
__global__ void __launch_bounds__(kQ1SplitWarps * 32) k_q1_m1_split(const __grid_constant__ Q1Group grp,
                                                                    const Q1Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float part[kQ1SplitRows];
    __shared__ float recv[kQ1SplitRows + kQ1MaxCluster];  // [slice][share]: the partial sums pushed to this rank
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = blockIdx.x, nsl = gridDim.x;
    const int bpm = (p.N + kQ1SplitRows - 1) / kQ1SplitRows;
    const int r = blockIdx.y / bpm, rb = blockIdx.y - r * bpm;
    const int blk = rb * kQ1SplitWarps + warp;  // 32-row block of this warp
    const int ch_lo = slice * p.L, ch_hi = min(p.nchunks, ch_lo + p.L);
    const int nsteps = blk * kQ1StepRows < p.N && ch_hi > ch_lo
                           ? (ch_hi - ch_lo + kQ1StepChunks - 1) / kQ1StepChunks : 0;
    uint8_t *ring = smem + p.act_smem + warp * kQ1SplitRing;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);

    int ist = 0;
    auto issue_next = [&]() {
        if (ist < nsteps)
            issue_any(ring_s + (ist % kQ1SplitStages) * kQ1StageBytes, grp, p, r, blk,
                      ch_lo + ist * kQ1StepChunks, ch_hi, lane);
        ++ist;
        cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < kQ1SplitStages - 1; ++t) issue_next();

    pdl_wait_primary();
    uint8_t *zero = smem + p.act_smem - kQ1ZeroBytes;
    if (ch_hi > ch_lo) {
        const int n = ch_hi - ch_lo;
        if (p.x != nullptr) {
            // fused: the warps turn the slice's chunks of x into fragments, one chunk half per task
            uint8_t *lw = smem + p.act_smem + kQ1SplitWarps * kQ1SplitRing + warp * kQ1LimbScratch;
            float2 *info = reinterpret_cast<float2 *>(smem + (size_t)n * kQ1FragBytesPerChunk);
            for (int c2 = warp; c2 < 2 * n; c2 += kQ1SplitWarps) {  // half c2 & 1 of chunk c2 >> 1
                const int c = c2 >> 1;
                q1_build_half_warp([&](int k) { return bf16_bits_to_float(p.x[k]); }, p.K, ch_lo + c, c2 & 1,
                                   smem + (size_t)c * kQ1FragBytesPerChunk, info + 4 * c, lw, lane);
            }
        } else {
            stage_act(smem, p, ch_lo, n);
        }
    }
    clear_zero_block(zero);
    __syncthreads();

    const LaneConst lc = lane_const(lane);
    const float2 *sinfo = reinterpret_cast<const float2 *>(smem + (size_t)(ch_hi - ch_lo) * kQ1FragBytesPerChunk) + lc.tq;
    float yacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    for (int s = 0; s < nsteps; ++s) {
        issue_next();
        cp_async_wait<kQ1SplitStages - 1>();
        __syncwarp();
        const int lch = s * kQ1StepChunks;
        consume_step(ring + (s % kQ1SplitStages) * kQ1StageBytes, bfrag_base(smem, zero, lch, lc),
                     sinfo + 4 * lch, min(kQ1StepChunks, ch_hi - ch_lo - lch), lc, yacc);
        __syncwarp();
    }
    cp_async_wait<0>();
    finish_cell(yacc, lane, [&](int row, float v) { part[warp * kQ1StepRows + row] = v; });

    if (nsl == 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < kQ1SplitRows; i += blockDim.x)
            if (rb * kQ1SplitRows + i < p.N) grp.y[r][rb * kQ1SplitRows + i] = part[i];
        return;
    }
    // rank q owns rows [q*per, (q+1)*per): every slice pushes its partial sums
    // of those rows into rank q's recv[slice], and after one cluster barrier
    // (release / acquire) rank q adds them up in rank order.  Nothing reads
    // another CTA's shared memory after the barrier, so each CTA may then
    // finish on its own.
    const int per = (kQ1SplitRows + nsl - 1) / nsl;
    __syncthreads();  // part[] is complete
    for (int i = threadIdx.x; i < kQ1SplitRows; i += blockDim.x) {
        const int q = i / per;
        st_cluster_f32(recv + slice * per + (i - q * per), (unsigned)q, part[i]);
    }
    cluster_sync();
    for (int j = threadIdx.x; j < per && slice * per + j < kQ1SplitRows; j += blockDim.x) {
        float sum = 0.f;
        for (int q = 0; q < nsl; ++q) sum += recv[q * per + j];
        const int row = rb * kQ1SplitRows + slice * per + j;
        if (row < p.N) grp.y[r][row] = sum;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static int num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

struct Q1Plan {
    bool lean;          // lean stream kernel
    int warps;          // its warps per CTA
    int mv;             // its vectors (1, 2 or 4)
    bool stream;        // stream kernel (else split kernel)
    int nchunks, blocksN, L, nslices, grid_x, grid_y;
    size_t act_smem, smem;
    size_t info_off, xcopy_off, act_bytes;
    bool ok;
};

// aligned: every matrix's signs and scales start on a 16-byte boundary.
// mv > 1: only the lean stream kernel for mv vectors is considered (lean =
// false when it does not apply).
static Q1Plan q1_plan(int R, int N, int K, int sms, bool aligned = false, int mv = 1)
{
    Q1Plan P = {};
    P.nchunks = (K + kQ1ChunkK - 1) / kQ1ChunkK;
    P.blocksN = (N + kQ1StepRows - 1) / kQ1StepRows;
    P.info_off = align256((size_t)P.nchunks * kQ1FragBytesPerChunk);
    P.xcopy_off = align256(P.info_off + (size_t)P.nchunks * kQ1InfoBytesPerChunk);
    P.act_bytes = align256(P.xcopy_off + (size_t)K * 2u);
    const long long units = (long long)R * P.blocksN;
    const size_t per_chunk = kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk;
    const size_t whole = (size_t)P.nchunks * per_chunk + kQ1ZeroBytes;  // fragments, constants, zero block
    const size_t ring_stream = (size_t)kQ1Warps * kQ1WarpRing;
    // lean stream kernel: whole 1024-k steps and 32-row blocks, as many warps
    // (at most kQ1LMaxWarps) as fit next to the activation, >= 2 cells per warp
    if (aligned && K % 1024 == 0 && N % kQ1StepRows == 0) {
        const size_t per_warp = (size_t)kQ1LStages * kQ1LStageBytes + kQ1LimbScratch;  // ring + build scratch
        const size_t cap = (size_t)kQ1MaxSmem - 2 * q1l_max_warps(mv) * mv * kQ1StepRows * 4;  // static cut buffers
        const size_t whole_mv = (size_t)mv * P.nchunks * per_chunk + kQ1ZeroBytes;
        const long long fit = whole_mv < cap ? (long long)((cap - whole_mv) / per_warp) : 0;
        // >= one cell per warp keeps every warp's step range at least one
        // cell long, so a cell is cut at most once
        const int warps = (int)std::min<long long>(std::min<long long>(q1l_max_warps(mv), fit), units / sms);
        if (warps >= kQ1LMinWarps) {
            P.lean = true;
            P.stream = true;
            P.warps = warps;
            P.mv = mv;
            P.L = P.nchunks;
            P.nslices = 1;
            P.act_smem = whole_mv;
            P.smem = whole_mv + (size_t)warps * per_warp;
            P.grid_x = sms;
            P.grid_y = 1;
            P.ok = true;
            return P;
        }
    }
    if (mv > 1) return P;
    // stream kernel: enough 32-row blocks for >= 2 cells per warp slot, and
    // the whole activation fits next to the rings
    if (units >= 2LL * sms * 2 * kQ1Warps && whole + ring_stream <= (size_t)kQ1MaxSmem) {
        P.stream = true;
        P.L = P.nchunks;
        P.nslices = 1;
        P.act_smem = whole;
        P.smem = whole + ring_stream;
        const int per_sm = 2 * (P.smem + 1024) <= 228 * 1024 ? 2 : 1;
        P.grid_x = (int)std::min<long long>((long long)per_sm * sms, (units + kQ1Warps - 1) / kQ1Warps);
        P.grid_y = 1;
        P.ok = true;
        return P;
    }
    // split kernel: S slices so that the CTAs fill the SMs several times over
    P.stream = false;
    const size_t ring_split = (size_t)kQ1SplitWarps * kQ1SplitRing;
    const long long blocks = (long long)R * ((N + kQ1SplitRows - 1) / kQ1SplitRows);
    int S = (int)std::min<long long>(
        kQ1MaxCluster, std::max<long long>(1, ((long long)LOWBIT_Q1_SPLIT_CTAS_PER_SM * sms + blocks - 1) / blocks));
    if (LOWBIT_Q1_SPLIT_FILL)  // whole slice in flight
        S = std::max(S, (P.nchunks + kQ1StepChunks * kQ1SplitStages - 1) / (kQ1StepChunks * kQ1SplitStages));
    S = std::min(std::min(S, kQ1MaxCluster), P.nchunks);
    while (true) {
        P.L = (P.nchunks + S - 1) / S;
        P.nslices = (P.nchunks + P.L - 1) / P.L;
        P.act_smem = (size_t)P.L * per_chunk + kQ1ZeroBytes;
        P.smem = P.act_smem + ring_split + kQ1BuildScratch;
        if (P.smem <= (size_t)kQ1SplitSmemCap || S >= kQ1MaxCluster) break;
        S = std::min(kQ1MaxCluster, S * 2);
    }
    P.grid_x = P.nslices;
    P.grid_y = (int)blocks;
    P.ok = P.smem <= (size_t)kQ1SplitSmemCap && blocks < 65536;
    return P;
}

size_t q1m1_act_bytes(int K) { return q1_plan(1, 1, K, 148).act_bytes; }
size_t q1m1_xcopy_off(int K) { return q1_plan(1, 1, K, 148).xcopy_off; }
int q1m1_max_group() { return kQ1MaxGroup; }

bool q1m1_shape_supported(int R, int N, int K)
{
    if ((K / 128) % 2 != 0) return false;  // scale pairs must be 4-byte aligned
    if (R < 1 || R > kQ1MaxGroup) return false;
    return q1_plan(R, N, K, num_sms()).ok;
}

lowbit_status q1m1_prepare_launch(const uint16_t *x, int K, void *act, cudaStream_t st)
{
    const Q1Plan P = q1_plan(1, 1, K, 148);
    cudaError_t e = launch_pdl(k_q1_prep_m1, dim3(P.nchunks), dim3(256), 0, st, x, K, static_cast<uint8_t *>(act),
                               P.info_off, P.xcopy_off);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

static lowbit_status q1m1_launch(const Q1Plan &P, const uint8_t *const *bits, const uint16_t *const *scales,
                                 const void *act, const uint16_t *x, float *const *y, int R, int N, int K,
                                 cudaStream_t st, int M = 1)
{
    Q1Group grp;
    for (int r = 0; r < R; ++r) {
        grp.bits[r] = bits[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    Q1Params p = {};
    p.act = static_cast<const uint8_t *>(act);
    p.x = x;
    p.info_off = P.info_off;
    p.R = R;
    p.N = N;
    p.K = K;
    p.nchunks = P.nchunks;
    p.L = P.L;
    p.blocksN = P.blocksN;
    p.cells = (int)((long long)R * P.blocksN);
    p.act_smem = (int)P.act_smem;
    p.M = M;
    void (*kern)(const Q1Group, const Q1Params) = k_q1_m1_split;
    if (P.lean)
        kern = P.mv == 2   ? k_q1_m1_lean<2, 0>
               : P.mv == 4 ? k_q1_m1_lean<4, 0>
               : K == 4096 ? k_q1_m1_lean<1, 4096>
               : K == 5120 ? k_q1_m1_lean<1, 5120>
               : K == 17408 ? k_q1_m1_lean<1, 17408>
                             : k_q1_m1_lean<1, 0>;
    else if (P.stream)
        kern = k_q1_m1_stream;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.grid_x, P.grid_y);
    cfg.blockDim = dim3(P.lean ? P.warps * 32 : P.stream ? kQ1Warps * 32 : kQ1SplitWarps * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    int na = 1;
    if (!P.stream) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = P.nslices;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, grp, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q1m1_gemv_launch(const uint8_t *const *bits, const uint16_t *const *scales, const void *act,
                               float *const *y, int R, int N, int K, cudaStream_t st)
{
    bool aligned = true;
    for (int r = 0; r < R; ++r)
        aligned = aligned && (reinterpret_cast<uintptr_t>(bits[r]) & 15u) == 0 &&
                  (reinterpret_cast<uintptr_t>(scales[r]) & 15u) == 0;
    return q1m1_launch(q1_plan(R, N, K, num_sms(), aligned), bits, scales, act, nullptr, y, R, N, K, st);
}

// R matrices straight from x ([M][K], 1 <= M <= 4) in one launch, when the
// shape takes the lean stream kernel (every CTA builds the activation
// itself; M = 3 runs the 4-vector form with a zero vector); otherwise
// LOWBIT_ERR_UNSUPPORTED_SHAPE and the caller takes another path.
static int q1_mv(int M) { return M <= 1 ? 1 : M == 2 ? 2 : 4; }

lowbit_status q1m1_gemv_x_group_launch(const uint8_t *const *bits, const uint16_t *const *scales, const uint16_t *x,
                                       float *const *y, int R, int M, int N, int K, cudaStream_t st)
{
    if (M < 1 || M > 4 || R < 1 || R > kQ1MaxGroup || !q1m1_shape_supported(R, N, K))
        return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    const Q1Plan P = q1_plan(R, N, K, num_sms(), true, q1_mv(M));
    if (!P.lean) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    return q1m1_launch(P, bits, scales, nullptr, x, y, R, N, K, st, M);
}

bool q1m1_x_group_supported(int R, int M, int N, int K)
{
    return M >= 1 && M <= 4 && R >= 1 && R <= kQ1MaxGroup && q1m1_shape_supported(R, N, K) &&
           q1_plan(R, N, K, num_sms(), true, q1_mv(M)).lean;
}

// One matrix straight from x, in one launch (the split kernel builds its
// slice of the activation itself).  q1m1_fused_supported: the shape takes it.
bool q1m1_fused_supported(int N, int K)
{
    return q1m1_shape_supported(1, N, K) && !q1_plan(1, N, K, num_sms()).stream;
}

// LOWBIT_ERR_UNSUPPORTED_SHAPE when the shape takes the stream kernel, which
// needs a prepared activation.
lowbit_status q1m1_gemv_fused_launch(const uint8_t *bits, const uint16_t *scales, const uint16_t *x, float *y, int N,
                                     int K, cudaStream_t st)
{
    if (!q1m1_shape_supported(1, N, K)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    const Q1Plan P = q1_plan(1, N, K, num_sms());
    if (P.stream) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    return q1m1_launch(P, &bits, &scales, nullptr, x, &y, 1, N, K, st);
}


// ---------------------------------------------------------------------------
// one decode step through a stack of Q1_0_g128 projections, in one launch
// ---------------------------------------------------------------------------
//
// Per layer: q, k, v, o (hidden -> hidden), gate and up (hidden -> ffn, the
// same input, outputs summed before the next normalisation), down (ffn ->
// hidden); each projection's input is bf16(RMSNorm(previous fp32 output)),
// unit gain; the layer's output, normalised, is the next layer's input.
// The step runs as 6 phases per layer in one cooperative launch (every CTA
// resident), separated by a grid barrier: a global counter every CTA adds to
// once per phase, waited on with a bounded spin.  In a phase every CTA
//   1. normalises the previous phase's output (it reads all of it) and turns
//      its own 1024-k slice into B fragments (four warps, one 256-k chunk
//      each);
//   2. its warps run (32-row block, slice) units through the same mma.sync
//      inner loop as the split kernel and add each unit's partial sums into
//      the phase's output with fp32 atomics (outputs rotate through three
//      buffers: the one two phases ahead is zeroed meanwhile);
// while the warps' cp.async rings keep fetching the next units' weights
// across the phase boundaries (weights never depend on activations).

constexpr int kStWarps = 16;
constexpr int kStThreads = kStWarps * 32;
constexpr int kStSliceK = 512;                  // k per slice: two 256-k chunks (one step)
constexpr int kStSliceChunks = kStSliceK / kQ1ChunkK;
constexpr int kStStages = 3;
constexpr int kStMaxProj = 512;
constexpr int kStPhasesPerLayer = 6;
constexpr unsigned long long kStWaitNs = 2000000000ull;

__device__ unsigned g_q1stack_fault;  // set when a grid-barrier wait ran out

struct StackW {
    const uint8_t *bits[kStMaxProj];     // projection 7 l + {q, k, v, o, gate, up, down}
    const uint16_t *scales[kStMaxProj];
};

struct StackP {
    uint16_t *x;         // [H] bf16: the step input, then its output
    float *buf;          // 3 x [2F] fp32 phase outputs
    unsigned *bar;       // grid barrier counter (zero at launch)
    uint16_t *rec_in;    // optional [7L][F] bf16: every projection's input
    float *rec_out;      // optional [7L][F] fp32: every projection's output
    int L, H, F;
    float eps;
};

struct StPhase {
    int ph, layer, K, N, nblocks, nmat;  // nmat: 1, or 2 for gate+up (rows of up follow those of gate)
};

__device__ __forceinline__ StPhase st_phase(const StackP &p, int ph_idx)
{
    StPhase q;
    q.layer = ph_idx / kStPhasesPerLayer;
    q.ph = ph_idx % kStPhasesPerLayer;
    q.K = q.ph == 5 ? p.F : p.H;
    q.N = q.ph == 4 ? p.F : (q.ph == 5 ? p.H : p.H);
    q.nmat = q.ph == 4 ? 2 : 1;
    q.nblocks = q.nmat * q.N / 32;
    return q;
}

__device__ __forceinline__ int st_proj(const StPhase &q, int mat) { return 7 * q.layer + (q.ph < 4 ? q.ph : (q.ph == 4 ? 4 + mat : 6)); }

// A warp's position in its sequence of steps (phase, j-th unit of the warp
// in that phase, step t of the unit).
struct StIt {
    int p, j, t;
};

// This CTA's K slice s, its rank rk among the CTAs of that slice and their
// count cps, for inputs of width H (index 0) and F (index 1): fixed for the
// launch, so computed once (divisions by a run-time count are long chains
// of dependent integer instructions).
struct StCta {
    int s[2], rk[2], cps[2];
};

__device__ __forceinline__ StCta st_cta(const StackP &p, int G, int c)
{
    StCta t;
    const int Ks[2] = {p.H, p.F};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int S = Ks[i] / kStSliceK;
        t.s[i] = c % S;
        t.rk[i] = c / S;
        t.cps[i] = (G - 1 - t.s[i]) / S + 1;  // CTAs that work on slice s
    }
    return t;
}

// Block of unit j of warp `warp` in phase q, or -1.
__device__ __forceinline__ int st_block(const StPhase &q, const StCta &ct, int warp, int j)
{
    const int f = q.ph == 5;  // down reads the ffn-wide vector
    const int b = ct.rk[f] + ct.cps[f] * (warp + j * kStWarps);
    return b < q.nblocks ? b : -1;
}

// Move to the next step that exists (or past the last phase).
__device__ __forceinline__ void st_next(StIt &it, const StackP &p, const StCta &ct, int warp, int nph)
{
    if (++it.t < kStSliceChunks / kQ1StepChunks) return;
    it.t = 0;
    ++it.j;
    while (it.p < nph && st_block(st_phase(p, it.p), ct, warp, it.j) < 0) {
        ++it.p;
        it.j = 0;
    }
}

__device__ __forceinline__ void st_first(StIt &it, const StackP &p, const StCta &ct, int warp, int nph)
{
    it.p = 0;
    it.j = 0;
    it.t = 0;
    while (it.p < nph && st_block(st_phase(p, it.p), ct, warp, 0) < 0) ++it.p;
}

// Copy one step: 32 rows x 2 chunks of one matrix (all rows and chunks
// exist).  W: the projections' pointers, copied to shared memory at the
// start (a run-time index into the parameter block is a constant-cache
// load that can miss).
__device__ __forceinline__ void st_issue(unsigned stage, const StackW &W, const StackP &p, const StIt &it,
                                         const StCta &ct, int warp, int lane)
{
    const StPhase q = st_phase(p, it.p);
    const int b = st_block(q, ct, warp, it.j);
    const int nb = q.N / 32;  // blocks per matrix (a power-of-two division)
    const int mat = b >= nb ? 1 : 0, row0 = (b - mat * nb) * 32;
    const int pi = st_proj(q, mat);
    const int ch0 = ct.s[q.ph == 5] * kStSliceChunks + it.t * kQ1StepChunks;
    const int rowbytes = q.K >> 3, G16 = q.K >> 7;
    const int col = lane & 3;
    const uint8_t *bsrc = W.bits[pi] + (size_t)(row0 + (lane >> 2)) * rowbytes + ch0 * 32 + col * 16;
    const unsigned bdst = stage + (lane >> 2) * kQ1RowStride + col * 16;
#pragma unroll
    for (int u = 0; u < 4; ++u) cp_async16(bdst + 8 * u * kQ1RowStride, bsrc + (size_t)(8 * u) * rowbytes, true);
    const int sc = lane & 1;
    const uint16_t *ssrc = W.scales[pi] + (size_t)(row0 + (lane >> 1)) * G16 + 2 * (ch0 + sc);
    const unsigned sdst = stage + kQ1StageW + (lane >> 1) * 8 + sc * 4;
#pragma unroll
    for (int u = 0; u < 2; ++u) cp_async4(sdst + 16 * u * 8, ssrc + (size_t)(16 * u) * G16, true);
}

// Bring phase ph's weights into L2 ahead of time: CTA c takes blocks c,
// c + G, ...; a block's 32 rows of signs (and of scales) are contiguous.
constexpr int kStPrefetchAhead = 2;  // phases

__device__ __forceinline__ void st_prefetch_l2(const StackW &W, const StackP &p, int ph, int G, int c)
{
    if (ph >= p.L * kStPhasesPerLayer) return;
    const StPhase q = st_phase(p, ph);
    const unsigned bbytes = 32u * (unsigned)(q.K / 8), sbytes = 32u * (unsigned)(q.K / 128) * 2u;
    for (int b = c + G * (int)threadIdx.x; b < q.nblocks; b += G * kStThreads) {
        const int mat = b / (q.N / 32), row0 = (b % (q.N / 32)) * 32;
        const int pi = st_proj(q, mat);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(W.bits[pi] + (size_t)row0 * (q.K / 8)),
                     "r"(bbytes)
                     : "memory");
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(W.scales[pi] + (size_t)row0 * (q.K / 128)),
                     "r"(sbytes)
                     : "memory");
    }
}

// Sum over the CTA.  red needs no barrier before it is written: its
// readers in the previous phase have passed the block barrier after that
// phase's fragment build since.
__device__ __forceinline__ float st_block_sum(float v, float *red)
{
    v = warp_sum(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kStWarps; ++w) t += red[w];
    return t;
}

// Grid barrier: every CTA adds 1 per phase; wait until all G have.  The
// add is a release at GPU scope (it orders every write of the CTA that the
// block barrier made visible to thread 0) and the poll an acquire, so no
// separate fence is needed on either side.
__device__ __forceinline__ void st_grid_sync(const StackP &p, unsigned target)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p.bar), "r"(1u) : "memory");
        unsigned v = 0;
        const unsigned long long t0 = globaltimer_ns_q1();
        while (true) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.bar) : "memory");
            if (v >= target) break;
            // after one wait has run out the results are void: do not wait again
            if (*reinterpret_cast<volatile unsigned *>(&g_q1stack_fault) != 0u) break;
            if (globaltimer_ns_q1() - t0 > kStWaitNs) {
                atomicExch(&g_q1stack_fault, 1u);
                break;
            }
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kStThreads, 1) k_q1_stack_m1(const __grid_constant__ StackW W, const StackP p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float red[kStWarps];
    __shared__ StackW Ws;  // the projections' pointers
    for (int i = threadIdx.x; i < 7 * p.L; i += blockDim.x) {
        Ws.bits[i] = W.bits[i];
        Ws.scales[i] = W.scales[i];
    }
    __syncthreads();
    uint8_t *frag = smem;                                                  // 4 chunks of fragments
    float2 *info = reinterpret_cast<float2 *>(smem + kStSliceChunks * kQ1FragBytesPerChunk);
    uint8_t *zero = smem + kStSliceChunks * (kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk);
    uint8_t *lwall = zero + kQ1ZeroBytes;                                                     // limb scratch
    float *xsf = reinterpret_cast<float *>(lwall + 2 * kStSliceChunks * kQ1LimbScratch);       // raw slice values
    uint8_t *rings = reinterpret_cast<uint8_t *>(xsf) + kStSliceK * 4;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = gridDim.x, c = blockIdx.x;
    const int nph = p.L * kStPhasesPerLayer;
    const size_t bufn = 2 * (size_t)p.F;
    uint8_t *ring = rings + warp * kStStages * kQ1StageBytes;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);

    for (int ph = 0; ph < kStPrefetchAhead; ++ph) st_prefetch_l2(Ws, p, ph, G, c);
    const StCta ct = st_cta(p, G, c);
    StIt is;  // issue position (runs up to kStStages - 1 steps ahead)
    st_first(is, p, ct, warp, nph);
    int nis = 0;
    auto issue_next = [&]() {
        if (is.p < nph) {
            st_issue(ring_s + (nis % kStStages) * kQ1StageBytes, Ws, p, is, ct, warp, lane);
            st_next(is, p, ct, warp, nph);
        }
        ++nis;
        cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < kStStages - 1; ++t) issue_next();

    pdl_wait_primary();  // x is produced by earlier kernels
    clear_zero_block(zero);  // ordered before its first read by the phase's barriers
    const LaneConst lc = lane_const(lane);
    StIt cs;  // consume position
    st_first(cs, p, ct, warp, nph);
    int ncs = 0;

    for (int ph_idx = 0; ph_idx <= nph; ++ph_idx) {
        st_prefetch_l2(Ws, p, ph_idx + kStPrefetchAhead, G, c);
        // ---- input of this phase: normalise the previous output (or take x) ----
        const bool last = ph_idx == nph;
        const StPhase q = st_phase(p, last ? nph - 1 : ph_idx);
        const int Kin = last ? p.H : q.K;
        const float *prev = ph_idx > 0 ? p.buf + (size_t)((ph_idx - 1) % 3) * bufn : nullptr;
        // down reads gate + up: kept apart only when they are recorded, else
        // the gate+up phase adds both into one vector
        const bool two = !last && q.ph == 5 && p.rec_out != nullptr;
        float inv = 1.f;
        const int S = q.K / kStSliceK, s = ct.s[q.ph == 5];
        if (prev != nullptr) {
            // sum of squares of the whole input, 16 loads in flight per thread;
            // this CTA's slice is kept on the way (raw, scaled once inv is known)
            const int sl0 = last ? -1 : s * (kStSliceK / 4), sl1 = sl0 + kStSliceK / 4;
            float ss = 0.f;
            const int n4 = Kin / 4;
            const float4 *a4 = reinterpret_cast<const float4 *>(prev);
            const float4 *b4 = reinterpret_cast<const float4 *>(prev + p.F);
            for (int base = threadIdx.x; base < n4; base += 16 * kStThreads) {
                float4 v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = base + u * kStThreads;
                    v[u] = i < n4 ? a4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                if (two) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int i = base + u * kStThreads;
                        if (i < n4) {
                            const float4 w = b4[i];
                            v[u].x += w.x; v[u].y += w.y; v[u].z += w.z; v[u].w += w.w;
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = base + u * kStThreads;
                    if (i >= sl0 && i < sl1) reinterpret_cast<float4 *>(xsf)[i - sl0] = v[u];
                    ss = fmaf(v[u].x, v[u].x, ss);
                    ss = fmaf(v[u].y, v[u].y, ss);
                    ss = fmaf(v[u].z, v[u].z, ss);
                    ss = fmaf(v[u].w, v[u].w, ss);
                }
            }
            ss = st_block_sum(ss, red);
            inv = 1.0f / sqrtf(ss / (float)Kin + p.eps);
        }
        // the previous phase's outputs, recorded (its buffer is stable until the next phase)
        if (p.rec_out != nullptr && ph_idx > 0) {
            const StPhase pq = st_phase(p, ph_idx - 1);
            for (int m = 0; m < pq.nmat; ++m) {
                const int pi = st_proj(pq, m);
                for (int i = c * kStThreads + threadIdx.x; i < pq.N; i += G * kStThreads)
                    p.rec_out[(size_t)pi * p.F + i] = prev[(size_t)m * p.F + i];
            }
        }
        if (last) {
            // the step's output: x = bf16(norm(down output)), written by slices of CTAs
            for (int i = c * kStThreads + threadIdx.x; i < p.H; i += G * kStThreads)
                p.x[i] = __bfloat16_as_ushort(__float2bfloat16_rn(prev[i] * inv));
            break;
        }
        // the projections' input: x_k = bf16(raw_k * inv) over this CTA's
        // slice; the builders round it themselves from the raw values (kept
        // in xsf before the block sum, whose barrier makes them visible)
        if (p.rec_in != nullptr && c < S)  // the first CTA of each slice records it
            for (int i = threadIdx.x; i < kStSliceK; i += kStThreads) {
                const int k = s * kStSliceK + i;
                const uint16_t xb = prev == nullptr ? p.x[k] : __bfloat16_as_ushort(__float2bfloat16_rn(xsf[i] * inv));
                for (int m = 0; m < q.nmat; ++m) p.rec_in[(size_t)st_proj(q, m) * p.F + k] = xb;
            }
        if (prev == nullptr) {  // the step input, exact as a float (inv = 1)
            for (int i = threadIdx.x; i < kStSliceK; i += kStThreads) xsf[i] = bf16_bits_to_float(p.x[s * kStSliceK + i]);
            __syncthreads();
        }
        // zero the buffer two phases ahead (read last by the previous phase's prologue)
        {
            float *z = p.buf + (size_t)((ph_idx + 1) % 3) * bufn;
            for (size_t i = (size_t)c * kStThreads + threadIdx.x; i < bufn; i += (size_t)G * kStThreads) z[i] = 0.f;
        }
        if (warp < 2 * kStSliceChunks)  // half warp & 1 of chunk warp >> 1
            q1_build_half_warp(
                [&](int k) { return __bfloat162float(__float2bfloat16_rn(xsf[k - s * kStSliceK] * inv)); }, q.K,
                s * kStSliceChunks + (warp >> 1), warp & 1, frag + (warp >> 1) * kQ1FragBytesPerChunk,
                info + 4 * (warp >> 1), lwall + warp * kQ1LimbScratch, lane);
        __syncthreads();

        // ---- this warp's units of the phase ----
        float *out = p.buf + (size_t)(ph_idx % 3) * bufn;
        const int fold = (q.ph == 4 && p.rec_out == nullptr) ? q.N : 0;  // up's rows land on gate's
        const float2 *sinfo = info + lc.tq;
        while (cs.p == ph_idx) {
            float yacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            const int b = st_block(q, ct, warp, cs.j);
            for (int t = 0; t < kStSliceChunks / kQ1StepChunks; ++t) {
                issue_next();
                cp_async_wait<kStStages - 1>();
                __syncwarp();
                const int lch = t * kQ1StepChunks;
                consume_step(ring + (ncs % kStStages) * kQ1StageBytes, bfrag_base(frag, zero, lch, lc),
                             sinfo + 4 * lch, kQ1StepChunks, lc, yacc);
                __syncwarp();
                ++ncs;
                st_next(cs, p, ct, warp, nph);
            }
            finish_cell(yacc, lane, [&](int row, float v) {
                size_t o = (size_t)b * 32 + row;
                if (fold != 0 && o >= (size_t)fold) o -= fold;
                atomicAdd(out + o, v);
            });
        }
        st_grid_sync(p, (unsigned)G * (unsigned)(ph_idx + 1));
    }
    cp_async_wait<0>();
}

lowbit_status q1stack_launch(const uint8_t *const *bits, const uint16_t *const *scales, int L, int H, int F,
                             uint16_t *x, float eps, void *ws, uint16_t *rec_in, float *rec_out, cudaStream_t st)
{
    if (L < 1 || 7 * L > kStMaxProj || H % kStSliceK != 0 || F % kStSliceK != 0) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    static StackW W;  // large: kept off the stack
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 7 * L; ++i) {
        W.bits[i] = bits[i];
        W.scales[i] = scales[i];
    }
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    StackP p = {};
    p.x = x;
    p.bar = reinterpret_cast<unsigned *>(w8);
    p.buf = reinterpret_cast<float *>(w8 + 256);
    p.rec_in = rec_in;
    p.rec_out = rec_out;
    p.L = L;
    p.H = H;
    p.F = F;
    p.eps = eps;
    const size_t smem = kStSliceChunks * (kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk) + kQ1ZeroBytes +
                        2 * kStSliceChunks * kQ1LimbScratch + kStSliceK * 4 +
                        (size_t)kStWarps * kStStages * kQ1StageBytes;
    if (cudaFuncSetAttribute(k_q1_stack_m1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    int per_sm = 0, sms = num_sms();
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_q1_stack_m1, kStThreads, smem) != cudaSuccess ||
        per_sm < 1)
        return LOWBIT_ERR_CUDA;
    // every K slice needs a CTA of its own (CTA c takes slice c % S)
    if (F / kStSliceK > sms * per_sm || H / kStSliceK > sms * per_sm) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    // the barrier counter and phase 0's output start at zero
    if (cudaMemsetAsync(w8, 0, 256 + 2 * (size_t)F * 4, st) != cudaSuccess) return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms * per_sm);
    cfg.blockDim = dim3(kStThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barrier cannot deadlock
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_q1_stack_m1, W, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

size_t q1stack_workspace_bytes(int F) { return 256 + 3 * 2 * (size_t)F * 4; }

int q1stack_fault_flag()
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_q1stack_fault, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_q1stack_fault, &zero, sizeof(zero));
    return (int)v;
}

}  // namespace lowbit
