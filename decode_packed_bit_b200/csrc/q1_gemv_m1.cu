// q1_gemv_m1.cu -- Q1_0_g128 matrix-vector products at M = 1 on the tensor
// cores (mma.sync m16n8k32, u8 x s8 -> s32), for a group of R weight
// matrices that multiply one activation vector.
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
// instruction.  The kernel feeds raw sign bits to the integer tensor cores:
//
//   A operand: for bit position i (0..7) one lop3 keeps bit i of each of the
//     four bytes of a 32-bit word of packed signs, giving four u8 values
//     b*2^i -- four weights per instruction, no shifts, no table.
//   B operand: x rewritten exactly as integers.  Per 128-group, x is scaled
//     to 24-bit fixed point X_k = round(x_k * 2^(23-E_g)) (E_g = the group's
//     binary exponent ceiling), multiplied by 2^(7-i) to cancel the bit
//     weight of its A slot, and split into four signed 8-bit limbs, one limb
//     per B column.  Each D column then holds sum_k b_k * limb_l(X_k 2^(7-i))
//     exactly, in int32.
//   Two groups share one accumulator: B columns 0-3 carry the four limbs of
//     the first group of a 256-k chunk, columns 4-7 those of the second.
//   Epilogue per (row, group): 2^7 sum_k b X = sum_l D_l 2^(8l); the signed
//     sum is sum s x = 2 sum b x - sum x, so y += d * (2^(E-29) * sum_l D_l
//     2^(8l) - S_g) with S_g = 2^(E-23) * sum_k X_k.  Integer-exact up to the
//     24-bit rounding of x and the fp32 epilogue.
//
// Work split.  A cell is 16 rows of one matrix times one K-slice; cells are
// ordered slice-major and cut into equal contiguous ranges, one per
// persistent CTA, so the CTA needs only the activation fragments of one or
// two slices, which it stages in shared memory for all its warps.  When the
// group has enough rows (R * N/16 fills the machine) the slice is all of K
// and no reduction is needed.  Otherwise K is split; the partial sums of one
// 16-row tile are reduced in fixed slice order (deterministic) by the last
// warp to finish the tile, found with a per-tile arrival counter that it
// resets to zero for the next call.
//
// Weight words and scales never depend on earlier kernels in the stream, so
// each warp loads its first step of weights before griddepcontrol.wait: the
// weight stream of this launch overlaps the tail of the previous kernel.
#include <algorithm>

#include "common.cuh"

namespace lowbit {

constexpr int kQ1ChunkK = 256;
constexpr int kQ1FragBytesPerChunk = 1024;  // 8 mma x 16 active lanes x 8 bytes
constexpr int kQ1InfoBytesPerChunk = 16;    // two groups x (G, S) floats
constexpr int kQ1Warps = 8;
constexpr int kQ1StepChunks = 4;            // chunks of one row pair loaded per step
constexpr int kQ1MinExp = -96;              // activations below 2^-96 round to 0
constexpr int kQ1MaxGroup = 256;
constexpr int kQ1CounterBytes = 64 * 1024;  // fixed counter region at the front of the workspace
constexpr int kQ1MaxSmem = 227 * 1024;

struct Q1Group {
    const uint8_t *bits[kQ1MaxGroup];
    const uint16_t *scales[kQ1MaxGroup];
    float *y[kQ1MaxGroup];
};

static inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// activation prepare: x (bf16) -> limb fragments + per-group (G, S)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA of 256 threads per 256-k chunk, one thread per k.  When `cnt` is
// not null the CTAs also zero the split-K arrival counters (one-shot path).
// A plain bf16 copy of x is kept after the fragments for shapes the tensor
// kernel does not take (K/128 odd), which the SIMT kernel then reads.
__global__ void __launch_bounds__(256) k_q1_prep_m1(const uint16_t *__restrict__ x, int K,
                                                    uint8_t *__restrict__ act, size_t info_off, size_t xcopy_off,
                                                    unsigned *__restrict__ cnt, int ncnt)
{
    __shared__ float smax[8];
    __shared__ int ssum[8];
    pdl_launch_dependents();
    const int ch = blockIdx.x;
    const int kk = threadIdx.x;
    const int k = ch * kQ1ChunkK + kk;
    const int warp = kk >> 5, lane = kk & 31;
    const int h = kk >> 7;  // group of this k within the chunk
    pdl_wait_primary();     // x is produced, and act last read, by earlier kernels

    if (cnt != nullptr)
        for (int i = ch * 256 + kk; i < ncnt; i += gridDim.x * 256) cnt[i] = 0u;

    const uint16_t xb = k < K ? x[k] : (uint16_t)0;
    if (k < K) reinterpret_cast<uint16_t *>(act + xcopy_off)[k] = xb;  // for the SIMT path
    const float xv = bf16_bits_to_float(xb);
    const float wm = warp_max(fabsf(xv));
    if (lane == 0) smax[warp] = wm;
    __syncthreads();
    const float m = fmaxf(fmaxf(smax[4 * h], smax[4 * h + 1]), fmaxf(smax[4 * h + 2], smax[4 * h + 3]));
    // E = smallest integer with m < 2^E (m normal: exponent field - 126)
    const int e8 = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    const int E = max(e8 == 0 ? kQ1MinExp : e8 - 126, kQ1MinExp);
    const int X = __float2int_rn(ldexpf(xv, 23 - E));       // |X| < 2^23
    const int B = X * (1 << (7 - (k & 7)));                 // cancels the A slot weight 2^i
    int l0 = (int)(int8_t)(B & 0xFF);
    int r = (B - l0) >> 8;
    int l1 = (int)(int8_t)(r & 0xFF);
    r = (r - l1) >> 8;
    int l2 = (int)(int8_t)(r & 0xFF);
    const int l3 = (r - l2) >> 8;                           // |B| < 2^30 keeps it in [-64, 64]

    // fragment position consumed by lane (n = 4h + limb, t = kk/64):
    //   byte (kk%32)/8 of register (kk%64)/32 of mma (kk%8), active lane index
    //   8h + 2*limb + (t&1)
    const int tq = kk >> 6, rem = kk & 63;
    const int half = rem >> 5, c = (rem >> 3) & 3, i = rem & 7;
    uint8_t *base = act + (size_t)ch * kQ1FragBytesPerChunk + i * 128 + half * 4 + c;
    const int a = 8 * h + (tq & 1);
    base[(a + 0) * 8] = (uint8_t)l0;
    base[(a + 2) * 8] = (uint8_t)l1;
    base[(a + 4) * 8] = (uint8_t)l2;
    base[(a + 6) * 8] = (uint8_t)l3;

    const int ws = warp_sum_int(X);
    if (lane == 0) ssum[warp] = ws;
    __syncthreads();
    if ((kk & 127) == 0) {
        const int T = ssum[4 * h] + ssum[4 * h + 1] + ssum[4 * h + 2] + ssum[4 * h + 3];  // |T| < 2^30
        const int grp = 2 * ch + h;
        float2 info = make_float2(0.f, 0.f);
        if (grp * 128 < K) info = make_float2(ldexpf(1.0f, E - 29), ldexpf((float)T, E - 23));
        reinterpret_cast<float2 *>(act + info_off)[grp] = info;
    }
}

// ---------------------------------------------------------------------------
// the product
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte (or 4-byte) asynchronous global -> shared copies; a copy with
// `valid` false writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, bool valid)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Staging ring of one warp: each stage holds 16 rows x 4 chunks of weight
// bytes (rows padded to 160 bytes so the consumers' 8-byte reads are bank-
// conflict free) and the 16 rows x 8 fp16 scales of those chunks.
constexpr int kQ1Stages = 3;
constexpr int kQ1RowStride = 160;
constexpr int kQ1StageW = 16 * kQ1RowStride;
constexpr int kQ1StageBytes = kQ1StageW + 16 * 16;
constexpr int kQ1WarpRing = kQ1Stages * kQ1StageBytes;

struct Q1Params {
    const uint8_t *act;
    size_t info_off;
    float *part;
    unsigned *cnt;
    int R, N, K, nchunks, L, nslices, tilesN, steps_per_cell;
    int cells;
    int act_smem;       // bytes reserved for staged activation chunks
};

// Position of a warp in its sequence of steps, advanced without divisions.
struct StepIter {
    int slice, r, tile;  // current cell
    int first;           // first chunk of the step within the slice
    int left;            // cells left for this warp (including the current)
};

__device__ __forceinline__ void iter_init(StepIter &it, const Q1Params &p, int cell, int ncells)
{
    const int per_slice = p.R * p.tilesN;
    it.slice = cell / per_slice;
    const int rem = cell - it.slice * per_slice;
    it.r = rem / p.tilesN;
    it.tile = rem - it.r * p.tilesN;
    it.first = 0;
    it.left = ncells;
}

// next step; moves to the cell kQ1Warps further when the slice is done
__device__ __forceinline__ void iter_next(StepIter &it, const Q1Params &p)
{
    it.first += kQ1StepChunks;
    if (it.first < p.L) return;
    it.first = 0;
    --it.left;
    it.tile += kQ1Warps;
    while (it.tile >= p.tilesN) {
        it.tile -= p.tilesN;
        if (++it.r == p.R) {
            it.r = 0;
            ++it.slice;
        }
    }
}

// Issue the asynchronous copies of one step (chunks first..first+3 of the
// cell's slice, 16 rows) into `stage`.  Lane L copies 16-byte column L%8 of
// rows L/8 + {0,4,8,12}, and the fp16 scale pairs (row L/4 + {0,8}, chunk
// L%4).  FULL: the step lies inside the matrix (no bounds tests).
template <bool FULL>
__device__ __forceinline__ void issue_step(uint8_t *stage, const Q1Group &grp, const Q1Params &p,
                                           const StepIter &it, int lane)
{
    const int rowbytes = p.K >> 3, G = p.K >> 7;
    const int ch0 = it.slice * p.L + it.first;
    const int col = lane & 7, c = col >> 1;
    const int row0 = it.tile * 16 + (lane >> 3);
    const uint8_t *bsrc = grp.bits[it.r] + (size_t)row0 * rowbytes + (ch0 + c) * 32 + (col & 1) * 16;
    uint8_t *bdst = stage + (lane >> 3) * kQ1RowStride + col * 16;
    const bool cok = FULL || (it.first + c < p.L && (ch0 + c) * 32 + (col & 1) * 16 + 16 <= rowbytes);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const bool ok = FULL || (cok && row0 + 4 * u < p.N);
        cp_async16(bdst + 4 * u * kQ1RowStride, ok ? bsrc + (size_t)(4 * u) * rowbytes : grp.bits[it.r], ok);
    }
    const int sc = lane & 3;
    const int srow0 = it.tile * 16 + (lane >> 2);
    const uint16_t *ssrc = grp.scales[it.r] + (size_t)srow0 * G + 2 * (ch0 + sc);
    uint8_t *sdst = stage + kQ1StageW + (lane >> 2) * 16 + sc * 4;
    const bool sok = FULL || (it.first + sc < p.L && 2 * (ch0 + sc) < G);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const bool ok = FULL || (sok && srow0 + 8 * u < p.N);
        cp_async4(sdst + 8 * u * 16, ok ? ssrc + (size_t)(8 * u) * G : grp.scales[it.r], ok);
    }
}

__device__ __forceinline__ void issue_any(uint8_t *stage, const Q1Group &grp, const Q1Params &p, const StepIter &it,
                                          int lane)
{
    const bool full = it.first + kQ1StepChunks <= p.L && it.tile * 16 + 16 <= p.N &&
                      (it.slice * p.L + it.first + kQ1StepChunks) * 256 <= p.K;
    if (full)
        issue_step<true>(stage, grp, p, it, lane);
    else
        issue_step<false>(stage, grp, p, it, lane);
}

// The product kernel.  Requires K/128 even (scale pairs 4-byte aligned).
__global__ void __launch_bounds__(kQ1Warps * 32, 2) k_q1_gemv_m1(const __grid_constant__ Q1Group grp,
                                                                 const Q1Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tq = lane & 3, h = tq >> 1;
    const int c0 = (int)((long long)blockIdx.x * p.cells / gridDim.x);
    const int c1 = (int)((long long)(blockIdx.x + 1) * p.cells / gridDim.x);
    const bool active = (g >> 2) == h;
    const int aidx = 8 * h + 2 * (g & 3) + (tq & 1);
    const float limb_scale = (tq & 1) ? 65536.f : 1.f;
    uint8_t *ring = smem + p.act_smem + warp * kQ1WarpRing;

    const int my_cells = c1 - c0 > warp ? (c1 - c0 - warp + kQ1Warps - 1) / kQ1Warps : 0;
    StepIter is;  // issue iterator, runs kQ1Stages-1 steps ahead
    iter_init(is, p, c0 + warp, my_cells);

    // prologue: the first stages of weights do not depend on earlier kernels
#pragma unroll
    for (int t = 0; t < kQ1Stages - 1; ++t) {
        if (is.left > 0) {
            issue_any(ring + t * kQ1StageBytes, grp, p, is, lane);
            iter_next(is, p);
        }
        cp_async_commit();
    }

    pdl_wait_primary();  // the activation and y / part / cnt follow stream order from here

    // stage the activation chunks of the slices this CTA touches
    int ch_lo = 0, nst = 0;
    if (c1 > c0) {
        const int per_slice = p.R * p.tilesN;
        const int s_lo = c0 / per_slice, s_hi = (c1 - 1) / per_slice;
        ch_lo = s_lo * p.L;
        nst = min(p.nchunks, (s_hi + 1) * p.L) - ch_lo;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.act + (size_t)ch_lo * kQ1FragBytesPerChunk);
        uint4 *dst = reinterpret_cast<uint4 *>(smem);
        for (int i = threadIdx.x; i < nst * (kQ1FragBytesPerChunk / 16); i += blockDim.x) dst[i] = __ldg(src + i);
        const uint4 *isrc = reinterpret_cast<const uint4 *>(p.act + p.info_off + (size_t)ch_lo * kQ1InfoBytesPerChunk);
        uint4 *idst = reinterpret_cast<uint4 *>(smem + (size_t)nst * kQ1FragBytesPerChunk);
        for (int i = threadIdx.x; i < nst; i += blockDim.x) idst[i] = __ldg(isrc + i);
    }
    __syncthreads();
    const uint8_t *bfrag = smem + aidx * 8;  // this lane's B fragments, chunk-major
    const float2 *sinfo = reinterpret_cast<const float2 *>(smem + (size_t)nst * kQ1FragBytesPerChunk) + h;
    const int woff0 = g * kQ1RowStride + tq * 8, woff1 = woff0 + 8 * kQ1RowStride;
    const int soff = kQ1StageW + g * 16 + h * 2;

    StepIter it;  // consume iterator
    iter_init(it, p, c0 + warp, my_cells);
    float yacc[2] = {0.f, 0.f};
    int slot = 0, islot = kQ1Stages - 1;
    while (it.left > 0) {
        if (is.left > 0) {
            issue_any(ring + islot * kQ1StageBytes, grp, p, is, lane);
            iter_next(is, p);
        }
        cp_async_commit();
        islot = islot + 1 == kQ1Stages ? 0 : islot + 1;
        cp_async_wait<kQ1Stages - 1>();
        __syncwarp();

        const uint8_t *st = ring + slot * kQ1StageBytes;
        const int chs = it.slice * p.L + it.first;      // first chunk of the step
        const int nch = min(kQ1StepChunks, min(p.L - it.first, p.nchunks - chs));
        const uint8_t *bf = bfrag + (chs - ch_lo) * kQ1FragBytesPerChunk;
        const float2 *inf = sinfo + 2 * (chs - ch_lo);

        uint2 w0[kQ1StepChunks], w1[kQ1StepChunks];
#pragma unroll
        for (int c = 0; c < kQ1StepChunks; ++c) {
            w0[c] = *reinterpret_cast<const uint2 *>(st + woff0 + c * 32);
            w1[c] = *reinterpret_cast<const uint2 *>(st + woff1 + c * 32);
        }
        int d[kQ1StepChunks][4];
#pragma unroll
        for (int c = 0; c < kQ1StepChunks; ++c) d[c][0] = d[c][1] = d[c][2] = d[c][3] = 0;
        if (nch == kQ1StepChunks) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t m = 0x01010101u << i;
#pragma unroll
                for (int c = 0; c < kQ1StepChunks; ++c) {
                    uint2 b = make_uint2(0u, 0u);
                    if (active) b = *reinterpret_cast<const uint2 *>(bf + c * kQ1FragBytesPerChunk + i * 128);
                    mma_u8s8(d[c], w0[c].x & m, w1[c].x & m, w0[c].y & m, w1[c].y & m, b.x, b.y);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t m = 0x01010101u << i;
#pragma unroll
                for (int c = 0; c < kQ1StepChunks; ++c) {
                    if (c < nch) {
                        uint2 b = make_uint2(0u, 0u);
                        if (active) b = *reinterpret_cast<const uint2 *>(bf + c * kQ1FragBytesPerChunk + i * 128);
                        mma_u8s8(d[c], w0[c].x & m, w1[c].x & m, w0[c].y & m, w1[c].y & m, b.x, b.y);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kQ1StepChunks; ++c) {
            // chunks past the end hold zero weights, zero scales and zero info
            const float2 gi = c < nch ? inf[2 * c] : make_float2(0.f, 0.f);
            const float coef = gi.x * limb_scale;
            const float sub = (tq & 1) ? 0.f : gi.y;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint16_t sc = *reinterpret_cast<const uint16_t *>(st + soff + 8 * r * 16 + c * 4);
                const float v = fmaf(256.f, (float)d[c][2 * r + 1], (float)d[c][2 * r]);
                yacc[r] = fmaf(f16_bits_to_float(sc), fmaf(coef, v, -sub), yacc[r]);
            }
        }
        __syncwarp();  // every lane is done with this stage before it is refilled
        slot = slot + 1 == kQ1Stages ? 0 : slot + 1;

        if (it.first + kQ1StepChunks >= p.L) {  // last step of this cell
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                yacc[r] += __shfl_xor_sync(0xffffffffu, yacc[r], 1);
                yacc[r] += __shfl_xor_sync(0xffffffffu, yacc[r], 2);
            }
            const int myrow = it.tile * 16 + g + 8 * (tq & 1);
            const bool writer = tq < 2 && myrow < p.N;
            const float myval = (tq & 1) ? yacc[1] : yacc[0];
            if (p.nslices == 1) {
                if (writer) grp.y[it.r][myrow] = myval;
            } else {
                const size_t tile_id = (size_t)it.r * p.tilesN + it.tile;
                if (writer) {
                    p.part[((size_t)it.slice * p.R + it.r) * p.N + myrow] = myval;
                    __threadfence();
                }
                __syncwarp();
                unsigned old = 0;
                if (lane == 0) old = atomicAdd(p.cnt + tile_id, 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == (unsigned)(p.nslices - 1)) {
                    __threadfence();
                    const int row = it.tile * 16 + (lane & 15);
                    if (lane < 16 && row < p.N) {
                        float s = 0.f;
                        const float *pp = p.part + (size_t)it.r * p.N + row;
                        const size_t stride = (size_t)p.R * p.N;
                        int q = 0;
                        for (; q + 4 <= p.nslices; q += 4) {
                            const float a0 = __ldcg(pp + (q + 0) * stride), a1 = __ldcg(pp + (q + 1) * stride);
                            const float a2 = __ldcg(pp + (q + 2) * stride), a3 = __ldcg(pp + (q + 3) * stride);
                            s += a0; s += a1; s += a2; s += a3;
                        }
                        for (; q < p.nslices; ++q) s += __ldcg(pp + q * stride);
                        grp.y[it.r][row] = s;
                    }
                    if (lane == 0) p.cnt[tile_id] = 0u;  // ready for the next call
                }
            }
            yacc[0] = yacc[1] = 0.f;
        }
        iter_next(it, p);
    }
    cp_async_wait<0>();
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
    int nchunks, L, nslices, tilesN, steps_per_cell, cells, grid;
    size_t smem, act_smem;
    size_t info_off, xcopy_off, act_bytes, part_bytes, ws_bytes;
};

// Choose the K-split: no split when the group's 16-row tiles alone give every
// warp slot several cells, else split K into slices of L chunks.
static Q1Plan q1_plan_ns(int R, int N, int K, int sms, int ns)
{
    Q1Plan P;
    P.nchunks = (K + kQ1ChunkK - 1) / kQ1ChunkK;
    P.tilesN = (N + 15) / 16;
    P.info_off = align256((size_t)P.nchunks * kQ1FragBytesPerChunk);
    P.xcopy_off = align256(P.info_off + (size_t)P.nchunks * kQ1InfoBytesPerChunk);
    P.act_bytes = align256(P.xcopy_off + (size_t)K * 2u);
    const long long units = (long long)R * P.tilesN;
    P.L = (P.nchunks + ns - 1) / ns;
    P.nslices = (P.nchunks + P.L - 1) / P.L;
    P.steps_per_cell = (P.L + kQ1StepChunks - 1) / kQ1StepChunks;
    const long long cells = units * P.nslices;
    P.cells = cells < (1LL << 31) ? (int)cells : -1;
    // two CTAs per SM when the staged activation leaves room for both rings
    const size_t act_est = (size_t)std::min(P.nchunks, 2 * P.L) * (kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk);
    const int per_sm = (2 * (act_est + (size_t)kQ1Warps * kQ1WarpRing) <= (size_t)kQ1MaxSmem) ? 2 : 1;
    P.grid = (int)std::min<long long>((long long)per_sm * sms,
                                      std::max<long long>(1, (cells + kQ1Warps - 1) / kQ1Warps));
    const long long cpc = (cells + P.grid - 1) / P.grid;
    const int span = (int)std::min<long long>(P.nslices, (cpc + units - 1) / units + 1);
    const int nst = std::min(P.nchunks, span * P.L);
    P.act_smem = ((size_t)nst * (kQ1FragBytesPerChunk + kQ1InfoBytesPerChunk) + 15) & ~size_t(15);
    P.smem = P.act_smem + (size_t)kQ1Warps * kQ1WarpRing;
    P.part_bytes = P.nslices > 1 ? align256((size_t)P.nslices * R * (size_t)N * sizeof(float)) : 0;
    P.ws_bytes = P.nslices > 1 ? kQ1CounterBytes + P.part_bytes : 0;
    return P;
}

// Choose the K-split: no split when the group's 16-row tiles alone give every
// warp slot several cells, else split K into slices of L chunks.  The split
// is widened if the slices one CTA stages would not fit in shared memory.
static Q1Plan q1_plan(int R, int N, int K, int sms)
{
    const int nchunks = (K + kQ1ChunkK - 1) / kQ1ChunkK;
    const long long units = (long long)R * ((N + 15) / 16);
    const long long want = 4LL * sms * kQ1Warps;  // cells wanted in flight
    int ns = (int)std::min<long long>(nchunks, std::max<long long>(1, (want + units - 1) / units));
    if (units > kQ1CounterBytes / 4) ns = 1;       // the counter region bounds the split tiles
    Q1Plan P = q1_plan_ns(R, N, K, sms, ns);
    while (P.smem > (size_t)kQ1MaxSmem && units <= kQ1CounterBytes / 4 && ns < nchunks) {
        ns = std::min(nchunks, ns * 2);
        P = q1_plan_ns(R, N, K, sms, ns);
    }
    return P;
}

size_t q1m1_act_bytes(int K) { return q1_plan(1, 1, K, 148).act_bytes; }

size_t q1m1_ws_bytes(int R, int N, int K)
{
    // the split decision depends on the SM count: size for the largest split
    const Q1Plan P = q1_plan(R, N, K, num_sms());
    return P.ws_bytes;
}

bool q1m1_shape_supported(int R, int N, int K)
{
    if ((K / 128) % 2 != 0) return false;  // scale pairs must be 4-byte aligned
    const Q1Plan P = q1_plan(R, N, K, num_sms());
    return P.smem <= (size_t)kQ1MaxSmem && P.cells > 0 && R >= 1 && R <= kQ1MaxGroup;
}

lowbit_status q1m1_prepare_launch(const uint16_t *x, int K, void *act, unsigned *cnt, cudaStream_t st)
{
    const Q1Plan P = q1_plan(1, 1, K, 148);
    cudaError_t e = launch_pdl(k_q1_prep_m1, dim3(P.nchunks), dim3(256), 0, st, x, K,
                               static_cast<uint8_t *>(act), P.info_off, P.xcopy_off, cnt,
                               cnt ? kQ1CounterBytes / 4 : 0);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q1m1_gemv_launch(const uint8_t *const *bits, const uint16_t *const *scales, const void *act,
                               float *const *y, int R, int N, int K, void *ws, cudaStream_t st)
{
    const Q1Plan P = q1_plan(R, N, K, num_sms());
    Q1Group grp;
    for (int r = 0; r < R; ++r) {
        grp.bits[r] = bits[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    Q1Params p;
    p.act = static_cast<const uint8_t *>(act);
    p.info_off = P.info_off;
    p.cnt = P.nslices > 1 ? static_cast<unsigned *>(ws) : nullptr;
    p.part = P.nslices > 1 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kQ1CounterBytes) : nullptr;
    p.R = R;
    p.N = N;
    p.K = K;
    p.nchunks = P.nchunks;
    p.L = P.L;
    p.nslices = P.nslices;
    p.tilesN = P.tilesN;
    p.steps_per_cell = P.steps_per_cell;
    p.cells = P.cells;
    p.act_smem = (int)P.act_smem;
    if (P.smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_q1_gemv_m1, cudaFuncAttributeMaxDynamicSharedMemorySize, kQ1MaxSmem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaError_t e = launch_pdl(k_q1_gemv_m1, dim3(P.grid), dim3(kQ1Warps * 32), P.smem, st, grp, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

int q1m1_max_group() { return kQ1MaxGroup; }
size_t q1m1_xcopy_off(int K) { return q1_plan(1, 1, K, 148).xcopy_off; }

}  // namespace lowbit
