// int4_gemv_m1.cu -- INT4_G64 matrix-vector product at M = 1 on the integer
// tensor cores (mma.sync m16n8k32, u8 x s8 -> s32).
//
// What is computed ("acorn-llm 0.11.4", section "int4 quantisation quality:
// group quantisation": one scale per group of values along the input
// dimension, here 64 values and an FP16 scale):
//     y[n] = sum_g d[n][g] * sum_{k in g} q[n][k] * x[k],  q in [-8, 7].
//
// As the acorn page observes, a grouped kernel must keep the scale switch and
// the group bookkeeping out of the inner loop.  Here the inner loop is pure
// integer tensor-core work and the scale is applied once per (row, group):
//
//   A operand: one lop3 per 32-bit word and nibble half, (w & 0x0F0F0F0F) ^
//     0x08080808 gives the four low nibbles as u8 q+8, (w & 0xF0F0F0F0) ^
//     0x80808080 the four high nibbles as u8 16*(q+8).
//   B operand: per 64-group, x as 24-bit fixed point X_k = round(x_k *
//     2^(23-E_g)); even k (low nibbles) take 16*X_k, odd k take X_k, so every
//     product is 16*(q+8)*X; split into four signed 8-bit limbs, one per B
//     column.  Columns 0-3 carry the first group of a 128-k pair, 4-7 the
//     second.
//   Epilogue: sum_k q X = D/16 - 8*sum_k X, with D = sum_l D_l 2^(8l); so
//     y += d * (2^(E-27) * D - 2^(E-20) * sum_k X_k).
//
// Work split and weight streaming follow the Q1 kernels: a step is 32 rows
// (two mma tiles) x one 128-k pair of groups, staged per warp by cp.async.
// One matrix: a thread-block cluster splits K and reduces through distributed
// shared memory when the rows alone cannot fill the GPU (k_i4_m1_split).  A
// group of matrices that read one x: one persistent CTA per SM streams an
// equal share of every matrix's 32-row blocks over all of K (k_i4_m1_lean).
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace lowbit {

constexpr int kI4PairK = 128;               // k per step (two 64-groups)
constexpr int kI4FragBytesPerPair = 1024;   // 4 mma x 32 lanes x 8 bytes
constexpr int kI4InfoBytesPerPair = 16;     // two groups x (G, S)
constexpr int kI4Warps = 8;
constexpr int kI4SplitWarps = 4;
constexpr int kI4StepRows = 32;
// Tuning knobs (compile-time; the defaults are the measured best).
#ifndef LOWBIT_I4_STAGES
#define LOWBIT_I4_STAGES 6
#endif
#ifndef LOWBIT_I4_CTAS_PER_SM
#define LOWBIT_I4_CTAS_PER_SM 2
#endif
#ifndef LOWBIT_I4_FILL
#define LOWBIT_I4_FILL 0
#endif
constexpr int kI4Stages = LOWBIT_I4_STAGES;  // steps of a warp in flight
constexpr int kI4RowStride = 64;            // 16-byte reads of a row quad are conflict free
constexpr int kI4StageW = kI4StepRows * kI4RowStride;
constexpr int kI4StageBytes = kI4StageW + kI4StepRows * 4;
constexpr int kI4WarpRing = kI4Stages * kI4StageBytes;
constexpr int kI4MinExp = -96;
constexpr int kI4MaxSmem = 226 * 1024;
constexpr int kI4MaxCluster = 8;
constexpr int kI4SplitRows = kI4SplitWarps * kI4StepRows;
// dynamic shared memory of the split kernel at most: its static partial-sum
// and receive buffers take the rest of the 227 KB
constexpr int kI4SplitSmemCap = kI4MaxSmem - (kI4SplitRows + kI4MaxCluster) * 4;


// ---------------------------------------------------------------------------
// product
// ---------------------------------------------------------------------------

__device__ __forceinline__ void i4_mma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1, bool zero)
{
    if (zero)
        asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%10,%10,%10,%10};"
                     : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
    else
        asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%0,%1,%2,%3};"
                     : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void i4_cp16(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void i4_cp4(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void i4_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void i4_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct I4Params {
    const uint16_t *x;  // bf16 activation; each CTA builds its slice's fragments from it
    const uint8_t *q;
    const uint16_t *scales;
    float *y;
    int N, K, npairs;
    int L;          // pairs per K-slice
    int act_smem;
};

// Issue one step: rows blk*32..+32, pair pidx (must be < pend).  Lane L
// copies 16-byte column L%4 of rows L/4 + {0,8,16,24}, and the two scales
// (4 bytes) of row L.
__device__ __forceinline__ void i4_issue(unsigned stage, const I4Params &p, int blk, int pidx, int pend, int lane)
{
    const int rowbytes = p.K >> 1, G = p.K >> 6;
    const int col = lane & 3;
    const int row0 = blk * kI4StepRows + (lane >> 2);
    const bool pok = pidx < pend;
    const uint8_t *src = p.q + (size_t)row0 * rowbytes + pidx * 64 + col * 16;
    const unsigned dst = stage + (lane >> 2) * kI4RowStride + col * 16;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const bool ok = pok && row0 + 8 * u < p.N;
        i4_cp16(dst + 8 * u * kI4RowStride, ok ? src + (size_t)(8 * u) * rowbytes : p.q, ok);
    }
    const int srow = blk * kI4StepRows + lane;
    const bool sok = pok && srow < p.N;
    i4_cp4(stage + kI4StageW + lane * 4, sok ? p.scales + (size_t)srow * G + 2 * pidx : p.scales, sok);
}

// Consume one staged step.  bf: this lane's fragments of the pair; gi: the
// (G, S) of this lane's group.
__device__ __forceinline__ void i4_consume(const uint8_t *st, const uint8_t *bf, float2 gi, int lane,
                                           float (&yacc)[2][2])
{
    const int g = lane >> 2, tq = lane & 3, h = tq >> 1;
    uint4 w[2][2];  // [tile][row g / g+8]: words 4(tq&1)..+3 of group h
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int r = 0; r < 2; ++r)
            w[t][r] = *reinterpret_cast<const uint4 *>(st + (16 * t + g + 8 * r) * kI4RowStride + h * 32 +
                                                       (tq & 1) * 16);
    int d[2][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint2 b = *reinterpret_cast<const uint2 *>(bf + u * 256);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t w0 = u == 0 ? w[t][0].x : u == 1 ? w[t][0].y : u == 2 ? w[t][0].z : w[t][0].w;
            const uint32_t w1 = u == 0 ? w[t][1].x : u == 1 ? w[t][1].y : u == 2 ? w[t][1].z : w[t][1].w;
            const uint32_t lo0 = (w0 & 0x0F0F0F0Fu) ^ 0x08080808u, hi0 = (w0 & 0xF0F0F0F0u) ^ 0x80808080u;
            const uint32_t lo1 = (w1 & 0x0F0F0F0Fu) ^ 0x08080808u, hi1 = (w1 & 0xF0F0F0F0u) ^ 0x80808080u;
            i4_mma(d[t], lo0, lo1, hi0, hi1, b.x, b.y, u == 0);
        }
    }
    const float coef = gi.x * ((tq & 1) ? 65536.f : 1.f);
    const float sub = (tq & 1) ? 0.f : gi.y;
    const float magic = 12582912.f;
    const float subc = fmaf(coef, magic, sub);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint16_t sc = *reinterpret_cast<const uint16_t *>(st + kI4StageW + (16 * t + g + 8 * r) * 4 + h * 2);
            const float hi = __int_as_float(d[t][2 * r + 1] + 0x4B400000) - magic;
            const float vm = fmaf(256.f, hi, __int_as_float(d[t][2 * r] + 0x4B400000));
            yacc[t][r] = fmaf(f16_bits_to_float(sc), fmaf(coef, vm, -subc), yacc[t][r]);
        }
}

constexpr int kI4BuildScratch = kI4SplitWarps * 4 * 128;  // limb scratch of the build

// Build the B fragments and group constants of one 128-k pair from x, in one
// warp: lane l takes k = 128 pr + 32 j + l (j = 0..3; j < 2 is the pair's
// first group), so every per-group reduction is a warp shuffle; the limbs
// go through lw (this warp's 4 x 128-byte scratch) to the fragment layout.
__device__ __forceinline__ void i4_build_pair_warp(const uint16_t *__restrict__ x, int K, int pr, uint8_t *frag,
                                                   float2 *info, int8_t (*lw)[128], int lane)
{
    float xv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = pr * kI4PairK + 32 * j + lane;
        xv[j] = k < K ? bf16_bits_to_float(x[k]) : 0.f;
    }
    int E[2], T[2] = {0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float mh = warp_max_nonneg(fmaxf(0.f, fmaxf(fabsf(xv[2 * h]), fabsf(xv[2 * h + 1]))));
        const int e8 = (int)((__float_as_uint(mh) >> 23) & 0xFFu);
        E[h] = max(e8 == 0 ? kI4MinExp : e8 - 126, kI4MinExp);  // smallest E with max|x| < 2^E
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int X = __float2int_rn(ldexpf(xv[j], 23 - E[j >> 1]));  // |X| <= 2^23
        T[j >> 1] += X;
        const int B = (lane & 1) ? X : X * 16;  // k & 1 == lane & 1: low nibbles carry q+8, high 16(q+8)
        const int l0 = (int)(int8_t)(B & 0xFF);
        int r = (B - l0) >> 8;
        const int l1 = (int)(int8_t)(r & 0xFF);
        r = (r - l1) >> 8;
        const int l2 = (int)(int8_t)(r & 0xFF);
        lw[0][32 * j + lane] = (int8_t)l0;
        lw[1][32 * j + lane] = (int8_t)l1;
        lw[2][32 * j + lane] = (int8_t)l2;
        lw[3][32 * j + lane] = (int8_t)((r - l2) >> 8);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int Th = warp_sum_int(T[h]);
        if (lane == 0)
            info[h] = (2 * pr + h) * 64 < K ? make_float2(ldexpf(1.0f, E[h] - 27), ldexpf((float)Th, E[h] - 20))
                                            : make_float2(0.f, 0.f);
    }
    __syncwarp();
    // B fragments: mma u (4 per pair), lane (n, t).  Register j, byte c holds
    // the k-slot of A register a(2j) byte c of thread t: nibble j of packed
    // byte 4*wi + c of group t/2, wi = 4(t&1) + u, i.e. k = 64(t/2) + 32(t&1)
    // + 8u + 2c + j.  Column n = 4*group + limb; the other group's lanes get 0.
    const int n = lane >> 2, t = lane & 3;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint32_t w[2] = {0u, 0u};
        if ((n >> 2) == (t >> 1)) {
            const int8_t *lb = lw[n & 3];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    w[j] |= (uint32_t)(uint8_t)lb[64 * (t >> 1) + 32 * (t & 1) + 8 * u + 2 * c + j] << (8 * c);
        }
        reinterpret_cast<uint2 *>(frag)[32 * u + lane] = make_uint2(w[0], w[1]);
    }
    __syncwarp();  // the scratch is reused for the warp's next pair
}

template <typename Out>
__device__ __forceinline__ void i4_finish(float (&yacc)[2][2], int lane, Out out)
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

__device__ __forceinline__ void i4_cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store a float into rank `rank`'s shared memory, at the address `local`
// has in this CTA.
__device__ __forceinline__ void i4_st_cluster(float *local, unsigned rank, float v)
{
    const unsigned a = (unsigned)__cvta_generic_to_shared(local);
    unsigned ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// grid: x = K-slice (cluster rank), y = 128-row block.  With one slice the
// cluster is a single CTA and its partial sums are the result.
__global__ void __launch_bounds__(kI4SplitWarps * 32) k_i4_m1_split(const I4Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float part[kI4SplitRows];
    __shared__ float recv[kI4SplitRows + kI4MaxCluster];  // [slice][share]: the partial sums pushed to this rank
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = blockIdx.x, nsl = gridDim.x, rb = blockIdx.y;
    const int blk = rb * kI4SplitWarps + warp;
    const int p_lo = slice * p.L, p_hi = min(p.npairs, p_lo + p.L);
    const int nsteps = blk * kI4StepRows < p.N && p_hi > p_lo ? p_hi - p_lo : 0;
    uint8_t *ring = smem + p.act_smem + warp * kI4WarpRing;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);

    int ist = 0;
    auto issue_next = [&]() {
        if (ist < nsteps) i4_issue(ring_s + (ist % kI4Stages) * kI4StageBytes, p, blk, p_lo + ist, p_hi, lane);
        ++ist;
        i4_commit();
    };
#pragma unroll
    for (int t = 0; t < kI4Stages - 1; ++t) issue_next();

    pdl_wait_primary();
    if (p_hi > p_lo) {
        const int n = p_hi - p_lo;
        int8_t(*lw)[128] = reinterpret_cast<int8_t(*)[128]>(smem + p.act_smem + kI4SplitWarps * kI4WarpRing +
                                                             warp * 4 * 128);
        float2 *info = reinterpret_cast<float2 *>(smem + (size_t)n * kI4FragBytesPerPair);
        for (int c = warp; c < n; c += kI4SplitWarps)
            i4_build_pair_warp(p.x, p.K, p_lo + c, smem + (size_t)c * kI4FragBytesPerPair, info + 2 * c, lw, lane);
    }
    __syncthreads();

    const uint8_t *bfrag = smem + lane * 8;
    const float2 *sinfo = reinterpret_cast<const float2 *>(smem + (size_t)(p_hi - p_lo) * kI4FragBytesPerPair) +
                          ((lane & 3) >> 1);
    float yacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    for (int s = 0; s < nsteps; ++s) {
        issue_next();
        i4_wait<kI4Stages - 1>();
        __syncwarp();
        i4_consume(ring + (s % kI4Stages) * kI4StageBytes, bfrag + s * kI4FragBytesPerPair, sinfo[2 * s], lane,
                   yacc);
        __syncwarp();
    }
    i4_wait<0>();
    i4_finish(yacc, lane, [&](int row, float v) { part[warp * kI4StepRows + row] = v; });

    if (nsl == 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < kI4SplitRows; i += blockDim.x)
            if (rb * kI4SplitRows + i < p.N) p.y[rb * kI4SplitRows + i] = part[i];
        return;
    }
    // rank q owns rows [q*per, (q+1)*per): every slice pushes its partial sums
    // of those rows into rank q's recv[slice], and after one cluster barrier
    // (release / acquire) rank q adds them up in rank order.  Nothing reads
    // another CTA's shared memory after the barrier, so each CTA may then
    // finish on its own.
    const int per = (kI4SplitRows + nsl - 1) / nsl;
    __syncthreads();  // part[] is complete
    for (int i = threadIdx.x; i < kI4SplitRows; i += blockDim.x) {
        const int q = i / per;
        i4_st_cluster(recv + slice * per + (i - q * per), (unsigned)q, part[i]);
    }
    i4_cluster_sync();
    for (int j = threadIdx.x; j < per && slice * per + j < kI4SplitRows; j += blockDim.x) {
        float sum = 0.f;
        for (int q = 0; q < nsl; ++q) sum += recv[q * per + j];
        const int row = rb * kI4SplitRows + slice * per + j;
        if (row < p.N) p.y[row] = sum;
    }
}

// ---------------------------------------------------------------------------
// grouped kernel: R matrices of one shape that read one x, persistent CTAs
// ---------------------------------------------------------------------------
//
// Cells are (matrix, 32-row block) over all of K, as in the Q1 persistent
// kernel: CTA b takes the cells [c0, c1), its warps take equal contiguous
// ranges of the cells' 128-k steps, and a cell cut between warps w and w+1
// is finished through shared memory (tail of w + head of w+1).  Every CTA
// builds the whole activation from x, one pair per warp at a time, with the
// limb scratch in the warp's idle ring slot.  Requires N % 32 == 0.

constexpr int kI4GMaxGroup = 256;
#ifndef LOWBIT_I4_LEAN_STAGES
#define LOWBIT_I4_LEAN_STAGES 3
#endif
#ifndef LOWBIT_I4_LEAN_WARPS
#define LOWBIT_I4_LEAN_WARPS 16
#endif
constexpr int kI4LStages = LOWBIT_I4_LEAN_STAGES;
constexpr int kI4LMaxWarps = LOWBIT_I4_LEAN_WARPS;
constexpr int kI4LMinWarps = 8;
static_assert(kI4LStages >= 2, "the build scratch lives in the last ring slot");

struct I4Group {
    const uint8_t *q[kI4GMaxGroup];
    const uint16_t *scales[kI4GMaxGroup];
    float *y[kI4GMaxGroup];
};

struct I4GParams {
    const uint16_t *x;
    int N, K, npairs, blocksN, cells, act_smem;
};

__global__ void __launch_bounds__(kI4LMaxWarps * 32, 1) k_i4_m1_lean(const __grid_constant__ I4Group grp,
                                                                     const I4GParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float part[2][kI4LMaxWarps][kI4StepRows];  // [head / tail][warp][row] of cut cells
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int c0 = (int)((long long)blockIdx.x * p.cells / gridDim.x);
    const int c1 = (int)((long long)(blockIdx.x + 1) * p.cells / gridDim.x);
    const int spc = p.npairs;  // steps per cell
    const int T = (c1 - c0) * spc;
    const int s0 = (int)((long long)warp * T / nw), s1 = (int)((long long)(warp + 1) * T / nw);
    const size_t rowbytes = (size_t)(p.K >> 1);
    const int G = p.K >> 6;
    uint8_t *ring = smem + p.act_smem + warp * (kI4LStages * kI4StageBytes);
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);

    // issue side: lane L copies 16-byte column L%4 of rows L/4 + {0,8,16,24}
    // and the scale pair of row L
    const unsigned wdst = (unsigned)((lane >> 2) * kI4RowStride + (lane & 3) * 16);
    const unsigned sdst = (unsigned)(kI4StageW + lane * 4);
    int is = s0, islot = 0, ir = 0, iblk = 0, ist = 0;
    const uint8_t *wsrc = nullptr;
    const uint16_t *ssrc = nullptr;
    auto cell_src = [&]() {
        wsrc = grp.q[ir] + (size_t)(iblk * kI4StepRows + (lane >> 2)) * rowbytes + (lane & 3) * 16 + ist * 64;
        ssrc = grp.scales[ir] + (size_t)(iblk * kI4StepRows + lane) * G + 2 * ist;
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
            const unsigned st = ring_s + islot * kI4StageBytes;
#pragma unroll
            for (int u = 0; u < 4; ++u) i4_cp16(st + wdst + 8 * u * kI4RowStride, wsrc + (size_t)(8 * u) * rowbytes, true);
            i4_cp4(st + sdst, ssrc, true);
            wsrc += 64;
            ssrc += 2;
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
        i4_commit();
        islot = islot + 1 == kI4LStages ? 0 : islot + 1;
    };
#pragma unroll
    for (int t = 0; t < kI4LStages - 1; ++t) issue_next();

    pdl_wait_primary();  // x and the outputs follow stream order from here
    float2 *info = reinterpret_cast<float2 *>(smem + (size_t)p.npairs * kI4FragBytesPerPair);
    {
        int8_t(*lw)[128] = reinterpret_cast<int8_t(*)[128]>(ring + (kI4LStages - 1) * kI4StageBytes);
        for (int pr = warp; pr < p.npairs; pr += nw)
            i4_build_pair_warp(p.x, p.K, pr, smem + (size_t)pr * kI4FragBytesPerPair, info + 2 * pr, lw, lane);
    }
    __syncthreads();

    const uint8_t *bfrag = smem + lane * 8;
    const float2 *sinfo = info + ((lane & 3) >> 1);
    int s = s0, slot = 0;
    while (s < s1) {
        const int cell = c0 + s / spc, st0 = s % spc;
        const int st1 = min(spc, st0 + (s1 - s));
        float yacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        for (int t = st0; t < st1; ++t) {
            issue_next();
            i4_wait<kI4LStages - 1>();
            __syncwarp();
            i4_consume(ring + slot * kI4StageBytes, bfrag + t * kI4FragBytesPerPair, sinfo[2 * t], lane, yacc);
            __syncwarp();  // every lane is done with this stage before it is refilled
            slot = slot + 1 == kI4LStages ? 0 : slot + 1;
        }
        s += st1 - st0;
        const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
        float *yr = grp.y[r] + blk * kI4StepRows;
        float *cut = st0 > 0 ? part[0][warp] : (st1 < spc ? part[1][warp] : nullptr);
        i4_finish(yacc, lane, [&](int row, float v) {
            if (cut != nullptr)
                cut[row] = v;
            else
                yr[row] = v;
        });
    }
    i4_wait<0>();
    __syncthreads();
    if (warp + 1 < nw && s1 % spc != 0 && s1 > s0) {
        const int cell = c0 + s1 / spc;
        const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
        grp.y[r][blk * kI4StepRows + lane] = part[1][warp][lane] + part[0][warp + 1][lane];
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct I4Plan {
    int npairs, L, nslices, blocks;
    size_t act_smem, smem;
    bool ok;
};

static I4Plan i4_plan(int N, int K, int sms)
{
    I4Plan P = {};
    P.npairs = (K + kI4PairK - 1) / kI4PairK;
    P.blocks = (N + kI4SplitRows - 1) / kI4SplitRows;
    const size_t per_pair = kI4FragBytesPerPair + kI4InfoBytesPerPair;
    const size_t ring = (size_t)kI4SplitWarps * kI4WarpRing;
    // enough CTAs for several per SM, and each CTA's activation slice in smem
    int S = (int)std::min<long long>(
        kI4MaxCluster, std::max<long long>(1, ((long long)LOWBIT_I4_CTAS_PER_SM * sms + P.blocks - 1) / P.blocks));
    if (LOWBIT_I4_FILL) S = std::max(S, (P.npairs + kI4Stages - 1) / kI4Stages);  // whole slice in flight
    S = std::min(std::min(S, kI4MaxCluster), P.npairs);
    while (true) {
        P.L = (P.npairs + S - 1) / S;
        P.nslices = (P.npairs + P.L - 1) / P.L;
        P.act_smem = ((size_t)P.L * per_pair + 15) & ~size_t(15);
        P.smem = P.act_smem + ring + kI4BuildScratch;
        if (P.smem <= (size_t)kI4SplitSmemCap || S >= kI4MaxCluster) break;
        S = std::min(kI4MaxCluster, S * 2);
    }
    P.ok = P.smem <= (size_t)kI4SplitSmemCap && P.blocks < 65536 && (K / 64) % 2 == 0;
    return P;
}

static int i4_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

bool i4m1_supported(int N, int K) { return i4_plan(N, K, i4_num_sms()).ok; }

lowbit_status i4m1_launch(const uint8_t *q, const uint16_t *scales, const uint16_t *x, float *y, int N, int K,
                          cudaStream_t st)
{
    // one launch: every CTA turns its K-slice of x into fragments itself
    const I4Plan P = i4_plan(N, K, i4_num_sms());
    cudaError_t e;
    I4Params p = {};
    p.x = x;
    p.q = q;
    p.scales = scales;
    p.y = y;
    p.N = N;
    p.K = K;
    p.npairs = P.npairs;
    p.L = P.L;
    p.act_smem = (int)P.act_smem;
    if (cudaFuncSetAttribute(k_i4_m1_split, cudaFuncAttributeMaxDynamicSharedMemorySize, kI4SplitSmemCap) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.nslices, P.blocks);
    cfg.blockDim = dim3(kI4SplitWarps * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = P.nslices;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, k_i4_m1_split, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// Grouped plan: one CTA per SM with as many warps (<= kI4LMaxWarps) as fit
// next to the whole activation and as there are cells per SM (each warp needs
// one cell's worth of steps); fewer than kI4LMinWarps falls back to single
// calls.  The smaller the rings, the more of the SM's memory stays L1 for
// the 4-byte scale copies, which is why three stages beat deeper rings.
struct I4GPlan {
    int npairs, blocksN, warps;
    size_t act_smem, smem;
    bool ok;
};

static I4GPlan i4g_plan(int R, int N, int K, int sms)
{
    I4GPlan P = {};
    P.npairs = K / kI4PairK;
    P.blocksN = N / kI4StepRows;
    if (R < 1 || R > kI4GMaxGroup || N % kI4StepRows != 0 || K % kI4PairK != 0 || P.npairs < 1) return P;
    P.act_smem = (size_t)P.npairs * (kI4FragBytesPerPair + kI4InfoBytesPerPair);
    const size_t cap = (size_t)kI4MaxSmem - 2 * kI4LMaxWarps * kI4StepRows * 4;  // static cut buffers
    const size_t per_warp = (size_t)kI4LStages * kI4StageBytes;
    const long long fit = P.act_smem < cap ? (long long)((cap - P.act_smem) / per_warp) : 0;
    P.warps = (int)std::min<long long>(std::min<long long>(kI4LMaxWarps, fit), (long long)R * P.blocksN / sms);
    P.smem = P.act_smem + (size_t)P.warps * per_warp;
    P.ok = P.warps >= kI4LMinWarps;
    return P;
}

bool i4m1_group_supported(int R, int N, int K) { return i4g_plan(R, N, K, i4_num_sms()).ok; }

lowbit_status i4m1_group_launch(const uint8_t *const *q, const uint16_t *const *scales, const uint16_t *x,
                                float *const *y, int R, int N, int K, cudaStream_t st)
{
    const int sms = i4_num_sms();
    const I4GPlan P = i4g_plan(R, N, K, sms);
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    static I4Group grp;  // large: kept off the stack
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int r = 0; r < R; ++r) {
        grp.q[r] = q[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    I4GParams p = {};
    p.x = x;
    p.N = N;
    p.K = K;
    p.npairs = P.npairs;
    p.blocksN = P.blocksN;
    p.cells = R * P.blocksN;
    p.act_smem = (int)P.act_smem;
    if (cudaFuncSetAttribute(k_i4_m1_lean, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(P.warps * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_i4_m1_lean, grp, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
