// q1_gemm_smallm.cu -- Q1_0_g128 products at small batch (2 <= M <= 16) on
// the bf16 tensor cores (mma.sync m16n8k16, fp32 accumulate).
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
// Work split (as for the M = 1 kernels): a warp owns 32 rows (two 16-row
// tiles); a CTA of four warps 128 rows of one K-slice; the S slices of a row
// block form a thread-block cluster and add their partial sums in rank order
// through distributed shared memory.  The CTA stages its slice of x in
// shared memory in fragment order; every warp streams its rows' sign bits
// and scales through a cp.async ring, 256 k per step.
#include <algorithm>

#include "common.cuh"

namespace lowbit {

constexpr int kSmWarps = 4;
constexpr int kSmRows = kSmWarps * 32;     // rows per CTA
constexpr int kSmStepK = 256;              // k per pipeline step (two groups)
constexpr int kSmRowStride = 48;           // 32 bytes of signs per row, padded: conflict-free 16-byte reads
constexpr int kSmStageW = 32 * kSmRowStride;
constexpr int kSmStageBytes = kSmStageW + 32 * 4;  // + two fp16 scales per row
constexpr int kSmStages = 4;
constexpr int kSmRing = kSmStages * kSmStageBytes;
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
    int NT;      // n8 tiles of the batch: 1 (M <= 8) or 2
    int xfrag;   // bytes of staged x fragments
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

// grid: x = K-slice (cluster rank), y = 128-row block
template <int NT>
__global__ void __launch_bounds__(kSmWarps * 32) k_q1_smallm(const SmParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ uint2 lut[16];
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = blockIdx.x, nsl = gridDim.x, rb = blockIdx.y;
    const int blk = rb * kSmWarps + warp;
    const int s_lo = slice * p.L, s_hi = min(p.nsteps, s_lo + p.L);
    const int nst = blk * 32 < p.N && s_hi > s_lo ? s_hi - s_lo : 0;
    uint8_t *ring = smem + p.xfrag + warp * kSmRing;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);
    float *part = reinterpret_cast<float *>(smem + p.xfrag + kSmWarps * kSmRing);  // [M][128]

    int ist = 0;
    auto issue_next = [&]() {
        if (ist < nst) sm_issue(ring_s + (ist % kSmStages) * kSmStageBytes, p, blk, s_lo + ist, lane);
        ++ist;
        sm_commit();
    };
#pragma unroll
    for (int t = 0; t < kSmStages - 1; ++t) issue_next();

    // nibble -> two bf16x2: bit j of the nibble is the sign of k slot 4t + j
    if (threadIdx.x < 16) {
        const uint32_t v = threadIdx.x;
        auto s = [&](int j) -> uint32_t { return ((v >> j) & 1u) ? 0x3F80u : 0xBF80u; };
        lut[threadIdx.x] = make_uint2(s(0) | (s(1) << 16), s(2) | (s(3) << 16));
    }
    pdl_wait_primary();  // x is produced by earlier kernels
    // x fragments of this slice: step ks, tile nt, lane (g, t) -> x[8 nt + g][k .. k+3], k = 16 ks + 4 t,
    // copied asynchronously (all in flight at once; zeros past the batch)
    uint2 *xf = reinterpret_cast<uint2 *>(smem);
    const unsigned xf_s = (unsigned)__cvta_generic_to_shared(xf);
    const int nfr = (s_hi - s_lo) * 16 * NT * 32;
    for (int i = threadIdx.x; i < nfr; i += blockDim.x) {
        const int ln = i & 31, nt = (i >> 5) % NT, ks = (i >> 5) / NT;
        const int m = 8 * nt + (ln >> 2);
        const int k = s_lo * kSmStepK + 16 * ks + 4 * (ln & 3);
        sm_cp8(xf_s + 8u * i, m < p.M ? p.x + (size_t)m * p.K + k : p.x, m < p.M);
    }
    sm_commit();
    sm_wait<0>();  // (also the weight stages issued so far)
    __syncthreads();

    float yacc[2][NT][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
    for (int s = 0; s < nst; ++s) {
        issue_next();
        sm_wait<kSmStages - 1>();
        __syncwarp();
        sm_consume<NT>(ring + (s % kSmStages) * kSmStageBytes, xf + s * 16 * NT * 32, lut, lane, yacc);
        __syncwarp();
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
    size_t xfrag, smem;
    bool ok;
};

static SmPlan sm_plan(int M, int N, int K, int sms)
{
    SmPlan P = {};
    P.NT = M <= 8 ? 1 : 2;
    P.nsteps = K / kSmStepK;
    P.blocks = (N + kSmRows - 1) / kSmRows;
    if (M < 2 || M > kSmMaxM || N < 1 || K % kSmStepK != 0 || P.nsteps < 1) return P;  // ok = false
    const size_t ring = (size_t)kSmWarps * kSmRing, part = (size_t)M * kSmRows * 4;
    int S = (int)std::min<long long>(kSmMaxCluster, std::max<long long>(1, (2LL * sms + P.blocks - 1) / P.blocks));
    S = std::min(S, P.nsteps);
    while (true) {
        P.L = (P.nsteps + S - 1) / S;
        P.S = (P.nsteps + P.L - 1) / P.L;
        P.xfrag = (size_t)P.L * 16 * P.NT * 32 * 8;
        P.smem = P.xfrag + ring + part;
        if (P.smem <= (size_t)kSmMaxSmem || S >= std::min(kSmMaxCluster, P.nsteps)) break;
        S = std::min(std::min(kSmMaxCluster, P.nsteps), S * 2);
    }
    P.ok = M >= 2 && M <= kSmMaxM && K % kSmStepK == 0 && P.nsteps >= 1 && P.smem <= (size_t)kSmMaxSmem &&
           P.blocks < 65536;
    return P;
}

static int sm_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

bool q1sm_supported(int M, int N, int K) { return sm_plan(M, N, K, sm_num_sms()).ok; }

lowbit_status q1sm_launch(const uint8_t *bits, const uint16_t *scales, const uint16_t *x, float *y, int M, int N,
                          int K, cudaStream_t st)
{
    const SmPlan P = sm_plan(M, N, K, sm_num_sms());
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
    p.xfrag = (int)P.xfrag;
    void (*kern)(const SmParams) = P.NT == 1 ? k_q1_smallm<1> : k_q1_smallm<2>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmMaxSmem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.S, P.blocks);
    cfg.blockDim = dim3(kSmWarps * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = P.S;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
