// int4_gemm_tc.cu -- INT4_G64 prefill GEMM on the 5th-generation tensor
// cores (tcgen05.mma, kind::f16, bf16 operands, fp32 accumulation in TMEM).
//
// What is computed ("acorn-llm 0.11.4", "int4 quantisation quality: group
// quantisation"; the page's GPU kernel does the same product as a "multi-row
// GEMM" for prefill):
//     y[m][n] = sum_g d[n][g] * sum_{k in g} q[n][k] * x[m][k].
//
// Exactness with one MMA per weight.  The integer q in [-8, 7] is exact in
// bf16, and so is x; the tensor core forms every product q x exactly and sums
// one 64-k group in fp32.  The group scale is applied outside the MMA: each
// group accumulates into a TMEM buffer of its own (two buffers, alternating),
// and the epilogue warps read it with tcgen05.ld and add d * D into fp32
// registers while the tensor core works on the next group.  (A bf16 copy of
// q * d would round the 15-bit product to 8 bits, about 1e-3 relative error.)
//
// q -> bf16: for a byte holding nibbles lo, hi, (byte * 0x1001) & 0x000F000F
// puts lo in the low half-word and hi in the high one; xor 8 maps a two's-
// complement nibble q to q + 8 in 0..15, and or-ing 0x4300 makes each half
// the bf16 number 128 + (q + 8) (exponent 2^7, mantissa step 1); subtracting
// 136 from both halves (bf16x2, exact) leaves q.
//
// CTA tile: 128 weight rows (the MMA's M) x BM batch rows (its N, <= 256),
// one of S slices of K (whole 64-k groups) when there are too few tiles to
// fill the SMs (S picked to minimise waves x groups per CTA; the slices add
// their sums into y, zeroed first, with fp32 reductions), in steps of one
// group, three shared-memory stages, two TMEM accumulators of BM columns:
//   warps 0-7  dequantise a stage's packed weights into the A tile (K-major,
//              128-byte swizzle), then drain the finished group's TMEM buffer
//              (warp w reads TMEM lanes 32 (w % 4).., columns of half w / 4)
//              and keep the scaled sums in registers; at the end they store
//              (one slice) or add (several) them to y;
//   warp 8     loads the x tile of a stage with TMA (128-byte swizzle);
//   warp 9     allocates TMEM, and one of its lanes issues a group's four
//              K = 16 MMAs and commits them to the stage's "empty" barrier
//              and to the TMEM buffer's "full" barrier.
// Every mbarrier wait is bounded in time; a wait that runs out records a
// fault flag and the CTA leaves its loops, releases TMEM and exits.
#include <algorithm>
#include <mutex>

#include "tc_common.cuh"

namespace lowbit {

constexpr int kTcBN = 128;             // weight rows per CTA
constexpr int kTcBK = 64;              // k per stage (one scale group)
constexpr int kTcStages = 3;
constexpr int kTcProdWarps = 8;
constexpr int kTcTmaWarp = kTcProdWarps;
constexpr int kTcMmaWarp = kTcProdWarps + 1;
constexpr int kTcThreads = (kTcProdWarps + 2) * 32;
constexpr int kTcATile = kTcBN * kTcBK * 2;        // 16 KiB of bf16
constexpr int kTcBTile = 256 * kTcBK * 2;          // 32 KiB of bf16 (BM <= 256)
constexpr int kTcStageBytes = kTcATile + kTcBTile;
constexpr int kTcPf = 4;                           // groups of packed weights copied ahead
constexpr int kTcPfBuf = kTcPf + 1;
constexpr int kTcPfBytes = kTcBN * 32;             // one group's packed nibbles of the tile (4 KiB)
constexpr int kTcSmemBytes = kTcStages * kTcStageBytes + kTcPfBuf * kTcPfBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr int kTcTmemCols = 512;       // two accumulators of up to 256 columns

__device__ unsigned g_tc_fault;  // set when a bounded wait ran out

// UMMA shared-memory descriptor: K-major operand with 128-byte swizzle, rows
// 128 bytes apart, 8-row groups 1024 bytes apart (tile base 1024-aligned).
__device__ __forceinline__ uint64_t umma_desc_sw128(const void *smem_tile)
{
    const uint64_t addr = (unsigned)__cvta_generic_to_shared(smem_tile);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) /*LBO (unused)*/ | (64ull << 32) /*SBO 1024 B*/ |
           (1ull << 46) /*version*/ | (2ull << 61) /*SWIZZLE_128B*/;
}

// D (+)= A x B, both from shared memory.  ACC (accumulate into D) is an
// immediate: a predicate computed from a register slows every MMA issue.
template <bool ACC>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "n"(ACC ? 1 : 0));
}

// Eight nibbles (k = 8c .. 8c+7, low nibble first) -> eight exact bf16.
__device__ __forceinline__ uint4 q8_to_bf16(uint32_t word)
{
    uint32_t o[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (word >> (8 * b)) & 0xFFu;
        const uint32_t v = ((byte * 0x1001u) & 0x000F000Fu) ^ 0x43084308u;   // 128 + q + 8 in each half
        uint32_t r;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x43084308u));  // minus 136: q, exactly
        o[b] = r;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// One thread's row of a finished group: 32 * NCH TMEM columns (BM / 2),
// read 16 at a time, LOWBIT_I4TC_DRAIN loads in flight before each wait
// (fewer live registers than one 32-column load next to the 128
// accumulators), and acc += d * D.
// fixed cost of a wave of CTAs, in groups, for the choice of K slices
#ifndef LOWBIT_I4TC_SLICE_COST
#define LOWBIT_I4TC_SLICE_COST 8
#endif
#ifndef LOWBIT_I4TC_DRAIN
#define LOWBIT_I4TC_DRAIN 2
#endif
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

template <int NCH>  // 32-column chunks a thread drains (BM / 64)
__device__ __forceinline__ void drain_group(uint32_t taddr, float d, float (&acc)[128])
{
    constexpr int D = LOWBIT_I4TC_DRAIN;
#pragma unroll
    for (int c0 = 0; c0 < 2 * NCH; c0 += D) {
        uint32_t v[D][16];
#pragma unroll
        for (int u = 0; u < D; ++u)
            if (c0 + u < 2 * NCH) tmem_ld16(taddr + 16u * (c0 + u), v[u]);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int u = 0; u < D; ++u)
            if (c0 + u < 2 * NCH)
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc[16 * (c0 + u) + i] = fmaf(d, __uint_as_float(v[u][i]), acc[16 * (c0 + u) + i]);
    }
}

template <int NCH>
__global__ void __launch_bounds__(kTcThreads, 1) k_i4_tc_gemm(const __grid_constant__ CUtensorMap tmap_x,
                                                              const uint8_t *__restrict__ q,
                                                              const uint16_t *__restrict__ scales,
                                                              float *__restrict__ y, int M, int N, int K)
{
    constexpr int BM = 64 * NCH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *pfbuf = smem + kTcStages * kTcStageBytes;     // packed weights copied ahead (cp.async)
    uint64_t *full_a = reinterpret_cast<uint64_t *>(pfbuf + kTcPfBuf * kTcPfBytes);
    uint64_t *full_b = full_a + kTcStages;
    uint64_t *empty = full_b + kTcStages;
    uint64_t *tfull = empty + kTcStages;    // [2]: a group's MMAs have completed in TMEM buffer b
    uint64_t *tempty = tfull + 2;           // [2]: the epilogue has read TMEM buffer b
    uint64_t *done = tempty + 2;            // every MMA the CTA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTcBN, m0 = blockIdx.y * BM;
    // this CTA's groups [g0, g0 + ngroups) of K: slice blockIdx.z of gridDim.z
    const int gall = K / kTcBK;
    const int g0 = gall * blockIdx.z / gridDim.z, ngroups = gall * (blockIdx.z + 1) / gridDim.z - g0;
    const bool sliced = gridDim.z > 1;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(full_a + s, kTcProdWarps);
            mbar_init(full_b + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, kTcProdWarps);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == kTcMmaWarp) tmem_alloc(tmem_slot, kTcTmemCols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    bool ok = true;

    if (warp < kTcProdWarps) {
        // ---- producers (weight row r, k half hf of each group) and drainers
        //      (TMEM lane quarter warp % 4, column half warp / 4) ----
        const int t = threadIdx.x, r = t >> 1, hf = t & 1;
        const int n = n0 + r;
        const bool valid = n < N;
        const uint8_t *qrow = q + (size_t)(valid ? n : 0) * (K / 2) + (size_t)g0 * 32 + hf * 16;
        const int quarter = warp & 3, half = warp >> 2;
        const int ne = n0 + quarter * 32 + lane;            // this thread's output row in the epilogue
        const uint16_t *srow = scales + (size_t)(ne < N ? ne : 0) * (K / 64) + g0;
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.f;

        // this thread's 16 bytes of packed nibbles of group it, copied kTcPf
        // groups ahead into a ring of its own (it reads back only what it
        // copied, so its own cp.async wait is all the ordering needed)
        const unsigned pf_s = (unsigned)__cvta_generic_to_shared(pfbuf) + (unsigned)(t * 16);
        auto prefetch = [&](int it) {
            if (valid && it < ngroups)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(pf_s + (unsigned)((it % kTcPfBuf) * kTcPfBytes)),
                             "l"(qrow + (size_t)it * 32)
                             : "memory");
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        auto produce = [&](int it) -> bool {   // dequantise group it into stage it % S
            const int s = it % kTcStages, j = it / kTcStages;
            prefetch(it + kTcPf);
            asm volatile("cp.async.wait_group %0;" ::"n"(kTcPf) : "memory");
            const uint4 pk = valid ? *reinterpret_cast<const uint4 *>(pfbuf + (it % kTcPfBuf) * kTcPfBytes + t * 16)
                                   : make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
            if (it >= kTcStages && !mbar_wait(empty + s, (j - 1) & 1, &g_tc_fault)) return false;
            uint8_t *a = smem + s * kTcStageBytes;
            const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int chunk = hf * 4 + c;                        // 16-byte chunk = 8 k
                *reinterpret_cast<uint4 *>(a + r * 128 + ((chunk ^ (r & 7)) << 4)) = q8_to_bf16(words[c]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(full_a + s);
            return true;
        };
        for (int it = 0; it < kTcPf; ++it) prefetch(it);
        // rows past N dequantise nibble 8 (q = -8); their outputs are not stored
        for (int it = 0; it < kTcStages - 1 && it < ngroups && ok; ++it) ok = produce(it);
        // the raw fp16 scales of the next two groups, converted only when used
        // (converting right after the load would wait out its latency)
        uint16_t d0 = ne < N ? __ldg(srow) : (uint16_t)0, d1 = ne < N && 1 < ngroups ? __ldg(srow + 1) : (uint16_t)0;
        for (int g = 0; g < ngroups && ok; ++g) {
            if (g + kTcStages - 1 < ngroups && !produce(g + kTcStages - 1)) {
                ok = false;
                break;
            }
            const uint16_t dbits = d0;
            d0 = d1;
            d1 = g + 2 < ngroups && ne < N ? __ldg(srow + g + 2) : (uint16_t)0;
            const float d = f16_bits_to_float(dbits);
            const int b = g & 1;
            if (!mbar_wait_warp(tfull + b, (g >> 1) & 1, &g_tc_fault)) {
                ok = false;
                break;
            }
            tc_fence_after();
            drain_group<NCH>(tmem_d + tlane + (uint32_t)(b * 256 + half * (BM / 2)), d, acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + b);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        pdl_wait_primary();  // y may still be read by an earlier kernel
        if (ok && ne < N) {
            if (sliced) {
#pragma unroll
                for (int i = 0; i < 32 * NCH; ++i) {
                    const int m = m0 + half * (BM / 2) + i;
                    if (m < M) atomicAdd(y + (size_t)m * N + ne, acc[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32 * NCH; ++i) {
                    const int m = m0 + half * (BM / 2) + i;
                    if (m < M) y[(size_t)m * N + ne] = acc[i];
                }
            }
        }
    } else if (warp == kTcTmaWarp) {
        if (lane == 0) {
            pdl_wait_primary();  // x follows stream order
            int issued = 0;
            for (int it = 0; it < ngroups; ++it) {
                const int s = it % kTcStages, j = it / kTcStages;
                if (it >= kTcStages && !mbar_wait(empty + s, (j - 1) & 1, &g_tc_fault)) break;
                mbar_arrive_expect_tx(full_b + s, (unsigned)(BM * kTcBK * 2));
                tma_load_2d(smem + s * kTcStageBytes + kTcATile, &tmap_x, (g0 + it) * kTcBK, m0, full_b + s);
                ++issued;
            }
            // the copies still in flight land before the CTA may exit (they
            // have, unless a wait somewhere ran out)
            for (int it = std::max(0, issued - kTcStages); it < issued; ++it)
                mbar_wait(full_b + it % kTcStages, (it / kTcStages) & 1, &g_tc_fault);
        }
    } else {
        // MMA issue: the whole warp runs the loop (uniform operands), one
        // elected lane issues.  instruction descriptor: f32 accumulate, bf16
        // A and B, both K-major, N = BM, M = 128
        const uint32_t idesc =
            (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BM >> 3) << 17) | ((uint32_t)(kTcBN >> 4) << 24);
        for (int it = 0; it < ngroups; ++it) {
            const int s = it % kTcStages, j = it / kTcStages, b = it & 1;
            if (!mbar_wait_warp(full_a + s, j & 1, &g_tc_fault) || !mbar_wait_warp(full_b + s, j & 1, &g_tc_fault) ||
                (it >= 2 && !mbar_wait_warp(tempty + b, ((it >> 1) - 1) & 1, &g_tc_fault))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint8_t *st = smem + s * kTcStageBytes;
            const uint64_t ad = umma_desc_sw128(st), bd = umma_desc_sw128(st + kTcATile);
            const uint32_t dt = tmem_d + (uint32_t)(b * 256);
            if (elect_one()) {
                // advancing 16 k (32 bytes) inside the swizzle atom: +2 in 16-byte units
                umma_bf16<false>(dt, ad, bd, idesc);
#pragma unroll
                for (int kk = 1; kk < kTcBK / 16; ++kk) umma_bf16<true>(dt, ad + 2 * kk, bd + 2 * kk, idesc);
                umma_commit(empty + s);
                umma_commit(tfull + b);
            }
            __syncwarp();
        }
        // also after a failed wait: `done` tells that every MMA issued has
        // completed, before tensor memory is released
        if (elect_one()) umma_commit(done);
        __syncwarp();
        mbar_wait_warp(done, 0, &g_tc_fault);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_d, kTcTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

bool i4tc_supported(int M, int N, int K)
{
    (void)N;
    return M >= 16 && K % 64 == 0 && K >= 64;
}

lowbit_status i4tc_launch(const uint8_t *q, const uint16_t *scales, const uint16_t *x, float *y, int M, int N, int K,
                          cudaStream_t st)
{
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return LOWBIT_ERR_CUDA;
    // BM a multiple of 64 keeps each drain warp's column range a multiple of
    // the 32-column TMEM load; rows past M are zero-filled by TMA
    const int BM = std::min(256, (M + 63) / 64 * 64);
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)BM};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LOWBIT_ERR_CUDA;
    void (*kern)(const CUtensorMap, const uint8_t *, const uint16_t *, float *, int, int, int) =
        BM == 64 ? k_i4_tc_gemm<1> : BM == 128 ? k_i4_tc_gemm<2> : BM == 192 ? k_i4_tc_gemm<3> : k_i4_tc_gemm<4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = ((N + kTcBN - 1) / kTcBN) * ((M + BM - 1) / BM), gall = K / kTcBK;
    // K slices: fewest waves x groups per CTA, plus a fixed cost of about
    // kTcSliceCost groups per wave (setup, pipeline fill, the final stores)
    constexpr int kTcMaxSlices = 8, kTcSliceCost = LOWBIT_I4TC_SLICE_COST;
    int S = 1;
    long long best = -1;
    for (int c = 1; c <= std::min(kTcMaxSlices, gall); ++c) {
        const long long waves = ((long long)tiles * c + sms - 1) / sms;
        const long long cost = waves * ((gall + c - 1) / c + kTcSliceCost);
        if (best < 0 || cost < best) {
            best = cost;
            S = c;
        }
    }
    if (S > 1 && cudaMemsetAsync(y, 0, (size_t)M * N * sizeof(float), st) != cudaSuccess) return LOWBIT_ERR_CUDA;
    dim3 grid((N + kTcBN - 1) / kTcBN, (M + BM - 1) / BM, S);
    cudaError_t e = launch_pdl(kern, grid, dim3(kTcThreads), kTcSmemBytes, st, map, q, scales, y, M, N, K);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// Read and clear the fault flag of the current device.
int i4tc_fault_flag()
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_fault, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_tc_fault, &zero, sizeof(zero));
    return (int)v;
}

}  // namespace lowbit
