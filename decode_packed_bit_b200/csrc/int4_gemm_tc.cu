// int4_gemm_tc.cu -- INT4_G64 prefill GEMM on the 5th-generation tensor
// cores (tcgen05.mma, kind::f16, bf16 operands, fp32 accumulation in TMEM).
//
// What is computed ("acorn-llm 0.11.4", "int4 quantisation quality: group
// quantisation"; the page's GPU kernel does the same product as a "multi-row
// GEMM" for prefill):
//     y[m][n] = sum_g d[n][g] * sum_{k in g} q[n][k] * x[m][k].
//
// Exact dequantisation.  A bf16 copy of q*d would round the product (15
// significant bits) to 8 and cost ~1e-3 relative error.  Instead each weight
// is written as two bf16 numbers, hi = bf16_rn(q*d) and lo = q*d - hi, whose
// sum is q*d exactly (the residual needs at most 7 significant bits).  The
// tensor core multiplies both halves by the same x tile and accumulates in
// fp32, so the only rounding is the fp32 accumulation; the group scale is
// inside the operand and no per-group epilogue is needed.
//
// CTA tile: 128 weight rows (the MMA's M) x BM batch rows (its N, <= 256),
// K in steps of one 64-k scale group, three pipeline stages:
//   warps 0-7  dequantise the packed weights of a stage into the hi and lo
//              A tiles (K-major, 128-byte swizzle) and, at the end, read the
//              accumulator out of TMEM and store y;
//   warp 8     loads the x tile of a stage with TMA (128-byte swizzle);
//   warp 9     allocates TMEM, and one of its lanes issues the MMAs
//              (4 x K=16 for hi, 4 for lo per stage) and commits them to the
//              stage's "empty" barrier.
// Every mbarrier wait is bounded in time; a wait that runs out records a
// fault flag and the CTA leaves its loops, releases TMEM and exits.
#include <algorithm>
#include <mutex>

#include "tc_common.cuh"

namespace lowbit {

constexpr int kTcBN = 128;             // weight rows per CTA
constexpr int kTcBK = 64;              // k per stage (one scale group)
constexpr int kTcStages = 3;
constexpr int kTcPrefetch = 4;          // groups of packed weights loaded ahead
constexpr int kTcProdWarps = 8;
constexpr int kTcTmaWarp = kTcProdWarps;
constexpr int kTcMmaWarp = kTcProdWarps + 1;
constexpr int kTcThreads = (kTcProdWarps + 2) * 32;
constexpr int kTcATile = kTcBN * kTcBK * 2;        // 16 KiB of bf16
constexpr int kTcBTile = 256 * kTcBK * 2;          // 32 KiB of bf16 (BM <= 256)
constexpr int kTcStageBytes = 2 * kTcATile + kTcBTile;
constexpr int kTcSmemBytes = kTcStages * kTcStageBytes + 1024 /*align*/ + 256 /*barriers*/;

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

// bf16 pair, round to nearest even, lo in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Dequantise 8 nibbles (k = 8c..8c+7 of a group, low nibble first) with
// scale d into 8 hi and 8 lo bf16 values.
__device__ __forceinline__ void dequant8(uint32_t word, float d, uint4 &hi, uint4 &lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float w[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t nib = (word >> (8 * b + 4 * j)) & 0xFu;
            // (nib ^ 8) in the mantissa of 2^23: exactly q + 8 after the subtraction
            const float q = __uint_as_float(0x4B000000u | (nib ^ 8u)) - 8388616.0f;
            w[j] = q * d;  // exact: 4-bit integer times an fp16 value
        }
        const uint32_t hh = pack_bf16x2(w[0], w[1]);
        const float r0 = w[0] - __uint_as_float(hh << 16);
        const float r1 = w[1] - __uint_as_float(hh & 0xFFFF0000u);
        h[b] = hh;
        l[b] = pack_bf16x2(r0, r1);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__global__ void __launch_bounds__(kTcThreads, 1) k_i4_tc_gemm(const __grid_constant__ CUtensorMap tmap_x,
                                                              const uint8_t *__restrict__ q,
                                                              const uint16_t *__restrict__ scales,
                                                              float *__restrict__ y, int M, int N, int K, int BM)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + kTcStages * kTcStageBytes);
    uint64_t *full_b = full_a + kTcStages;
    uint64_t *empty = full_b + kTcStages;
    uint64_t *done = empty + kTcStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTcBN, m0 = blockIdx.y * BM;
    const int ngroups = K / kTcBK;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(full_a + s, kTcProdWarps);
            mbar_init(full_b + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == kTcMmaWarp) {
        tmem_alloc(tmem_slot, 256);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    bool ok = true;

    if (warp < kTcProdWarps) {
        // ---- producers: weight row r, k half hf of each group ----
        const int t = threadIdx.x, r = t >> 1, hf = t & 1;
        const int n = n0 + r;
        const bool valid = n < N;
        const uint8_t *qrow = q + (size_t)(valid ? n : 0) * (K / 2) + hf * 16;
        const uint16_t *srow = scales + (size_t)(valid ? n : 0) * (K / 64);
        // packed weights and scales are loaded kTcPrefetch groups ahead
        uint4 pkb[kTcPrefetch];
        float db[kTcPrefetch];
#pragma unroll
        for (int u = 0; u < kTcPrefetch; ++u) {
            pkb[u] = make_uint4(0u, 0u, 0u, 0u);
            db[u] = 0.f;
            if (valid && u < ngroups) {
                pkb[u] = __ldg(reinterpret_cast<const uint4 *>(qrow + u * 32));
                db[u] = f16_bits_to_float(__ldg(srow + u));
            }
        }
        for (int it0 = 0; it0 < ngroups && ok; it0 += kTcPrefetch) {
#pragma unroll
            for (int u = 0; u < kTcPrefetch; ++u) {
                const int it = it0 + u;
                if (it >= ngroups || !ok) break;
                const int s = it % kTcStages, j = it / kTcStages;
                const uint4 pk = pkb[u];
                const float d = db[u];
                const int nx = it + kTcPrefetch;
                if (valid && nx < ngroups) {
                    pkb[u] = __ldg(reinterpret_cast<const uint4 *>(qrow + nx * 32));
                    db[u] = f16_bits_to_float(__ldg(srow + nx));
                }
                if (it >= kTcStages && !mbar_wait(empty + s, (j - 1) & 1, &g_tc_fault)) {
                    ok = false;
                    break;
                }
                uint8_t *ahi = smem + s * kTcStageBytes, *alo = ahi + kTcATile;
                const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 hi, lo;
                    dequant8(words[c], d, hi, lo);
                    const int chunk = hf * 4 + c;                       // 16-byte chunk = 8 k
                    const int off = r * 128 + ((chunk ^ (r & 7)) << 4); // 128-byte swizzle
                    *reinterpret_cast<uint4 *>(ahi + off) = hi;
                    *reinterpret_cast<uint4 *>(alo + off) = lo;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(full_a + s);
            }
        }
    } else if (warp == kTcTmaWarp) {
        if (lane == 0) {
            pdl_wait_primary();  // x follows stream order
            for (int it = 0; it < ngroups; ++it) {
                const int s = it % kTcStages, j = it / kTcStages;
                if (it >= kTcStages && !mbar_wait(empty + s, (j - 1) & 1, &g_tc_fault)) break;
                mbar_arrive_expect_tx(full_b + s, (unsigned)(BM * kTcBK * 2));
                tma_load_2d(smem + s * kTcStageBytes + 2 * kTcATile, &tmap_x, it * kTcBK, m0, full_b + s);
            }
        }
    } else {
        // MMA issue: the whole warp runs the loop (uniform operands), one
        // elected lane issues.  instruction descriptor: f32 accumulate, bf16
        // A and B, both K-major, N = BM, M = 128
        const uint32_t idesc =
            (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BM >> 3) << 17) | ((uint32_t)(kTcBN >> 4) << 24);
        for (int it = 0; it < ngroups; ++it) {
            const int s = it % kTcStages, j = it / kTcStages;
            if (!mbar_wait_warp(full_a + s, j & 1, &g_tc_fault) || !mbar_wait_warp(full_b + s, j & 1, &g_tc_fault)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint8_t *st = smem + s * kTcStageBytes;
            const uint64_t ahi = umma_desc_sw128(st), alo = umma_desc_sw128(st + kTcATile),
                           bd = umma_desc_sw128(st + 2 * kTcATile);
            if (elect_one()) {
                // advancing 16 k (32 bytes) inside the swizzle atom: +2 in 16-byte units
                if (it == 0)
                    umma_bf16<false>(tmem_d, ahi, bd, idesc);
                else
                    umma_bf16<true>(tmem_d, ahi, bd, idesc);
                umma_bf16<true>(tmem_d, alo, bd, idesc);
#pragma unroll
                for (int kk = 1; kk < kTcBK / 16; ++kk) {
                    umma_bf16<true>(tmem_d, ahi + 2 * kk, bd + 2 * kk, idesc);
                    umma_bf16<true>(tmem_d, alo + 2 * kk, bd + 2 * kk, idesc);
                }
                umma_commit(empty + s);
            }
            __syncwarp();
        }
        // also after a failed wait: `done` then tells that every MMA issued
        // has completed, before tensor memory is released
        if (elect_one()) umma_commit(done);
        __syncwarp();
        mbar_wait_warp(done, 0, &g_tc_fault);
    }

    // ---- epilogue: TMEM -> y (warps 0-7: lane quarter warp%4, column half warp/4) ----
    if (warp < kTcProdWarps) {
        const bool got = mbar_wait_warp(done, 0, &g_tc_fault) && ok;
        tc_fence_after();
        pdl_wait_primary();  // y may still be read by an earlier kernel
        const int quarter = warp & 3, half = warp >> 2;
        const int n = n0 + quarter * 32 + lane;
        const int cols = BM / 2;
        for (int c0 = 0; c0 < cols; c0 += 32) {
            const int col = half * cols + c0;
            uint32_t v[32];
            const uint32_t taddr = tmem_d + ((uint32_t)(quarter * 32) << 16) + (uint32_t)col;
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                  "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                  "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                : "r"(taddr));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            if (got && n < N) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int m = m0 + col + i;
                    if (m < M) y[(size_t)m * N + n] = __uint_as_float(v[i]);
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_d, 256);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

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
    // a multiple of 64 keeps each epilogue warp's column range a multiple of
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
    if (cudaFuncSetAttribute(k_i4_tc_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    dim3 grid((N + kTcBN - 1) / kTcBN, (M + BM - 1) / BM);
    cudaError_t e = launch_pdl(k_i4_tc_gemm, grid, dim3(kTcThreads), kTcSmemBytes, st, map, q, scales, y, M, N, K,
                               BM);
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
