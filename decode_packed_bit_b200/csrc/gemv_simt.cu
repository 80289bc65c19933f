// gemv_simt.cu -- CUDA-core (SIMT) weight-streaming kernels for Q1_0_g128
// and INT4_G64 at any batch M.  These are the general-shape paths; the
// tensor-core paths for the shapes that matter most live in their own files.
//
// Q1_0_g128 ("Bonsai-27B-gguf technical white paper digest", "technical
// architecture highlights"): y[m][n] = sum_g d[n][g] sum_{k in g} s(b) x[m][k].
// INT4_G64 ("acorn-llm 0.11.4", "int4 quantisation quality"): the same with a
// signed 4-bit q in place of s(b) and groups of 64.  As the acorn page notes,
// the grouped kernel must not re-reduce per group: each lane keeps one fp32
// partial per batch row, applies the group scale once per group, and the warp
// reduces once per output at the end.
#include "common.cuh"

namespace lowbit {

// One warp per output row n; each lane consumes 32 consecutive weights (one
// 32-bit word of sign bits, inside one 128-group) per step.
template <int MT>
__global__ void __launch_bounds__(256) k_q1_gemv_simt(const uint32_t *__restrict__ bits,
                                                      const uint16_t *__restrict__ scales,
                                                      const uint16_t *__restrict__ x,
                                                      float *__restrict__ y, int M, int N, int K)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    pdl_wait_primary();
    if (n >= N) return;
    const int words = K / 32;
    const uint32_t *wrow = bits + (int64_t)n * words;
    const uint16_t *srow = scales + (int64_t)n * (K / 128);
    for (int m0 = 0; m0 < M; m0 += MT) {
        float acc[MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) acc[j] = 0.f;
        for (int w = lane; w < words; w += 32) {
            const uint32_t b = __ldg(wrow + w);
            const float d = f16_bits_to_float(__ldg(srow + (w >> 2)));
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                if (m0 + j >= M) break;
                const uint4 *xp = reinterpret_cast<const uint4 *>(x + (int64_t)(m0 + j) * K + 32 * w);
                float part = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = __ldg(xp + q);
                    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int kk = 8 * q + 2 * h;
                        // sign bit of weight kk moved onto bit 31 of the fp32
                        const uint32_t s0 = ((~b >> kk) & 1u) << 31;
                        const uint32_t s1 = ((~b >> (kk + 1)) & 1u) << 31;
                        part += __uint_as_float((vv[h] << 16) ^ s0);
                        part += __uint_as_float((vv[h] & 0xFFFF0000u) ^ s1);
                    }
                }
                acc[j] = fmaf(d, part, acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            if (m0 + j >= M) break;
            const float s = warp_sum(acc[j]);
            if (lane == 0) y[(int64_t)(m0 + j) * N + n] = s;
        }
    }
}

// One warp per output row; each lane consumes 8 nibbles (one 32-bit word)
// per step, always inside one 64-group.
template <int MT>
__global__ void __launch_bounds__(256) k_int4_gemv_simt(const uint32_t *__restrict__ q,
                                                        const uint16_t *__restrict__ scales,
                                                        const uint16_t *__restrict__ x,
                                                        float *__restrict__ y, int M, int N, int K)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    pdl_wait_primary();
    if (n >= N) return;
    const int words = K / 8;
    const uint32_t *wrow = q + (int64_t)n * words;
    const uint16_t *srow = scales + (int64_t)n * (K / 64);
    for (int m0 = 0; m0 < M; m0 += MT) {
        float acc[MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) acc[j] = 0.f;
        for (int w = lane; w < words; w += 32) {
            const uint32_t b = __ldg(wrow + w);
            const float d = f16_bits_to_float(__ldg(srow + (w >> 3)));
            float wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) wv[i] = (float)(((int32_t)(b << (28 - 4 * i))) >> 28);
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                if (m0 + j >= M) break;
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)(m0 + j) * K + 8 * w));
                const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
                float part = 0.f;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    part = fmaf(wv[2 * h], __uint_as_float(vv[h] << 16), part);
                    part = fmaf(wv[2 * h + 1], __uint_as_float(vv[h] & 0xFFFF0000u), part);
                }
                acc[j] = fmaf(d, part, acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            if (m0 + j >= M) break;
            const float s = warp_sum(acc[j]);
            if (lane == 0) y[(int64_t)(m0 + j) * N + n] = s;
        }
    }
}

lowbit_status q1_gemv_simt_launch(const uint8_t *bits, const uint16_t *scales, const uint16_t *x,
                                  float *y, int M, int N, int K, cudaStream_t st)
{
    dim3 grid((N + 7) / 8), block(256);
    cudaError_t e = launch_pdl(k_q1_gemv_simt<4>, grid, block, 0, st,
                               reinterpret_cast<const uint32_t *>(bits), scales, x, y, M, N, K);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status int4_gemv_simt_launch(const uint8_t *q, const uint16_t *scales, const uint16_t *x,
                                    float *y, int M, int N, int K, cudaStream_t st)
{
    dim3 grid((N + 7) / 8), block(256);
    cudaError_t e = launch_pdl(k_int4_gemv_simt<4>, grid, block, 0, st,
                               reinterpret_cast<const uint32_t *>(q), scales, x, y, M, N, K);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
