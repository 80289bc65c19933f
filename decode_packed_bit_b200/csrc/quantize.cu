// quantize.cu -- float weights to the packed formats: Q1_0_g128 signs and
// INT4_G64 codes, with their FP16 group scales, written straight in the
// packed layout the product kernels read.
//
// What is computed:
//   Q1_0_g128 ("Bonsai-27B-gguf technical white paper digest", "technical
//   architecture highlights": one sign bit per weight, one FP16 scale per 128
//   weights): bit = (w >= 0); the group's scale is its mean |w|, the d that
//   minimises sum (w - d * sign)^2.
//   INT4_G64 ("acorn-llm 0.11.4", "int4 quantisation quality: group
//   quantisation": round-to-nearest int4, one scale per group along the input
//   dimension): d = max |w| / 7, q = w / d rounded to nearest (ties to even),
//   clamped to [-8, 7]; q = 0 where d = 0 or w is NaN.
//
// Results are bit-exact with a plain CPU statement of the same steps: every
// step is an IEEE double operation in a fixed order (one thread per group,
// sums with k ascending), and the FP16 rounding is to nearest, ties to even,
// with magnitudes at or above 65504 saturating to 65504.
#include "common.cuh"

#include <cuda_fp16.h>

namespace lowbit {

// FP16 bits of v: nearest, ties to even; |v| >= 65504 -> +-65504; NaN -> 0.
__device__ __forceinline__ uint16_t f16_rne_sat(double v)
{
    if (v != v) return 0;
    const double a = fmin(fabs(v), 65504.0);
    const uint16_t h = __half_as_ushort(__double2half(a));
    return signbit(v) ? (uint16_t)(h | 0x8000u) : h;
}

// One thread per (row, 128-group): 16 bytes of signs (LSB first) and a scale.
__global__ void k_quant_q1(const float *__restrict__ w, int64_t rows, int64_t cols, uint8_t *__restrict__ packed,
                           uint16_t *__restrict__ scales)
{
    const int64_t G = cols / 128;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= rows * G) return;
    const int64_t n = id / G, g = id - n * G;
    const float4 *src = reinterpret_cast<const float4 *>(w + n * cols + g * 128);
    double s = 0.0;
    uint32_t word[4] = {0u, 0u, 0u, 0u};  // word j: k = 32 j .. 32 j + 31 of the group, bit k % 32
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {  // k = 4 i .. 4 i + 3
        const float4 v = src[i];
        s += fabs((double)v.x);
        s += fabs((double)v.y);
        s += fabs((double)v.z);
        s += fabs((double)v.w);
        const uint32_t b = (v.x >= 0.f ? 1u : 0u) | (v.y >= 0.f ? 2u : 0u) | (v.z >= 0.f ? 4u : 0u) |
                           (v.w >= 0.f ? 8u : 0u);
        word[i >> 3] |= b << (4 * (i & 7));
    }
    *reinterpret_cast<uint4 *>(packed + n * (cols / 8) + g * 16) = make_uint4(word[0], word[1], word[2], word[3]);
    scales[id] = f16_rne_sat(s / 128.0);
}

// One thread per (row, 64-group): 32 bytes of nibbles (even k low) and a scale.
__global__ void k_quant_int4(const float *__restrict__ w, int64_t rows, int64_t cols, uint8_t *__restrict__ packed,
                             uint16_t *__restrict__ scales)
{
    const int64_t G = cols / 64;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= rows * G) return;
    const int64_t n = id / G, g = id - n * G;
    const float4 *src = reinterpret_cast<const float4 *>(w + n * cols + g * 64);
    double amax = 0.0;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const float4 v = src[i];
        const double a[4] = {fabs((double)v.x), fabs((double)v.y), fabs((double)v.z), fabs((double)v.w)};
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (a[c] > amax) amax = a[c];
    }
    const uint16_t dh = f16_rne_sat(amax / 7.0);
    scales[id] = dh;
    const double d = (double)__half2float(__ushort_as_half(dh));
    uint32_t word[8];  // word j: k = 8 j .. 8 j + 7 of the group, nibble k % 8
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 v0 = src[2 * j], v1 = src[2 * j + 1];
        const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t acc = 0u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const double v = (double)f[c];
            double q = 0.0;
            if (d > 0.0 && v == v) q = fmin(fmax(rint(v / d), -8.0), 7.0);
            acc |= ((uint32_t)(int)q & 0xFu) << (4 * c);
        }
        word[j] = acc;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(packed + n * (cols / 2) + g * 32);
    dst[0] = make_uint4(word[0], word[1], word[2], word[3]);
    dst[1] = make_uint4(word[4], word[5], word[6], word[7]);
}

lowbit_status quantize_launch(int fmt, const float *w, int64_t rows, int64_t cols, uint8_t *packed, uint16_t *scales,
                              cudaStream_t st)
{
    const int64_t groups = rows * (cols / (fmt == 1 ? 128 : 64));
    if (groups == 0) return LOWBIT_OK;
    const int threads = 128;
    const int64_t blocks = (groups + threads - 1) / threads;
    if (blocks > 0x7FFFFFFF) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    if (fmt == 1)
        k_quant_q1<<<(unsigned)blocks, threads, 0, st>>>(w, rows, cols, packed, scales);
    else
        k_quant_int4<<<(unsigned)blocks, threads, 0, st>>>(w, rows, cols, packed, scales);
    return cudaGetLastError() == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
