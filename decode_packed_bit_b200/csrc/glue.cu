// glue.cu -- the normalisation step between consecutive projections of a
// layer stack: out = bf16_rne(v / sqrt(mean(v^2) + eps)), v = a (+ b), fp32.
// One CTA per row; the row is read twice (sum of squares, then scale), which
// costs nothing next to the weight stream of the projections around it.
#include "common.cuh"

namespace lowbit {

constexpr int kNormThreads = 512;

__global__ void __launch_bounds__(kNormThreads) k_rmsnorm_bf16(const float *__restrict__ a,
                                                               const float *__restrict__ b, int D,
                                                               float eps, uint16_t *__restrict__ out)
{
    __shared__ float red[kNormThreads / 32];
    pdl_launch_dependents();
    pdl_wait_primary();
    const int64_t row = blockIdx.x;
    const float4 *a4 = reinterpret_cast<const float4 *>(a + row * D);
    const float4 *b4 = b ? reinterpret_cast<const float4 *>(b + row * D) : nullptr;
    float ss = 0.f;
    for (int i = threadIdx.x; i < D / 4; i += blockDim.x) {
        float4 v = a4[i];
        if (b4) {
            const float4 w = b4[i];
            v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
        }
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < kNormThreads / 32 ? red[threadIdx.x] : 0.f;
        t = warp_sum(t);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] / (float)D + eps);
    uint2 *o = reinterpret_cast<uint2 *>(out + row * D);
    for (int i = threadIdx.x; i < D / 4; i += blockDim.x) {
        float4 v = a4[i];
        if (b4) {
            const float4 w = b4[i];
            v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
        }
        const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x * inv)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y * inv)) << 16);
        const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z * inv)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w * inv)) << 16);
        o[i] = make_uint2(lo, hi);
    }
}

lowbit_status rmsnorm_launch(const float *a, const float *b, int M, int D, float eps, uint16_t *out,
                             cudaStream_t st)
{
    cudaError_t e = launch_pdl(k_rmsnorm_bf16, dim3(M), dim3(kNormThreads), 0, st, a, b, D, eps, out);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
