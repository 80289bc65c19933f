// glue.cu -- the normalisation step between consecutive projections of a
// layer stack: out = bf16_rne(v / sqrt(mean(v^2) + eps)), v = a (+ b), fp32.
//
// A row is spread over a cluster of kNormCluster CTAs, which keep their part
// of v in registers: each CTA sums its squares (thread, then warp and CTA
// trees), the cluster adds the kNormCluster partial sums in rank order
// through distributed shared memory (every CTA the same way, so the result
// does not depend on timing), and each CTA scales and rounds its part.
// Rows too long for the registers take the one-CTA kernel, which reads the
// row twice.
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

constexpr int kNormCluster = 8;
constexpr int kNormCThreads = 256;
constexpr int kNormPer = 8;  // float4 of v per thread at most
constexpr int kNormMaxD = 4 * kNormPer * kNormCThreads * kNormCluster;

// Store a float into rank `rank`'s shared memory, at the address `local`
// has in this CTA.
__device__ __forceinline__ void norm_st_peer(float *local, unsigned rank, float v)
{
    unsigned ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"((unsigned)__cvta_generic_to_shared(local)),
                 "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

__device__ __forceinline__ void norm_cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// grid (kNormCluster, M), cluster (kNormCluster, 1, 1): CTA q of a row takes
// its float4 range [q n4 / C, (q+1) n4 / C)
__global__ void __launch_bounds__(kNormCThreads) k_rmsnorm_bf16_cl(const float *__restrict__ a,
                                                                   const float *__restrict__ b, int D, float eps,
                                                                   uint16_t *__restrict__ out)
{
    __shared__ float red[kNormCThreads / 32];
    __shared__ float recv[kNormCluster];  // every CTA's partial sum of squares, pushed by its owner
    pdl_launch_dependents();
    pdl_wait_primary();
    const unsigned q = blockIdx.x;
    const int64_t row = blockIdx.y;
    const int n4 = D / 4, lo = (int)((int64_t)q * n4 / kNormCluster), hi = (int)((int64_t)(q + 1) * n4 / kNormCluster);
    const float4 *a4 = reinterpret_cast<const float4 *>(a + row * D);
    const float4 *b4 = b ? reinterpret_cast<const float4 *>(b + row * D) : nullptr;
    float4 v[kNormPer];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
        const int i = lo + (int)threadIdx.x + j * kNormCThreads;
        v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < hi) {
            v[j] = a4[i];
            if (b4) {
                const float4 w = b4[i];
                v[j].x += w.x; v[j].y += w.y; v[j].z += w.z; v[j].w += w.w;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
        ss = fmaf(v[j].x, v[j].x, ss);
        ss = fmaf(v[j].y, v[j].y, ss);
        ss = fmaf(v[j].z, v[j].z, ss);
        ss = fmaf(v[j].w, v[j].w, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < kNormCThreads / 32 ? red[threadIdx.x] : 0.f;
        t = warp_sum(t);
        // this CTA's partial sum (in every lane after the butterfly sum) goes
        // into recv[q] of every CTA of the row, one lane per destination
        if (threadIdx.x < kNormCluster) norm_st_peer(&recv[q], threadIdx.x, t);
    }
    norm_cluster_sync();  // every partial sum has arrived (release / acquire)
    float tot = 0.f;
#pragma unroll
    for (int r = 0; r < kNormCluster; ++r) tot += recv[r];  // rank order
    const float inv = 1.0f / sqrtf(tot / (float)D + eps);
    uint2 *o = reinterpret_cast<uint2 *>(out + row * D);
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
        const int i = lo + (int)threadIdx.x + j * kNormCThreads;
        if (i < hi) {
            const uint32_t l = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[j].x * inv)) |
                               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[j].y * inv)) << 16);
            const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[j].z * inv)) |
                               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[j].w * inv)) << 16);
            o[i] = make_uint2(l, h);
        }
    }
    // nothing reads another CTA's shared memory after the barrier: no second one
}

lowbit_status rmsnorm_launch(const float *a, const float *b, int M, int D, float eps, uint16_t *out,
                             cudaStream_t st)
{
    if (D > kNormMaxD || M > 65535) {
        cudaError_t e = launch_pdl(k_rmsnorm_bf16, dim3(M), dim3(kNormThreads), 0, st, a, b, D, eps, out);
        return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kNormCluster, M);
    cfg.blockDim = dim3(kNormCThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kNormCluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_rmsnorm_bf16_cl, a, b, D, eps, out);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
