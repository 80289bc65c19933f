// q1_noalloc.cu -- lowbit_q1g128_gemv_noalloc: the Q1_0_g128 product for
// callers that cannot allocate device memory.
//
// lowbit_q1g128_gemv needs scratch for the prepared activation and expects
// the caller to provide it.  Some callers cannot: a plugin running under a
// host framework that owns every device allocation, a real-time or embedded
// deployment that reserves all device memory up front, or code that must not
// call cudaMalloc at the point where the product runs.  This entry point
// keeps that scratch in a fixed array in the library's own device memory
// instead (kNoAllocScratchBytes, allocated when the library is loaded on a
// device and held until the process exits) and allocates nothing itself.
#include <mutex>

#include "common.cuh"

namespace lowbit {
size_t q1m1_act_bytes(int K);
bool q1m1_shape_supported(int R, int N, int K);
lowbit_status q1m1_prepare_launch(const uint16_t *, int, void *, cudaStream_t);
lowbit_status q1m1_gemv_launch(const uint8_t *const *, const uint16_t *const *, const void *, float *const *,
                               int, int, int, cudaStream_t);
lowbit_status q1_gemv_simt_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int,
                                  cudaStream_t);
bool q1sm_supported(int M, int N, int K);
lowbit_status q1sm_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int, cudaStream_t);
}  // namespace lowbit

using namespace lowbit;

// 512 KiB: the prepared activation of one vector with K up to 32768.
constexpr size_t kNoAllocScratchBytes = 512u * 1024u;
constexpr int kNoAllocMaxK = 32768;

static __device__ __align__(256) uint8_t g_q1_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on each device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current, and cached here.
constexpr int kNoAllocMaxDevices = 64;
static void *g_scratch_addr[kNoAllocMaxDevices];
static std::mutex g_scratch_mu;

static lowbit_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return LOWBIT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_q1_noalloc_scratch) != cudaSuccess || p == nullptr) return LOWBIT_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LOWBIT_OK;
}

extern "C" lowbit_status lowbit_q1g128_gemv_noalloc(const uint8_t *w_bits, const uint16_t *w_scales,
                                                    const uint16_t *x, float *y, int M, int N, int K,
                                                    void *stream)
{
    if (M < 1 || M > 16 || N < 1 || K < 1) return LOWBIT_ERR_INVALID_ARG;
    if (K % 128 != 0 || (int64_t)N * K >= (int64_t(1) << 40)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    if (!w_bits || !w_scales || !x || !y) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned16(w_bits) || !aligned16(w_scales) || !aligned16(x) || !aligned16(y)) return LOWBIT_ERR_MISALIGNED;
    cudaStream_t st = as_stream(stream);
    // Only the M = 1 tensor-core path needs scratch; the others read x directly.
    if (M >= 2 && q1sm_supported(M, N, K)) return q1sm_launch(w_bits, w_scales, x, y, M, N, K, st);
    if (M != 1 || !q1m1_shape_supported(1, N, K)) return q1_gemv_simt_launch(w_bits, w_scales, x, y, M, N, K, st);
    if (K > kNoAllocMaxK || q1m1_act_bytes(K) > kNoAllocScratchBytes) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    void *scratch = nullptr;
    lowbit_status s = scratch_for_current_device(&scratch);
    if (s != LOWBIT_OK) return s;
    // The prepare kernel overwrites every byte of the scratch that the product
    // reads, so nothing has to start at zero.
    s = q1m1_prepare_launch(x, K, scratch, st);
    if (s != LOWBIT_OK) return s;
    return q1m1_gemv_launch(&w_bits, &w_scales, scratch, &y, 1, N, K, st);
}
