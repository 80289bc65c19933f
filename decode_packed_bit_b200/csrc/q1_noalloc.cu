// q1_noalloc.cu -- lowbit_q1g128_gemv_noalloc: the Q1_0_g128 product for
// callers that cannot allocate device memory.
//
// lowbit_q1g128_gemv needs scratch for the prepared activation on the shapes
// its persistent kernel takes, and expects the caller to provide it.  Some
// callers cannot: a plugin running under a host framework that owns every
// device allocation, a real-time or embedded deployment that reserves all
// device memory up front, or code that must not call cudaMalloc at the point
// where the product runs.  This entry point keeps that scratch in a fixed
// array in the library's own device memory instead (kNoAllocScratchBytes,
// allocated when the library is loaded on a device and held until the
// process exits) and allocates nothing itself.  The dispatch is the same as
// lowbit_q1g128_gemv's: one-launch shapes need no scratch at all.
#include <mutex>

#include "common.cuh"

namespace lowbit {
size_t q1m1_act_bytes(int K);
bool q1m1_shape_supported(int R, int N, int K);
lowbit_status q1m1_prepare_launch(const uint16_t *, int, void *, cudaStream_t);
lowbit_status q1m1_gemv_launch(const uint8_t *const *, const uint16_t *const *, const void *, float *const *,
                               int, int, int, cudaStream_t);
lowbit_status q1m1_gemv_fused_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int,
                                     cudaStream_t);
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
// with the device current and cached here, together with the id of the
// context it was looked up in: a different current context (the device was
// reset, or a host framework re-created its context) triggers a new lookup.
constexpr int kNoAllocMaxDevices = 64;
struct ScratchSlot {
    void *addr;
    unsigned long long ctx_id;
    bool have_id;
};
static ScratchSlot g_scratch[kNoAllocMaxDevices];
static std::mutex g_scratch_mu;

// The driver's cuCtxGetCurrent / cuCtxGetId, reached through the runtime so
// that the library does not link the driver library directly.  Absent
// entries leave the cache keyed by device alone.
typedef int (*CtxGetCurrentFn)(void **);
typedef int (*CtxGetIdFn)(void *, unsigned long long *);

static bool current_context_id(unsigned long long *id)
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {  // called with g_scratch_mu held
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", reinterpret_cast<void **>(&get_current), cudaEnableDefault,
                                    &q1) != cudaSuccess || q1 != cudaDriverEntryPointSuccess)
            get_current = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", reinterpret_cast<void **>(&get_id), cudaEnableDefault, &q2) !=
                cudaSuccess || q2 != cudaDriverEntryPointSuccess)
            get_id = nullptr;
        resolved = true;
    }
    if (get_current == nullptr || get_id == nullptr) return false;
    void *ctx = nullptr;
    if (get_current(&ctx) != 0 || ctx == nullptr) return false;
    return get_id(ctx, id) == 0;
}

static lowbit_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return LOWBIT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot &slot = g_scratch[dev];
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (slot.addr == nullptr || have_id != slot.have_id || (have_id && id != slot.ctx_id)) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_q1_noalloc_scratch) != cudaSuccess || p == nullptr) return LOWBIT_ERR_CUDA;
        slot.addr = p;
        // the lookup may have created the context: take its id afterwards
        slot.have_id = current_context_id(&slot.ctx_id);
    }
    *out = slot.addr;
    return LOWBIT_OK;
}

extern "C" lowbit_status lowbit_q1g128_gemv_noalloc(const uint8_t *w_bits, const uint16_t *w_scales,
                                                    const uint16_t *x, float *y, int M, int N, int K,
                                                    void *stream)
{
    if (M < 1 || M > 16 || N < 1 || K < 1) return LOWBIT_ERR_INVALID_ARG;
    if (K % 128 != 0 || (int64_t)N * K >= (int64_t(1) << 40)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    // the scratch bound holds for every M = 1 shape, whichever kernel it takes
    if (M == 1 && (K > kNoAllocMaxK || q1m1_act_bytes(K) > kNoAllocScratchBytes))
        return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    if (!w_bits || !w_scales || !x || !y) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned16(w_bits) || !aligned16(w_scales) || !aligned16(x) || !aligned16(y)) return LOWBIT_ERR_MISALIGNED;
    cudaStream_t st = as_stream(stream);
    // Only the M = 1 persistent kernel needs scratch; the others read x directly.
    if (M >= 2 && q1sm_supported(M, N, K)) return q1sm_launch(w_bits, w_scales, x, y, M, N, K, st);
    if (M != 1 || !q1m1_shape_supported(1, N, K)) return q1_gemv_simt_launch(w_bits, w_scales, x, y, M, N, K, st);
    lowbit_status s = q1m1_gemv_fused_launch(w_bits, w_scales, x, y, N, K, st);  // one launch, no scratch
    if (s != LOWBIT_ERR_UNSUPPORTED_SHAPE) return s;
    void *scratch = nullptr;
    s = scratch_for_current_device(&scratch);
    if (s != LOWBIT_OK) return s;
    // The prepare kernel overwrites every byte of the scratch that the product
    // reads, so nothing has to start at zero.
    s = q1m1_prepare_launch(x, K, scratch, st);
    if (s != LOWBIT_OK) return s;
    return q1m1_gemv_launch(&w_bits, &w_scales, scratch, &y, 1, N, K, st);
}
