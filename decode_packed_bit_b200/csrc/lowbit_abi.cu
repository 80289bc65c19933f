// lowbit_abi.cu -- the extern "C" entry points declared in include/lowbit.h.
// Every argument is validated here, on the host, before anything is enqueued.
#include "common.cuh"

namespace lowbit {
lowbit_status pack_launch(lowbit_format, const int8_t *, int64_t, int64_t, uint8_t *, cudaStream_t);
lowbit_status t3_pack_launch(const int8_t *, int64_t, int64_t, uint8_t *, cudaStream_t);
lowbit_status t3_unpack_launch(const uint8_t *, int64_t, int64_t, int8_t *, cudaStream_t);
bool t3_fast_supported(int R, int N, int K);
lowbit_status t3_group_launch(const uint8_t *const *, const uint16_t *const *, const uint16_t *, float *const *, int,
                              int, int, cudaStream_t);
lowbit_status t3_simt_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int,
                             cudaStream_t);
lowbit_status unpack_launch(lowbit_format, const uint8_t *, int64_t, int64_t, int8_t *, cudaStream_t);
lowbit_status q1_gemv_simt_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int,
                                  int, cudaStream_t);
lowbit_status int4_gemv_simt_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int,
                                    int, cudaStream_t);
lowbit_status q2_mlp_launch(const uint8_t *const *, const int32_t *, int, const int16_t *, int, int16_t *,
                            int32_t *, cudaStream_t);
int q2_weight_bytes_padded(const int32_t *, int);
size_t z80_smem_bytes(const int32_t *dims, int n_layers);
lowbit_status z80_generate_launch(const uint8_t *const *, const int32_t *, int, const uint8_t *, int, int,
                                  const uint8_t *, int, uint8_t *, int32_t *, cudaStream_t);
lowbit_status rmsnorm_launch(const float *, const float *, int, int, float, uint16_t *, cudaStream_t);
size_t q1m1_act_bytes(int K);
bool q1m1_shape_supported(int R, int N, int K);
int q1m1_max_group();
size_t q1m1_xcopy_off(int K);
bool i4m1_supported(int N, int K);
bool i4tc_supported(int M, int N, int K);
lowbit_status i4tc_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int, cudaStream_t);
int i4tc_fault_flag();
lowbit_status i4m1_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, cudaStream_t);
lowbit_status q1m1_prepare_launch(const uint16_t *, int, void *, cudaStream_t);
bool q1sm_supported(int M, int N, int K);
bool i4sm_supported(int M, int N, int K);
lowbit_status i4sm_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int, cudaStream_t);
lowbit_status q1stack_launch(const uint8_t *const *, const uint16_t *const *, int, int, int, uint16_t *, float, void *,
                             uint16_t *, float *, cudaStream_t);
size_t q1stack_workspace_bytes(int F);
int q1stack_fault_flag();
int smg_fault_flag();
lowbit_status q1sm_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int, int, cudaStream_t);
lowbit_status q1m1_gemv_fused_launch(const uint8_t *, const uint16_t *, const uint16_t *, float *, int, int,
                                     cudaStream_t);
bool q1m1_fused_supported(int N, int K);
lowbit_status quantize_launch(int fmt, const float *w, int64_t rows, int64_t cols, uint8_t *packed, uint16_t *scales,
                              cudaStream_t st);
bool smg_supported(int fmt, int R, int M, int N, int K);
lowbit_status smr_launch(int fmt, const uint8_t *const *, const uint16_t *const *, const uint16_t *, float *const *,
                         int R, int M, int N, int K, cudaStream_t);
lowbit_status smg_launch(int fmt, const uint8_t *const *, const uint16_t *const *, const uint16_t *, float *const *,
                         int R, int M, int N, int K, cudaStream_t);
bool i4m1_group_supported(int R, int N, int K);
lowbit_status i4m1_group_launch(const uint8_t *const *, const uint16_t *const *, const uint16_t *, float *const *,
                                int, int, int, cudaStream_t);
lowbit_status q1m1_gemv_x_group_launch(const uint8_t *const *, const uint16_t *const *, const uint16_t *,
                                       float *const *, int, int, int, int, cudaStream_t);
bool q1m1_x_group_supported(int R, int M, int N, int K);
lowbit_status q1m1_gemv_launch(const uint8_t *const *, const uint16_t *const *, const void *, float *const *,
                               int, int, int, cudaStream_t);

constexpr int64_t kMaxElems = int64_t(1) << 40;
constexpr int kQ1MaxM = 16;
// INT4_G64 single calls with 2 <= M <= this take the mma.sync small-batch
// kernel; larger M (from 16 up, where the tensor-core GEMM applies) the
// tcgen05 GEMM.
#ifndef LOWBIT_I4_SMALLM_MAX
#define LOWBIT_I4_SMALLM_MAX 32
#endif
constexpr int kI4SmallMMax = LOWBIT_I4_SMALLM_MAX;
}  // namespace lowbit

using namespace lowbit;

#define LB_CHECK(cond, code) \
    do {                     \
        if (!(cond)) return (code); \
    } while (0)

static int per_byte(lowbit_format f)
{
    switch (f) {
    case LOWBIT_FMT_Q1_G128: return 8;
    case LOWBIT_FMT_Q2: return 4;
    case LOWBIT_FMT_INT4_G64: return 2;
    case LOWBIT_FMT_TERNARY_G128: return -1;  // 26 bytes per 128 columns
    default: return 0;
    }
}

extern "C" {

const char *lowbit_status_string(lowbit_status s)
{
    switch (s) {
    case LOWBIT_OK: return "ok";
    case LOWBIT_ERR_INVALID_ARG: return "invalid argument";
    case LOWBIT_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case LOWBIT_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case LOWBIT_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
    }
}

int lowbit_version(void) { return 100; }

int lowbit_fault_flags(void)
{
    const int f4 = i4tc_fault_flag(), fs = q1stack_fault_flag(), fg = smg_fault_flag();
    if (f4 < 0 || fs < 0 || fg < 0) return -1;
    return (f4 ? 1 : 0) | (fs ? 4 : 0) | (fg ? 8 : 0);
}

lowbit_status lowbit_pack(lowbit_format fmt, const int8_t *codes, int64_t rows, int64_t cols,
                          uint8_t *packed, void *stream)
{
    const int per = per_byte(fmt);
    LB_CHECK(per != 0, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(rows >= 0 && cols >= 0 && rows * cols < kMaxElems, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(cols % (per > 0 ? per : 128) == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    if (rows == 0 || cols == 0) return LOWBIT_OK;
    LB_CHECK(codes != nullptr && packed != nullptr, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(codes) && aligned16(packed), LOWBIT_ERR_MISALIGNED);
    if (per < 0) return t3_pack_launch(codes, rows, cols, packed, as_stream(stream));
    return pack_launch(fmt, codes, rows, cols, packed, as_stream(stream));
}

lowbit_status lowbit_quantize(lowbit_format fmt, const float *w, int64_t rows, int64_t cols, uint8_t *packed,
                              uint16_t *scales, void *stream)
{
    LB_CHECK(fmt == LOWBIT_FMT_Q1_G128 || fmt == LOWBIT_FMT_INT4_G64 || fmt == LOWBIT_FMT_Q2 ||
                 fmt == LOWBIT_FMT_TERNARY_G128,
             LOWBIT_ERR_INVALID_ARG);
    // the pages give no rule for 2-bit or ternary codes
    LB_CHECK(fmt != LOWBIT_FMT_Q2 && fmt != LOWBIT_FMT_TERNARY_G128, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(rows >= 0 && cols >= 0 && rows * cols < kMaxElems, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(cols % (fmt == LOWBIT_FMT_Q1_G128 ? 128 : 64) == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    if (rows == 0 || cols == 0) return LOWBIT_OK;
    LB_CHECK(w != nullptr && packed != nullptr && scales != nullptr, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(w) && aligned16(packed) && aligned16(scales), LOWBIT_ERR_MISALIGNED);
    return quantize_launch(fmt == LOWBIT_FMT_Q1_G128 ? 1 : 3, w, rows, cols, packed, scales, as_stream(stream));
}

lowbit_status lowbit_unpack(lowbit_format fmt, const uint8_t *packed, int64_t rows, int64_t cols,
                            int8_t *codes, void *stream)
{
    const int per = per_byte(fmt);
    LB_CHECK(per != 0, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(rows >= 0 && cols >= 0 && rows * cols < kMaxElems, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(cols % (per > 0 ? per : 128) == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    if (rows == 0 || cols == 0) return LOWBIT_OK;
    LB_CHECK(codes != nullptr && packed != nullptr, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(codes) && aligned16(packed), LOWBIT_ERR_MISALIGNED);
    if (per < 0) return t3_unpack_launch(packed, rows, cols, codes, as_stream(stream));
    return unpack_launch(fmt, packed, rows, cols, codes, as_stream(stream));
}

// ---------------------------------------------------------------------------
// Q1_0_g128
// ---------------------------------------------------------------------------

static lowbit_status q1_shape_ok(int M, int N, int K)
{
    LB_CHECK(M >= 1 && M <= kQ1MaxM && N >= 1 && K >= 1, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(K % 128 == 0 && (int64_t)N * K < kMaxElems, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    return LOWBIT_OK;
}

static size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

size_t lowbit_q1g128_act_bytes(int M, int K)
{
    if (M < 1 || M > kQ1MaxM || K < 128 || K % 128 != 0) return 0;
    if (M == 1) return q1m1_act_bytes(K);
    return al256((size_t)M * (size_t)K * 2u);
}

// M = 1 runs on the tensor-core kernel when the shape allows (K/128 even and
// the activation slices fit in shared memory); otherwise, and for M >= 2, the
// SIMT kernel reads a bf16 copy of x (kept in the prepared buffer at M = 1).
static bool q1_tc_path(int R, int M, int N, int K) { return M == 1 && q1m1_shape_supported(R, N, K); }

static const uint16_t *q1_simt_x(const void *act, int M, int K)
{
    const uint8_t *a = static_cast<const uint8_t *>(act);
    return reinterpret_cast<const uint16_t *>(M == 1 ? a + q1m1_xcopy_off(K) : a);
}

size_t lowbit_q1g128_act_workspace_bytes(int R, int M, int N, int K)
{
    (void)R; (void)M; (void)N; (void)K;
    return 0;  // the split-K partial sums stay in thread-block-cluster shared memory
}

size_t lowbit_q1g128_workspace_bytes(int M, int N, int K)
{
    if (M < 1 || M > kQ1MaxM || N < 1 || K < 128 || K % 128 != 0) return 0;
    if (!q1_tc_path(1, M, N, K)) return 0;
    if (q1m1_fused_supported(N, K)) return 0;  // one launch builds the activation in shared memory
    return al256(q1m1_act_bytes(K));           // the persistent kernel reads a prepared activation
}

lowbit_status lowbit_q1g128_gemv(const uint8_t *w_bits, const uint16_t *w_scales, const uint16_t *x,
                                 float *y, int M, int N, int K, void *workspace, size_t workspace_bytes,
                                 void *stream)
{
    lowbit_status s = q1_shape_ok(M, N, K);
    if (s != LOWBIT_OK) return s;
    LB_CHECK(w_bits && w_scales && x && y, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(w_bits) && aligned16(w_scales) && aligned16(x) && aligned16(y), LOWBIT_ERR_MISALIGNED);
    const size_t need = lowbit_q1g128_workspace_bytes(M, N, K);
    LB_CHECK(workspace_bytes >= need && (need == 0 || workspace != nullptr), LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(workspace == nullptr || aligned16(workspace), LOWBIT_ERR_MISALIGNED);
    cudaStream_t st = as_stream(stream);
    if (q1_tc_path(1, M, N, K)) {
        s = q1m1_gemv_fused_launch(w_bits, w_scales, x, y, N, K, st);  // one launch when the shape allows
        if (s != LOWBIT_ERR_UNSUPPORTED_SHAPE) return s;
        uint8_t *act = static_cast<uint8_t *>(workspace);
        s = q1m1_prepare_launch(x, K, act, st);
        if (s != LOWBIT_OK) return s;
        return q1m1_gemv_launch(&w_bits, &w_scales, act, &y, 1, N, K, st);
    }
    if (M >= 2 && q1sm_supported(M, N, K)) return q1sm_launch(w_bits, w_scales, x, y, M, N, K, st);
    return q1_gemv_simt_launch(w_bits, w_scales, x, y, M, N, K, st);
}

lowbit_status lowbit_q1g128_prepare_act(const uint16_t *x, int M, int K, void *act, size_t act_bytes,
                                        void *stream)
{
    LB_CHECK(M >= 1 && M <= kQ1MaxM && K >= 1, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(K % 128 == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(x && act, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(x) && aligned16(act), LOWBIT_ERR_MISALIGNED);
    const size_t need = lowbit_q1g128_act_bytes(M, K);
    LB_CHECK(act_bytes >= need, LOWBIT_ERR_INVALID_ARG);
    cudaStream_t st = as_stream(stream);
    if (M == 1) return q1m1_prepare_launch(x, K, act, st);
    return cudaMemcpyAsync(act, x, (size_t)M * K * 2u, cudaMemcpyDeviceToDevice, st) == cudaSuccess
               ? LOWBIT_OK
               : LOWBIT_ERR_CUDA;
}

lowbit_status lowbit_q1g128_gemv_act_group(const uint8_t *const *w_bits, const uint16_t *const *w_scales,
                                           const void *act, float *const *y, int R, int M, int N, int K,
                                           void *workspace, size_t workspace_bytes, void *stream)
{
    LB_CHECK(R >= 1 && R <= q1m1_max_group() && w_bits && w_scales && y, LOWBIT_ERR_INVALID_ARG);
    lowbit_status s = q1_shape_ok(M, N, K);
    if (s != LOWBIT_OK) return s;
    LB_CHECK(act != nullptr, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(act), LOWBIT_ERR_MISALIGNED);
    for (int r = 0; r < R; ++r) {
        LB_CHECK(w_bits[r] && w_scales[r] && y[r], LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_bits[r]) && aligned16(w_scales[r]) && aligned16(y[r]), LOWBIT_ERR_MISALIGNED);
    }
    const size_t need = lowbit_q1g128_act_workspace_bytes(R, M, N, K);
    LB_CHECK(workspace_bytes >= need && (need == 0 || workspace != nullptr), LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(workspace == nullptr || aligned16(workspace), LOWBIT_ERR_MISALIGNED);
    cudaStream_t st = as_stream(stream);
    if (q1_tc_path(R, M, N, K)) return q1m1_gemv_launch(w_bits, w_scales, act, y, R, N, K, st);
    const bool sm = M >= 2 && q1sm_supported(M, N, K);
    for (int r = 0; r < R; ++r) {
        const uint16_t *xr = q1_simt_x(act, M, K);
        s = sm ? q1sm_launch(w_bits[r], w_scales[r], xr, y[r], M, N, K, st)
               : q1_gemv_simt_launch(w_bits[r], w_scales[r], xr, y[r], M, N, K, st);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

size_t lowbit_q1g128_group_workspace_bytes(int R, int M, int N, int K)
{
    if (R < 1 || q1_shape_ok(M, N, K) != LOWBIT_OK) return 0;
    if (q1m1_x_group_supported(R, M, N, K)) return 0;
    if (M >= 2 && (smg_supported(1, R, M, N, K) || q1sm_supported(M, N, K))) return 0;
    return al256(lowbit_q1g128_act_bytes(M, K)) + lowbit_q1g128_act_workspace_bytes(R, M, N, K);
}

lowbit_status lowbit_q1g128_gemv_group(const uint8_t *const *w_bits, const uint16_t *const *w_scales,
                                       const uint16_t *x, float *const *y, int R, int M, int N, int K,
                                       void *workspace, size_t workspace_bytes, void *stream)
{
    LB_CHECK(R >= 1 && R <= q1m1_max_group() && w_bits && w_scales && y && x, LOWBIT_ERR_INVALID_ARG);
    lowbit_status s = q1_shape_ok(M, N, K);
    if (s != LOWBIT_OK) return s;
    LB_CHECK(aligned16(x), LOWBIT_ERR_MISALIGNED);
    for (int r = 0; r < R; ++r) {
        LB_CHECK(w_bits[r] && w_scales[r] && y[r], LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_bits[r]) && aligned16(w_scales[r]) && aligned16(y[r]), LOWBIT_ERR_MISALIGNED);
    }
    const size_t need = lowbit_q1g128_group_workspace_bytes(R, M, N, K);
    LB_CHECK(workspace_bytes >= need && (need == 0 || workspace != nullptr), LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(workspace == nullptr || aligned16(workspace), LOWBIT_ERR_MISALIGNED);
    cudaStream_t st = as_stream(stream);
    s = q1m1_gemv_x_group_launch(w_bits, w_scales, x, y, R, M, N, K, st);  // M <= 4: integer bit planes
    if (s != LOWBIT_ERR_UNSUPPORTED_SHAPE) return s;
    if (M >= 2 && smg_supported(1, R, M, N, K)) return smg_launch(1, w_bits, w_scales, x, y, R, M, N, K, st);
    // too few row blocks for the persistent kernel: up to 8 matrices per split-K launch
    if (M >= 2 && q1sm_supported(M, N, K)) return smr_launch(1, w_bits, w_scales, x, y, R, M, N, K, st);
    uint8_t *act = static_cast<uint8_t *>(workspace);
    const size_t act_bytes = al256(lowbit_q1g128_act_bytes(M, K));
    s = lowbit_q1g128_prepare_act(x, M, K, act, act_bytes, stream);
    if (s != LOWBIT_OK) return s;
    return lowbit_q1g128_gemv_act_group(w_bits, w_scales, act, y, R, M, N, K, act + act_bytes,
                                        workspace_bytes - act_bytes, stream);
}

lowbit_status lowbit_q1g128_gemv_act(const uint8_t *w_bits, const uint16_t *w_scales, const void *act,
                                     float *y, int M, int N, int K, void *workspace, size_t workspace_bytes,
                                     void *stream)
{
    return lowbit_q1g128_gemv_act_group(&w_bits, &w_scales, act, &y, 1, M, N, K, workspace, workspace_bytes,
                                        stream);
}

size_t lowbit_q1g128_stack_workspace_bytes(int n_layers, int hidden, int ffn)
{
    if (n_layers < 1 || hidden < 1 || ffn < 1) return 0;
    return al256(q1stack_workspace_bytes(ffn));
}

lowbit_status lowbit_q1g128_stack_step(const uint8_t *const *w_bits, const uint16_t *const *w_scales, int n_layers,
                                       int hidden, int ffn, uint16_t *x, float eps, void *workspace,
                                       size_t workspace_bytes, uint16_t *record_inputs, float *record_outputs,
                                       void *stream)
{
    LB_CHECK(w_bits && w_scales && x && workspace, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(n_layers >= 1 && n_layers <= 73 && hidden >= 1 && ffn >= hidden && eps >= 0.f, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(hidden % 512 == 0 && ffn % 512 == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(workspace_bytes >= lowbit_q1g128_stack_workspace_bytes(n_layers, hidden, ffn), LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(x) && aligned16(workspace), LOWBIT_ERR_MISALIGNED);
    LB_CHECK(record_inputs == nullptr || aligned16(record_inputs), LOWBIT_ERR_MISALIGNED);
    LB_CHECK(record_outputs == nullptr || aligned16(record_outputs), LOWBIT_ERR_MISALIGNED);
    for (int i = 0; i < 7 * n_layers; ++i) {
        LB_CHECK(w_bits[i] && w_scales[i], LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_bits[i]) && aligned16(w_scales[i]), LOWBIT_ERR_MISALIGNED);
    }
    return q1stack_launch(w_bits, w_scales, n_layers, hidden, ffn, x, eps, workspace, record_inputs, record_outputs,
                          as_stream(stream));
}

// ---------------------------------------------------------------------------
// INT4_G64
// ---------------------------------------------------------------------------

lowbit_status lowbit_int4g64_gemm(const uint8_t *w_q, const uint16_t *w_scales, const uint16_t *x, float *y,
                                  int M, int N, int K, void *stream)
{
    LB_CHECK(M >= 1 && N >= 1 && K >= 1, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(K % 64 == 0 && (int64_t)N * K < kMaxElems && (int64_t)M * K < kMaxElems,
             LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(w_q && w_scales && x && y, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(w_q) && aligned16(w_scales) && aligned16(x) && aligned16(y), LOWBIT_ERR_MISALIGNED);
    cudaStream_t st = as_stream(stream);
    if (M == 1 && i4m1_supported(N, K)) return i4m1_launch(w_q, w_scales, x, y, N, K, st);
    if (M >= 2 && M <= kI4SmallMMax && i4sm_supported(M, N, K)) return i4sm_launch(w_q, w_scales, x, y, M, N, K, st);
    if (i4tc_supported(M, N, K)) return i4tc_launch(w_q, w_scales, x, y, M, N, K, st);
    return int4_gemv_simt_launch(w_q, w_scales, x, y, M, N, K, st);
}

lowbit_status lowbit_int4g64_gemm_group(const uint8_t *const *w_q, const uint16_t *const *w_scales,
                                        const uint16_t *x, float *const *y, int R, int M, int N, int K,
                                        void *stream)
{
    LB_CHECK(R >= 1 && R <= 256 && w_q && w_scales && y && x, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(M >= 1 && N >= 1 && K >= 1, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(K % 64 == 0 && (int64_t)N * K < kMaxElems && (int64_t)M * K < kMaxElems,
             LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(aligned16(x), LOWBIT_ERR_MISALIGNED);
    for (int r = 0; r < R; ++r) {
        LB_CHECK(w_q[r] && w_scales[r] && y[r], LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_q[r]) && aligned16(w_scales[r]) && aligned16(y[r]), LOWBIT_ERR_MISALIGNED);
    }
    cudaStream_t st = as_stream(stream);
    if (M == 1 && i4m1_group_supported(R, N, K)) return i4m1_group_launch(w_q, w_scales, x, y, R, N, K, st);
    if (M >= 2 && smg_supported(3, R, M, N, K)) return smg_launch(3, w_q, w_scales, x, y, R, M, N, K, st);
    if (M >= 2 && M <= kI4SmallMMax && i4sm_supported(M, N, K))
        return smr_launch(3, w_q, w_scales, x, y, R, M, N, K, st);
    for (int r = 0; r < R; ++r) {
        const lowbit_status s = lowbit_int4g64_gemm(w_q[r], w_scales[r], x, y[r], M, N, K, stream);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

// ---------------------------------------------------------------------------
// ternary, FP16 scale per 128
// ---------------------------------------------------------------------------

static lowbit_status t3_shape_ok(int M, int N, int K)
{
    LB_CHECK(M >= 1 && M <= 16 && N >= 1 && K >= 1, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(K % 128 == 0 && (int64_t)N * K < kMaxElems, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    return LOWBIT_OK;
}

lowbit_status lowbit_t3g128_gemv_group(const uint8_t *const *w, const uint16_t *const *w_scales, const uint16_t *x,
                                       float *const *y, int R, int M, int N, int K, void *stream)
{
    LB_CHECK(R >= 1 && R <= 256 && w && w_scales && y && x, LOWBIT_ERR_INVALID_ARG);
    lowbit_status s = t3_shape_ok(M, N, K);
    if (s != LOWBIT_OK) return s;
    LB_CHECK(aligned16(x), LOWBIT_ERR_MISALIGNED);
    for (int r = 0; r < R; ++r) {
        LB_CHECK(w[r] && w_scales[r] && y[r], LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w[r]) && aligned16(w_scales[r]) && aligned16(y[r]), LOWBIT_ERR_MISALIGNED);
    }
    cudaStream_t st = as_stream(stream);
    if (M == 1 && t3_fast_supported(R, N, K)) return t3_group_launch(w, w_scales, x, y, R, N, K, st);
    for (int r = 0; r < R; ++r) {
        s = t3_simt_launch(w[r], w_scales[r], x, y[r], M, N, K, st);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

lowbit_status lowbit_t3g128_gemv(const uint8_t *w, const uint16_t *w_scales, const uint16_t *x, float *y, int M, int N,
                                 int K, void *stream)
{
    return lowbit_t3g128_gemv_group(&w, &w_scales, x, &y, 1, M, N, K, stream);
}

// ---------------------------------------------------------------------------
// Q2 MLP
// ---------------------------------------------------------------------------

lowbit_status lowbit_q2_mlp_forward(const uint8_t *const *w_packed, const int32_t *dims, int n_layers,
                                    const int16_t *x, int batch, int16_t *logits, int32_t *argmax,
                                    void *stream)
{
    LB_CHECK(w_packed && dims && n_layers >= 1 && n_layers <= 8 && batch >= 0, LOWBIT_ERR_INVALID_ARG);
    for (int l = 0; l < n_layers; ++l) {
        LB_CHECK(dims[l] >= 4 && dims[l] <= 1024, LOWBIT_ERR_UNSUPPORTED_SHAPE);
        LB_CHECK(dims[l] % 4 == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
        LB_CHECK(w_packed[l] != nullptr, LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_packed[l]), LOWBIT_ERR_MISALIGNED);
    }
    LB_CHECK(dims[n_layers] >= 1 && dims[n_layers] <= 1024, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(q2_weight_bytes_padded(dims, n_layers) <= 96 * 1024, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    if (batch == 0) return LOWBIT_OK;
    LB_CHECK(x && logits, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(x) && aligned16(logits) && (argmax == nullptr || aligned16(argmax)),
             LOWBIT_ERR_MISALIGNED);
    return q2_mlp_launch(w_packed, dims, n_layers, x, batch, logits, argmax, as_stream(stream));
}

lowbit_status lowbit_z80_generate(const uint8_t *const *w_packed, const int32_t *dims, int n_layers,
                                  const uint8_t *queries, int batch, int qlen, const uint8_t *charset, int max_new,
                                  uint8_t *reply, int32_t *reply_len, void *stream)
{
    LB_CHECK(w_packed && dims && charset && n_layers >= 1 && n_layers <= 8 && batch >= 0, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(qlen >= 1 && qlen <= 4096 && max_new >= 0 && max_new <= 250, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(dims[0] == 256, LOWBIT_ERR_UNSUPPORTED_SHAPE);  // 128 query + 128 context buckets
    for (int l = 0; l < n_layers; ++l) {
        LB_CHECK(dims[l] >= 4 && dims[l] <= 256 && dims[l] % 4 == 0, LOWBIT_ERR_UNSUPPORTED_SHAPE);
        LB_CHECK(w_packed[l] != nullptr, LOWBIT_ERR_INVALID_ARG);
        LB_CHECK(aligned16(w_packed[l]), LOWBIT_ERR_MISALIGNED);
    }
    LB_CHECK(dims[n_layers] >= 1 && dims[n_layers] <= 256, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    const size_t smem = z80_smem_bytes(dims, n_layers);
    LB_CHECK(smem > 0 && smem <= 226u * 1024u, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    if (batch == 0) return LOWBIT_OK;
    LB_CHECK(queries && reply_len && (reply || max_new == 0), LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(aligned16(queries) && aligned16(reply_len) && (reply == nullptr || aligned16(reply)),
             LOWBIT_ERR_MISALIGNED);
    return z80_generate_launch(w_packed, dims, n_layers, queries, batch, qlen, charset, max_new, reply, reply_len,
                               as_stream(stream));
}

// ---------------------------------------------------------------------------
// glue
// ---------------------------------------------------------------------------

lowbit_status lowbit_rmsnorm_bf16(const float *a, const float *b, int M, int D, float eps, uint16_t *out,
                                  void *stream)
{
    LB_CHECK(M >= 1 && D >= 1 && eps >= 0.f && a && out, LOWBIT_ERR_INVALID_ARG);
    LB_CHECK(D % 8 == 0 && (int64_t)M * D < kMaxElems, LOWBIT_ERR_UNSUPPORTED_SHAPE);
    LB_CHECK(aligned16(a) && aligned16(out) && (b == nullptr || aligned16(b)), LOWBIT_ERR_MISALIGNED);
    return rmsnorm_launch(a, b, M, D, eps, out, as_stream(stream));
}

}  // extern "C"
