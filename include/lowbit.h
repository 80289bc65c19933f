/*
 * lowbit.h -- packed low-bit matrix-vector and small-batch matrix products
 * for NVIDIA B200 (sm_100a).  C ABI of liblowbit.so.
 *
 * Three weight formats are supported.  Their definitions come from three web
 * pages (named by title and section):
 *
 *   Q1_0_g128  "Bonsai-27B-gguf technical white paper digest", section
 *              "technical architecture highlights": every weight is one sign
 *              bit (-1 or +1) and every 128 weights share one FP16 scale
 *              (1.125 bits per weight).
 *   Q2         "Show HN: Z80-uLM, a conversational AI that fits in 40KB":
 *              2-bit weights {-2,-1,0,+1}, four per byte (the "unpack 2-bit
 *              weight" listing), a 16-bit two's-complement accumulator (the
 *              MULADD listing), an arithmetic shift right by 2 after every
 *              layer (the shift listing), ReLU between hidden layers (the
 *              architecture list).
 *   INT4_G64   "acorn-llm 0.11.4", section "int4 quantisation quality: group
 *              quantisation": symmetric int4 with one scale per group of 64
 *              values along the input dimension; here the scale is FP16.
 *
 * Conventions shared by every entry point
 *   - N = output rows, K = reduction length, M = batch rows of x.
 *   - Matrices are row-major.  x is [M][K] bfloat16, y is [M][N] float32.
 *   - fp16 and bf16 values are passed as uint16_t bit patterns.
 *   - Every pointer is a DEVICE pointer unless marked HOST.  All device
 *     pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     Calls are asynchronous and ordered on `stream`; none synchronises.
 *   - Arguments are checked on the host before anything is enqueued.  On a
 *     non-OK status nothing has been enqueued.  LOWBIT_ERR_CUDA reports a
 *     failed launch (cudaGetLastError).  Faults inside a kernel are
 *     asynchronous and surface at the caller's next synchronisation.
 *   - The caller owns every buffer.  The library allocates no device memory
 *     and keeps no state across calls besides the fault flags
 *     (lowbit_fault_flags) and the scratch array of the allocation-free
 *     entry point; entry points are safe to call from several host threads
 *     on different streams.  Only the Q1_0_g128 entry points take a
 *     caller-provided workspace, for the shapes whose kernel reads a
 *     prepared activation from global memory; its size comes from the
 *     matching *_workspace_bytes() query, which returns 0 for every shape a
 *     one-launch kernel takes (the activation is then built in shared
 *     memory).
 *
 * Packed layouts (one row of a matrix is packed along K):
 *   Q1_0_g128  bits   [N][K/8]:   weight k is bit (k%8) of byte k/8; bit 1
 *                                 means +1, bit 0 means -1.
 *              scales [N][K/128]: fp16; scale g covers k in [128g, 128g+128).
 *   Q2         bytes  [out][in/4]: the code of input i is bits 2*(i%4)..+1
 *                                 of byte i/4 (lowest field first); code c
 *                                 stands for the weight c-2.
 *   INT4_G64   bytes  [N][K/2]:   weight k is the low nibble (k even) or the
 *                                 high nibble (k odd) of byte k/2, a 4-bit
 *                                 two's-complement value in [-8, 7].
 *              scales [N][K/64]:  fp16; scale g covers k in [64g, 64g+64).
 *   TERNARY_G128 bytes [N][26*K/128]: weights w in {-1, 0, +1}; the trits
 *                                 t = w + 1 of group g (k in [128g, 128g+128))
 *                                 fill its 26 bytes five per byte in base 3:
 *                                 byte 26g + j (j < 25) = sum_i t[128g+5j+i]
 *                                 3^i, byte 26g + 25 = sum_{i<3}
 *                                 t[128g+125+i] 3^i.  A byte b holds digits
 *                                 floor(b / 3^i) mod 3; the packer writes
 *                                 only b < 243 (b < 27 in the last byte).
 *              scales [N][K/128]: fp16.  1.75 bits per weight.
 */
#ifndef LOWBIT_H
#define LOWBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LOWBIT_OK = 0,
    LOWBIT_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, size < 0, ... */
    LOWBIT_ERR_MISALIGNED = 2,        /* a device pointer is not 16-byte aligned */
    LOWBIT_ERR_UNSUPPORTED_SHAPE = 3, /* K or a dimension breaks a format rule */
    LOWBIT_ERR_CUDA = 4               /* a CUDA launch failed */
} lowbit_status;

typedef enum {
    LOWBIT_FMT_Q1_G128 = 1,
    LOWBIT_FMT_Q2 = 2,
    LOWBIT_FMT_INT4_G64 = 3,
    LOWBIT_FMT_TERNARY_G128 = 4
} lowbit_format;

/* Static string for a status code (never NULL). */
const char *lowbit_status_string(lowbit_status s);

/* Library version, major*10000 + minor*100 + patch. */
int lowbit_version(void);

/* Faults the kernels of the current device recorded since the last call,
 * and clears them: 0 = none; bit 0 = a bounded wait inside the INT4_G64
 * tcgen05 GEMM ran out, bit 2 = a grid barrier of lowbit_q1g128_stack_step,
 * bit 3 = a wait on the shared activation ring of a small-batch kernel
 * (Q1_0_g128 at 2 <= M <= 16, INT4_G64 at 2 <= M <= 32; the results of such
 * a call are then not valid); -1 = the flags could not
 * be read.  This is a diagnostic call, not part of any product: it reads the
 * flags from device memory and therefore synchronises with the device (every
 * other entry point is asynchronous). */
int lowbit_fault_flags(void);

/* ---------------------------------------------------------------------------
 * Packing (all three formats).
 *
 * lowbit_pack: codes int8 [rows][cols] -> packed uint8 [rows][cols/per_byte]
 * with per_byte = 8 (Q1_0_g128; codes 0 or 1), 4 (Q2; codes 0..3) or 2
 * (INT4_G64; codes -8..7); TERNARY_G128 (codes -1..1) writes 26 bytes per
 * 128 columns.  Codes outside the format's range are masked to the field
 * width (clamped to [-1, 1] for TERNARY_G128; the packer does not read the
 * data on the host to check).  lowbit_unpack is the exact inverse, and
 * decodes every packed byte value as the layout above defines.
 * cols must be a multiple of per_byte (of 128 for TERNARY_G128), else
 * LOWBIT_ERR_UNSUPPORTED_SHAPE.
 * rows == 0 is a no-op that returns LOWBIT_OK.
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_pack(lowbit_format fmt, const int8_t *codes, int64_t rows, int64_t cols,
                          uint8_t *packed, void *stream);
/* Quantisation of float weights straight into the packed layouts above.
 *   w       [rows][cols] float32 (16-byte aligned)
 *   packed  [rows][cols/8] (Q1_0_g128) or [rows][cols/2] (INT4_G64)
 *   scales  [rows][cols/128] or [rows][cols/64] FP16 bit patterns
 * Q1_0_g128 ("Bonsai-27B-gguf technical white paper digest", "technical
 * architecture highlights" fixes one sign per weight and one FP16 scale per
 * 128): bit = (w >= 0), so -0.0 gives +1 and NaN -1; the scale is the
 * group's mean |w| (the d minimising sum (w - d*sign)^2).
 * INT4_G64 ("acorn-llm 0.11.4", "int4 quantisation quality: group
 * quantisation": round-to-nearest int4, one scale per group along the input
 * dimension): d = max|w| / 7 per 64-group; q = w / d rounded to nearest,
 * ties to even, clamped to [-8, 7] (-8 never occurs); q = 0 where d = 0 or w
 * is NaN.
 * Scales round to FP16 nearest-even; magnitudes >= 65504 saturate to 65504.
 * Every step is an IEEE double operation in a fixed order, so the result is
 * the same bits on every run.  LOWBIT_FMT_Q2 returns
 * LOWBIT_ERR_UNSUPPORTED_SHAPE (the pages give no rule for its codes);
 * cols must be a multiple of the group size; rows == 0 is a no-op. */
lowbit_status lowbit_quantize(lowbit_format fmt, const float *w, int64_t rows, int64_t cols,
                              uint8_t *packed, uint16_t *scales, void *stream);
lowbit_status lowbit_unpack(lowbit_format fmt, const uint8_t *packed, int64_t rows, int64_t cols,
                            int8_t *codes, void *stream);

/* ---------------------------------------------------------------------------
 * Q1_0_g128 product (Bonsai white-paper digest, "technical architecture
 * highlights"):
 *     y[m][n] = sum_g d[n][g] * sum_{k in group g} s(b[n][k]) * x[m][k]
 * with s(1) = +1, s(0) = -1, groups of 128 consecutive k, fp32 accumulate.
 *
 *   w_bits   [N][K/8]   packed sign bits
 *   w_scales [N][K/128] fp16 scales
 *   x        [M][K]     bf16
 *   y        [M][N]     fp32 (written, not accumulated into)
 * Shapes: 1 <= M <= 16, N >= 1, K >= 128, K % 128 == 0, N*K < 2^40.
 * Activations must be finite; values below 2^-96 in magnitude count as 0 at
 * M = 1 (the tensor-core path works in per-group 24-bit fixed point).
 * workspace: device scratch of at least lowbit_q1g128_workspace_bytes(M, N,
 * K) bytes (may be NULL when that size is 0).  The size is 0 whenever the
 * product is one launch (M >= 2, and at M = 1 every shape whose matrix is
 * split across the GPU by K slices, e.g. 4096 x 4096); it is the prepared
 * activation otherwise (M = 1 with so many rows -- above about 150k on 148
 * SMs -- that the persistent kernel takes the product).  It needs no
 * initialisation.  Calls that share one workspace must be ordered on one
 * stream.
 * The weights are read before the kernel waits for the previous kernel on
 * the stream (programmatic dependent launch): a kernel that writes w_bits or
 * w_scales must not trigger its dependents early.  The library's packers
 * never do.
 * ------------------------------------------------------------------------- */
size_t lowbit_q1g128_workspace_bytes(int M, int N, int K);
lowbit_status lowbit_q1g128_gemv(const uint8_t *w_bits, const uint16_t *w_scales,
                                 const uint16_t *x, float *y, int M, int N, int K,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* Split form of the same product for an activation that feeds several
 * weight matrices (for example the projections that read one normalised
 * hidden state).  lowbit_q1g128_prepare_act converts x once into the operand
 * form the product kernels read (act, lowbit_q1g128_act_bytes(M, K) bytes).
 * lowbit_q1g128_gemv_act_group then computes y_r = W_r x for R matrices of
 * the same shape [N][K] in one launch:
 *   w_bits, w_scales, y: HOST arrays of R device pointers (1 <= R <= 256);
 *   each y_r equals a separate lowbit_q1g128_gemv call up to fp32 summation
 *   order (the K-split depends on the amount of work in the launch).
 * lowbit_q1g128_gemv_act is the R = 1 case.  Same shape rules as above.
 * Workspace: lowbit_q1g128_act_workspace_bytes(R, M, N, K) bytes (NULL
 * allowed when 0; the current kernels need none: split-K partial sums are
 * reduced in thread-block-cluster shared memory).  Calls that share an act
 * buffer must be ordered on one stream.
 * At M = 1 the tensor-core kernel takes every shape with K/128 even; other
 * shapes run a CUDA-core kernel (same results within the float bar). */
size_t lowbit_q1g128_act_bytes(int M, int K);
size_t lowbit_q1g128_act_workspace_bytes(int R, int M, int N, int K);
lowbit_status lowbit_q1g128_prepare_act(const uint16_t *x, int M, int K, void *act,
                                        size_t act_bytes, void *stream);
lowbit_status lowbit_q1g128_gemv_act(const uint8_t *w_bits, const uint16_t *w_scales,
                                     const void *act, float *y, int M, int N, int K,
                                     void *workspace, size_t workspace_bytes, void *stream);
lowbit_status lowbit_q1g128_gemv_act_group(const uint8_t *const *w_bits,
                                           const uint16_t *const *w_scales, const void *act,
                                           float *const *y, int R, int M, int N, int K,
                                           void *workspace, size_t workspace_bytes, void *stream);

/* The same group product straight from x: y_r = W_r x for R matrices of one
 * shape [N][K] that read one activation x [M][K] (bf16).
 *   w_bits, w_scales, y: HOST arrays of R device pointers (1 <= R <= 256),
 *   16-byte aligned; results as lowbit_q1g128_gemv_act_group.
 * At M <= 4, with K % 1024 == 0, N % 32 == 0 and at least SMs * 8
 * (32-row block, matrix) pairs (e.g. 10 or more 4096-row matrices on 148
 * SMs), this is one launch: every CTA turns x into the operand form itself,
 * the masked sign planes feed one integer mma per vector, and no workspace is
 * needed (at M = 2..4 while all M vectors' operands fit in shared memory:
 * K up to about 12k at M = 3, 4).  At 2 <= M <= 16 otherwise, with
 * K % 256 == 0 and at least SMs * 8 32-row blocks over the group, it is one
 * launch of a persistent bf16 kernel (each warp owns a 32-row block over all
 * of K; the warps of a CTA share x); with fewer blocks, one split-K launch
 * per 8 matrices.  Neither needs a workspace.  Other shapes (M = 1) prepare
 * the activation in the workspace and run lowbit_q1g128_gemv_act_group.
 * Workspace: lowbit_q1g128_group_workspace_bytes(R, M, N, K) bytes (NULL
 * allowed when 0).  Calls that share a workspace must be ordered on one
 * stream. */
size_t lowbit_q1g128_group_workspace_bytes(int R, int M, int N, int K);
lowbit_status lowbit_q1g128_gemv_group(const uint8_t *const *w_bits,
                                       const uint16_t *const *w_scales, const uint16_t *x,
                                       float *const *y, int R, int M, int N, int K,
                                       void *workspace, size_t workspace_bytes, void *stream);

/* Allocation-free form of lowbit_q1g128_gemv.  The pages have no
 * counterpart: it exists for callers that cannot allocate device memory --
 * a plugin whose host framework owns every device allocation, a real-time or
 * embedded deployment that reserves all device memory up front, or code that
 * must not call cudaMalloc at the point where the product runs.
 *   Same arguments and result as lowbit_q1g128_gemv, without a workspace.
 *   Shapes that lowbit_q1g128_gemv runs in one launch need no scratch and
 *   take that launch.  The others (M = 1 with very many rows) keep the
 *   prepared activation in a fixed 512 KiB array in the library's own device
 *   memory, present on every device that loads the library until the process
 *   exits.  That array limits K to 32768 at M = 1: a larger K returns
 *   LOWBIT_ERR_UNSUPPORTED_SHAPE for every N, before anything is enqueued.
 *   The call allocates nothing.
 *   The device address of the array is looked up (with the device current)
 *   on a device's first call that needs it, and again whenever the device's
 *   context has changed since (for example after cudaDeviceReset); make the
 *   first call before any stream capture.
 *   All calls share the one array, so calls that overlap on the GPU (for
 *   example on two streams without ordering between them) race; order them
 *   on one stream.  Each call overwrites the part it reads, so the contents a
 *   previous call left behind do no harm. */
lowbit_status lowbit_q1g128_gemv_noalloc(const uint8_t *w_bits, const uint16_t *w_scales,
                                         const uint16_t *x, float *y, int M, int N, int K,
                                         void *stream);

/* ---------------------------------------------------------------------------
 * One decode step (M = 1) through a stack of Q1_0_g128 linear projections,
 * in one launch.  The pages fix only the weight format ("Bonsai-27B-gguf
 * technical white paper digest", "technical architecture highlights") and
 * that decode streams every layer's weights once per token; the chaining is
 * this library's reading of the workload: per layer q, k, v, o (hidden ->
 * hidden), gate and up (hidden -> ffn, same input, outputs summed), down
 * (ffn -> hidden); every projection's input is bf16_rne(v / sqrt(mean(v^2)
 * + eps)) of the previous fp32 output (v = gate + up before down), and the
 * step output is that normalisation of the last down output.  Layer 0's q
 * reads x as given.
 *   w_bits, w_scales: HOST arrays of 7 * n_layers device pointers, in the
 *     order q, k, v, o, gate, up, down for each layer; shapes as for
 *     lowbit_q1g128_gemv ([N][K/8] and [N][K/128]).
 *   x: [hidden] bf16, the step input, overwritten with the step output.
 *   workspace: lowbit_q1g128_stack_workspace_bytes(...) bytes; the call
 *     initialises what it needs (it enqueues a memset first).
 *   record_inputs / record_outputs: NULL, or [7 * n_layers][ffn] bf16 /
 *     fp32 that receive every projection's input and fp32 output (row i
 *     uses the first K or N entries).
 * Needs hidden and ffn multiples of 512, ffn >= hidden, 1 <= n_layers <=
 * 73, and ffn / 512 at most the number of CTAs resident at once (one per SM;
 * else LOWBIT_ERR_UNSUPPORTED_SHAPE).  The kernel is a cooperative launch (every CTA resident) whose phases
 * are separated by a grid barrier; a barrier wait bounded at 2 s that runs
 * out sets bit 2 of lowbit_fault_flags().  The projections' partial sums
 * are added with fp32 atomics, so results can differ in the last bits from
 * run to run. */
size_t lowbit_q1g128_stack_workspace_bytes(int n_layers, int hidden, int ffn);
lowbit_status lowbit_q1g128_stack_step(const uint8_t *const *w_bits, const uint16_t *const *w_scales,
                                       int n_layers, int hidden, int ffn, uint16_t *x, float eps,
                                       void *workspace, size_t workspace_bytes,
                                       uint16_t *record_inputs, float *record_outputs, void *stream);

/* ---------------------------------------------------------------------------
 * INT4_G64 product (acorn-llm 0.11.4, "int4 quantisation quality: group
 * quantisation"):
 *     y[m][n] = sum_g d[n][g] * sum_{k in group g} q[n][k] * x[m][k]
 * with q in [-8, 7], groups of 64 consecutive k, fp32 accumulate.
 *
 *   w_q      [N][K/2]  packed nibbles
 *   w_scales [N][K/64] fp16 scales
 *   x        [M][K]    bf16
 *   y        [M][N]    fp32
 * Shapes: M >= 1, N >= 1, K >= 64, K % 64 == 0, M*K, N*K < 2^40.
 * The kernel is chosen by M: at M = 1 a weight-streaming tensor-core GEMV
 * (mma.sync on the packed nibbles, integer limbs of x); for 2 <= M <= 32
 * (K % 128 == 0) mma.sync on bf16 operands, q exact in bf16 and the group
 * scale applied once per group; above that a tcgen05 GEMM that dequantises
 * each weight tile into shared memory as exact bf16 integers q, accumulates
 * each 64-k group in TMEM and applies the group scale in fp32 (with few
 * 128-row tiles, K is cut into slices whose sums are added into y, which the
 * call zeroes first with a memset on the stream); other shapes a CUDA-core
 * kernel.  Every kernel builds its operands on chip: no workspace.
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_int4g64_gemm(const uint8_t *w_q, const uint16_t *w_scales,
                                  const uint16_t *x, float *y, int M, int N, int K,
                                  void *stream);

/* Group form: y_r = W_r x for R matrices of one shape [N][K] that read one
 * activation x [M][K] (w_q, w_scales, y: HOST arrays of R device pointers,
 * 1 <= R <= 256, 16-byte aligned).  At M = 1, with N % 32 == 0 and at least
 * SMs * 8 (32-row block, matrix) pairs (e.g. 4 or more 11008-row matrices
 * on 148 SMs), this is one launch of a persistent kernel: one CTA per SM
 * builds the activation from x and streams its equal share of every matrix's
 * weights.  At 2 <= M <= 32 with K % 128 == 0 and at least SMs * 8 32-row
 * blocks over the group, one launch of the persistent small-batch kernel
 * (as for Q1_0_g128); with fewer blocks, one split-K launch per 8 matrices.
 * Other shapes run lowbit_int4g64_gemm once per matrix.  Results equal the
 * single calls up to fp32 summation order. */
lowbit_status lowbit_int4g64_gemm_group(const uint8_t *const *w_q,
                                        const uint16_t *const *w_scales, const uint16_t *x,
                                        float *const *y, int R, int M, int N, int K,
                                        void *stream);

/* ---------------------------------------------------------------------------
 * Ternary product with an FP16 scale per 128 ("Bonsai-27B-gguf technical
 * white paper digest": the ternary 27B model is 5.9 GB where the 1.125-bit
 * one is 3.79 GB, about 1.75 bits per weight; the page gives no layout, the
 * TERNARY_G128 layout above is this library's reading, and it stores exactly
 * 1.75 bits per weight):
 *     y[m][n] = sum_g d[n][g] * sum_{k in group g} w[n][k] * x[m][k]
 * with w in {-1, 0, +1}, groups of 128, fp32 accumulate.
 *   w        [N][26*K/128] packed trits
 *   w_scales [N][K/128]    fp16 scales
 *   x        [M][K]        bf16
 *   y        [M][N]        fp32
 * Shapes: 1 <= M <= 16, N >= 1, K % 128 == 0.  At M = 1 with K % 1024 == 0
 * the product streams 32 rows per warp (x as per-group 22-bit fixed point,
 * exact int32 group sums), writing y directly, or, when the group has too
 * few 32-row blocks to fill the GPU, adding K-slice partial sums into y
 * after zeroing it (fp32 atomics: the last bits may differ run to run).
 * Other shapes run a plain CUDA-core kernel.  Packed bytes >= 243 are not
 * part of the format and give unspecified products.
 * Group form: R matrices of one shape that read one x (HOST arrays of R
 * device pointers, 1 <= R <= 256).
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_t3g128_gemv(const uint8_t *w, const uint16_t *w_scales, const uint16_t *x,
                                 float *y, int M, int N, int K, void *stream);
lowbit_status lowbit_t3g128_gemv_group(const uint8_t *const *w, const uint16_t *const *w_scales,
                                       const uint16_t *x, float *const *y, int R, int M, int N,
                                       int K, void *stream);

/* ---------------------------------------------------------------------------
 * Z80-style 2-bit integer MLP ("Show HN: Z80-uLM"), fused over all layers:
 * for each input vector, a_0 = x; for each layer l with weights w = code-2,
 *     acc   = sum_i w[o][i] * a_l[i]   reduced mod 2^16 (16-bit wrapping)
 *     z     = acc >> 2                 arithmetic shift (floor division by 4)
 *     a_l+1 = max(z, 0) on hidden layers; logits = z on the last layer;
 * argmax = smallest index of the largest logit.
 *
 *   w_packed  HOST array of n_layers device pointers; layer l is
 *             [dims[l+1]][dims[l]/4] packed Q2 codes
 *   dims      HOST array of n_layers+1 widths
 *   x         [batch][dims[0]] int16
 *   logits    [batch][dims[n_layers]] int16
 *   argmax    [batch] int32, or NULL
 * Shapes: 1 <= n_layers <= 8; 4 <= dims[l] <= 1024 and dims[l] % 4 == 0 for
 * l < n_layers; 1 <= dims[n_layers] <= 1024; the packed weights of all layers
 * together at most 96 KiB; batch >= 0.
 * Bit-exact: the result equals the integer definition above for any input.
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_q2_mlp_forward(const uint8_t *const *w_packed, const int32_t *dims,
                                    int n_layers, const int16_t *x, int batch,
                                    int16_t *logits, int32_t *argmax, void *stream);

/* ---------------------------------------------------------------------------
 * Autoregressive replies of the 2-bit network ("Show HN: Z80-uLM",
 * architecture list: 128 query + 128 context trigram buckets in, one output
 * neuron per character; feature list: autoregressive generation, one
 * character at a time; "trigram hash encoding": text hashed into 128
 * buckets, word order does not matter).  For every conversation b:
 *     q = buckets(query b);  reply = ""
 *     repeat up to max_new times:
 *         logits = network([q, buckets(reply)])   (as lowbit_q2_mlp_forward)
 *         c = charset[argmax(logits)];  stop if c == 0;  reply += c
 * buckets(text): the text is split into words at spaces; each word (at most
 * 255 characters kept), lower-cased (A-Z only) and padded with one space on
 * each side, adds 32 to bucket FNV-1a-32(w) mod 128 for every 3-byte window
 * w.  The page shows the buckets and the loop but not the hash, the per-
 * trigram value or how the context is kept; these are this library's
 * readings (the context is the encoding of the reply so far, and charset
 * byte 0 ends a reply).  The kernel updates the context buckets in place as
 * characters arrive; the result equals the re-encoding above exactly.
 *
 *   w_packed, dims, n_layers: the network as for lowbit_q2_mlp_forward, with
 *             dims[0] == 256 and every width <= 256
 *   queries   [batch][qlen] bytes; a query ends at its first 0 byte or at
 *             qlen (1 <= qlen <= 4096)
 *   charset   HOST array of dims[n_layers] bytes: output index -> character;
 *             the byte 0 ends a reply
 *   reply     [batch][max_new] bytes (0 <= max_new <= 250); bytes after a
 *             reply's end are set to 0 (may be NULL when max_new == 0)
 *   reply_len [batch] int32: characters in each reply
 * The weights of all layers, expanded to bytes, must fit in shared memory
 * (about 190 KB; the 256->192->128->40 network takes 85 KB), else
 * LOWBIT_ERR_UNSUPPORTED_SHAPE.  Bit-exact: integer arithmetic throughout.
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_z80_generate(const uint8_t *const *w_packed, const int32_t *dims, int n_layers,
                                  const uint8_t *queries, int batch, int qlen, const uint8_t *charset,
                                  int max_new, uint8_t *reply, int32_t *reply_len, void *stream);

/* ---------------------------------------------------------------------------
 * Glue between the projections of a layer stack: RMS normalisation with unit
 * gain, rounded to bf16.
 *     v[m][d] = a[m][d] (+ b[m][d] when b is not NULL)
 *     out[m][d] = bf16_rne( v[m][d] / sqrt(mean_d v[m][d]^2 + eps) )
 * computed in fp32.  a, b [M][D] fp32; out [M][D] bf16.  M >= 1, 1 <= D,
 * D % 8 == 0, eps >= 0.
 * ------------------------------------------------------------------------- */
lowbit_status lowbit_rmsnorm_bf16(const float *a, const float *b, int M, int D, float eps,
                                  uint16_t *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LOWBIT_H */
