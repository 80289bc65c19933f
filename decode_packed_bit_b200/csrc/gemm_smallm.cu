// gemm_smallm.cu -- products at small batch on the bf16 tensor cores
// (mma.sync m16n8k16, fp32 accumulate): Q1_0_g128 for 2 <= M <= 16 and
// INT4_G64 for 2 <= M <= 32, for one matrix (k_smallm: cluster split-K) or a
// group of R matrices that read one x (k_smallm_grp: persistent).
//
// What is computed, for every matrix:
//   Q1_0_g128 ("Bonsai-27B-gguf technical white paper digest", "technical
//   architecture highlights": one sign bit per weight, one FP16 scale per
//   128 weights):
//     y[m][n] = sum_g d[n][g] * sum_{k in g} s(b[n][k]) * x[m][k],  s(1) = +1, s(0) = -1;
//   INT4_G64 ("acorn-llm 0.11.4", "int4 quantisation quality: group
//   quantisation"): y[m][n] = sum_g d[n][g] * sum_{k in g} q[n][k] * x[m][k].
//
// Operands.  A is a weight tile with every weight as an exact bf16 (+-1, or
// the integer q), B is x (bf16, exact), so the tensor core sums exact
// products in fp32, one accumulator per group (the group's first MMA starts
// from zero); the group's scale is applied once per (row, group, vector)
// with an FMA.  A is built in registers:
//   Q1_0_g128, no table: for a 32-bit word w of a row's signs (bits j <->
//     k0 + j), w * 2^(15-j) has bit j at bit 15 and bit j+16 at bit 31, so
//     one LOP3 (~v & 0x80008000 | 0x3F803F80) gives the bf16 pair
//     {s(j), s(j+16)}.  In MMA step sigma of a 32-k unit, lane t's slots
//     2t, 2t+1 take j = 4t + 2 sigma (and j + 16), slots 2t+8, 2t+9 take
//     j + 1 (and j + 17); x is stored as pairs P[i] = {x[k0+i], x[k0+i+16]},
//     so the B registers of both steps are one 16-byte load, P[4t .. 4t+3].
//     The multipliers come from shared memory, which keeps the products on
//     the integer multiply-add pipe and the ALU pipe free for the LOP3s.
//   INT4_G64: a lane's four k slots of a 16-k step are the two packed bytes
//     2t, 2t+1 of the row's 8 (k 4t .. 4t+3, low nibble first), so B is
//     x[m][k .. k+3] in natural order.  A byte b becomes the bf16 pair
//     {q_lo, q_hi}: prmt isolates b, b * 0x1001 puts its nibbles at bits 0
//     and 16, and with the sign bit of each nibble flipped and 0x4300
//     (128.0) or-ed in, each half reads 136 + q exactly; a bf16 subtraction
//     of 136 leaves q.
//
// Data movement (both kernels).  Each consumer warp owns 32 rows (two
// 16-row tiles) and streams their packed weights and scales through a
// cp.async ring of its own, one step (256 k for Q1_0_g128, 128 k for
// INT4_G64) at a time, so it waits only for its own copies.  x is shared by
// the CTA's consumer warps through a ring of slots guarded by mbarriers:
// one producer warp fills slot u % SLOTS with the u-th step of x and
// signals `full`; every consumer warp signals `empty` once it has read the
// slot.  For INT4_G64 one 2-D tensor copy per step lands x in the slot
// directly (each row one step of k plus 16 more, read past the step or zero
// filled past K, which puts rows 288 bytes apart: a half warp's 8-byte reads
// of four rows are free of bank conflicts).  For Q1_0_g128 the tensor copies
// go to a raw ring a few steps ahead and the producer rewrites each raw
// slice once into the P order.  Every wait is bounded (a wait that runs out
// sets the fault word and the warp leaves its loop).
//
// Work split.  k_smallm: a CTA of four consumer warps takes 128 rows of one
// K-slice of one of up to 8 matrices that read the same x; the S slices of a
// row block form a thread-block cluster and add their partial sums in rank
// order through distributed shared memory.
// k_smallm_grp: one CTA per SM; every consumer warp owns one 32-row block
// of one matrix over all of K per round, and the rounds walk the group's
// (matrix, block) list; warps may drift apart by up to SLOTS steps.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc_common.cuh"

namespace lowbit {

// ---------------------------------------------------------------------------
// formats: steps and weight stages
// ---------------------------------------------------------------------------

constexpr int kSmStepK = 256;              // Q1_0_g128: k per step (two groups)
constexpr int kSmRowStride = 48;           // 32 bytes of signs per row, padded: conflict-free 16-byte reads
constexpr int kSmStageW = 32 * kSmRowStride;
constexpr int kSmStageBytes = kSmStageW + 32 * 4;  // + two fp16 scales per row
constexpr int kSmMaxM = 16;
constexpr int kI4sStepK = 128;             // INT4_G64: k per step (two groups of 64)
constexpr int kI4sRowStride = 80;          // 64 bytes per row, padded: conflict-free 4-byte reads
constexpr int kI4sStageW = 32 * kI4sRowStride;
constexpr int kI4sStageBytes = kI4sStageW + 32 * 4;  // + two fp16 scales per row
constexpr int kI4sMaxM = 32;
constexpr int kSmMaxSmem = 220 * 1024;

template <int FMT>
struct SgFmt;
template <>
struct SgFmt<1> {
    static constexpr int kStepK = kSmStepK, kStageBytes = kSmStageBytes, kRowStride = kSmRowStride,
                         kStageW = kSmStageW, kStepBytes = kSmStepK / 8;
};
template <>
struct SgFmt<3> {
    static constexpr int kStepK = kI4sStepK, kStageBytes = kI4sStageBytes, kRowStride = kI4sRowStride,
                         kStageW = kI4sStageW, kStepBytes = kI4sStepK / 2;
};

// Bytes of one row of an x slot.  Q1_0_g128 (P order): 64 per 32-k unit plus
// 64, so that rows sit 64 bytes (mod 128) apart and a quarter warp's 16-byte
// reads of two rows are free of bank conflicts.  INT4_G64 (natural order,
// filled by the tensor copy): the step's k plus 16 more.
__host__ __device__ constexpr int sg_xrow(int fmt) { return fmt == 1 ? kSmStepK * 2 + 64 : (kI4sStepK + 16) * 2; }

// Shared memory of both kernels starts with the raw ring (the grouped
// kernel: one step of the M rows of x per slot, natural order) and the x
// ring, both written by tensor copies, which want 128-byte aligned
// destinations: every slot size is a multiple of 128.
__host__ __device__ constexpr size_t sg_raw_bytes(int fmt, int raw, int M)
{
    return (size_t)raw * M * (fmt == 1 ? kSmStepK : kI4sStepK) * 2;
}
__host__ __device__ constexpr size_t sg_xring_bytes(int fmt, int slots, int NT)
{
    return (size_t)slots * 8 * NT * sg_xrow(fmt);
}

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void sm_cp16(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void sm_cp4(unsigned dst, const void *src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void sm_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void sm_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void hmma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                     uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the same MMA with a zero accumulator input
__device__ __forceinline__ void hmma0(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%10,%10,%10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void sm_cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float sm_ld_peer(const float *local, unsigned rank)
{
    unsigned ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"((unsigned)__cvta_generic_to_shared(local)),
                 "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

// Store a float into rank `rank`'s shared memory, at the address `local`
// has in this CTA.
__device__ __forceinline__ void sm_st_peer(float *local, unsigned rank, float v)
{
    unsigned ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"((unsigned)__cvta_generic_to_shared(local)),
                 "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// bf16 pair {s(j), s(j+16)} of sign word w, m = 2^(15-j): one LOP3 computing
// (~(w m) & 0x80008000) | 0x3F803F80
__device__ __forceinline__ uint32_t sg_sign_pair(uint32_t w, uint32_t m)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xAE;" : "=r"(r) : "r"(w * m), "r"(0x80008000u), "r"(0x3F803F80u));
    return r;
}

// bf16 pair {q(low nibble), q(high nibble)} of byte `sel` (0..3) of w, exact
__device__ __forceinline__ uint32_t i4_pair_bf16(uint32_t w, uint32_t sel)
{
    const uint32_t b = __byte_perm(w, 0u, sel | 0x4440u);           // the byte alone
    const uint32_t v = ((b * 0x1001u) & 0x000F000Fu) ^ 0x43084308u;  // 136 + q in each half
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x43084308u));  // - 136
    return r;
}

__device__ unsigned g_sg_fault;  // set when a bounded wait of either kernel ran out

// Wait until the phase with parity `parity` of `bar` has completed; false
// (and the fault word set) after kTcWaitNs.  The clock is read once per 16
// tests.
__device__ __forceinline__ bool sg_wait(uint64_t *bar, unsigned parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kTcWaitNs) {
            atomicExch(&g_sg_fault, 1u);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// one step of a consumer warp
// ---------------------------------------------------------------------------

template <int NT>
__device__ __forceinline__ void sg_mma(bool first, float (&acc)[NT][4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, const uint4 (&bx)[NT], int sg)
{
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = sg ? bx[nt].z : bx[nt].x, b1 = sg ? bx[nt].w : bx[nt].y;
        if (first)
            hmma0(acc[nt], a0, a1, a2, a3, b0, b1);
        else
            hmma(acc[nt], a0, a1, a2, a3, b0, b1);
    }
}

// yacc += d * acc for the rows g, g+8 of both tiles; d from the stage's scale
// words (fp16 pair per row: group 0 low, group 1 high)
template <int FMT, int NT>
__device__ __forceinline__ void sg_scale(const uint8_t *stage, int g, int grp, const float (&acc)[2][NT][4],
                                         float (&yacc)[2][NT][4])
{
    constexpr int kSW = SgFmt<FMT>::kStageW;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        const float d0 = f16_bits_to_float(*reinterpret_cast<const uint16_t *>(stage + kSW + (16 * tt + g) * 4 + 2 * grp));
        const float d1 =
            f16_bits_to_float(*reinterpret_cast<const uint16_t *>(stage + kSW + (16 * tt + 8 + g) * 4 + 2 * grp));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            yacc[tt][nt][0] = fmaf(d0, acc[tt][nt][0], yacc[tt][nt][0]);
            yacc[tt][nt][1] = fmaf(d0, acc[tt][nt][1], yacc[tt][nt][1]);
            yacc[tt][nt][2] = fmaf(d1, acc[tt][nt][2], yacc[tt][nt][2]);
            yacc[tt][nt][3] = fmaf(d1, acc[tt][nt][3], yacc[tt][nt][3]);
        }
    }
}

// Q1_0_g128 step (two groups) from a weight stage and an x slot in P order.
// mul[i] = 2^(15 - 4t - i).
template <int NT>
__device__ __forceinline__ void sg_consume_q1(const uint8_t *stage, const uint8_t *xs, int lane, const uint32_t (&mul)[4],
                                              float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(1);
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 16 * t;
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
        uint4 w4[2][2];  // the group's 16 bytes of signs of rows 16 tt + g (+8)
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int r = 0; r < 2; ++r)
                w4[tt][r] = *reinterpret_cast<const uint4 *>(stage + (16 * tt + 8 * r + g) * kSmRowStride + 16 * grp);
#pragma unroll
        for (int cu = 0; cu < 4; ++cu) {
            const int c = 4 * grp + cu;  // 32-k unit within the step
            uint4 bx[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) bx[nt] = *reinterpret_cast<const uint4 *>(xl + 8 * nt * kXR + 64 * c);
#pragma unroll
            for (int sg = 0; sg < 2; ++sg) {
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    const uint32_t w0 = cu == 0 ? w4[tt][0].x : cu == 1 ? w4[tt][0].y : cu == 2 ? w4[tt][0].z : w4[tt][0].w;
                    const uint32_t w1 = cu == 0 ? w4[tt][1].x : cu == 1 ? w4[tt][1].y : cu == 2 ? w4[tt][1].z : w4[tt][1].w;
                    const uint32_t a0 = sg_sign_pair(w0, mul[2 * sg]), a2 = sg_sign_pair(w0, mul[2 * sg + 1]);
                    const uint32_t a1 = sg_sign_pair(w1, mul[2 * sg]), a3 = sg_sign_pair(w1, mul[2 * sg + 1]);
                    sg_mma<NT>(cu == 0 && sg == 0, acc[tt], a0, a1, a2, a3, bx, sg);
                }
            }
        }
        sg_scale<1, NT>(stage, g, grp, acc, yacc);
    }
}

// Q1_0_g128 step (two groups) from a weight stage and an x slot in natural
// order: the step's two 128-k halves in two regions (8 NT rows of
// sg_xrow(3) bytes each, rows 32 mod 128 bytes apart).  The B pairs
// {x[k0+j], x[k0+j+16]} are formed in registers: two 8-byte loads and four
// prmt per unit and batch tile.  mul[i] = 2^(15 - 4t - i).
template <int NT>
__device__ __forceinline__ void sg_consume_q1n(const uint8_t *stage, const uint8_t *xs, int lane,
                                               const uint32_t (&mul)[4], float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(3);
    constexpr int kHalf = 8 * NT * kXR;  // bytes of one half's region
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 8 * t;
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
        uint4 w4[2][2];  // the group's 16 bytes of signs of rows 16 tt + g (+8)
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int r = 0; r < 2; ++r)
                w4[tt][r] = *reinterpret_cast<const uint4 *>(stage + (16 * tt + 8 * r + g) * kSmRowStride + 16 * grp);
#pragma unroll
        for (int cu = 0; cu < 4; ++cu) {
            // unit c = 4 grp + cu: half grp, 64 cu bytes into its rows
            uint4 bx[NT];  // {b0, b1} of step 0, then of step 1
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint8_t *a = xl + grp * kHalf + 8 * nt * kXR + 64 * cu;
                const uint2 lo = *reinterpret_cast<const uint2 *>(a);
                const uint2 hi = *reinterpret_cast<const uint2 *>(a + 32);
                bx[nt] = make_uint4(prmt(lo.x, hi.x, 0x5410u), prmt(lo.x, hi.x, 0x7632u), prmt(lo.y, hi.y, 0x5410u),
                                    prmt(lo.y, hi.y, 0x7632u));
            }
#pragma unroll
            for (int sg = 0; sg < 2; ++sg) {
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    const uint32_t w0 = cu == 0 ? w4[tt][0].x : cu == 1 ? w4[tt][0].y : cu == 2 ? w4[tt][0].z : w4[tt][0].w;
                    const uint32_t w1 = cu == 0 ? w4[tt][1].x : cu == 1 ? w4[tt][1].y : cu == 2 ? w4[tt][1].z : w4[tt][1].w;
                    const uint32_t a0 = sg_sign_pair(w0, mul[2 * sg]), a2 = sg_sign_pair(w0, mul[2 * sg + 1]);
                    const uint32_t a1 = sg_sign_pair(w1, mul[2 * sg]), a3 = sg_sign_pair(w1, mul[2 * sg + 1]);
                    sg_mma<NT>(cu == 0 && sg == 0, acc[tt], a0, a1, a2, a3, bx, sg);
                }
            }
        }
        sg_scale<1, NT>(stage, g, grp, acc, yacc);
    }
}

// INT4_G64 step (two groups) from a weight stage and an x slot in natural order.
template <int NT>
__device__ __forceinline__ void sg_consume_i4(const uint8_t *stage, const uint8_t *xs, int lane, float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(3);
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 8 * t;
    const uint32_t s0 = 2u * (t & 1);
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int ks = 4 * grp + s;  // 16-k step within the stage: bytes 8 ks .. 8 ks + 7 of a row
            uint2 b[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) b[nt] = *reinterpret_cast<const uint2 *>(xl + 8 * nt * kXR + 32 * ks);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t a[2][2];  // [row g / g+8][k 4t..4t+1 / 4t+2..4t+3]
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    // this lane's two bytes: 2t, 2t+1 of the step's 8
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(
                        stage + (16 * tt + 8 * r + g) * kI4sRowStride + 8 * ks + 4 * (t >> 1));
                    a[r][0] = i4_pair_bf16(w, s0);
                    a[r][1] = i4_pair_bf16(w, s0 + 1u);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (s == 0)
                        hmma0(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                    else
                        hmma(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                }
            }
        }
        sg_scale<3, NT>(stage, g, grp, acc, yacc);
    }
}

// The weight pair (k = j, j + 4) of a word of eight nibbles (k = 0..7, low
// nibble first) as exact bf16: (word >> 4j) & 0x000F000F holds the two
// nibbles in the low bits of each half; xor 8 and the exponent of 128 make
// each half 136 + q, and one bf16x2 subtract leaves q.
__device__ __forceinline__ uint32_t i4_pair4_bf16(uint32_t w, uint32_t sh)
{
    const uint32_t v = ((w >> sh) & 0x000F000Fu) ^ 0x43084308u;
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x43084308u));
    return r;
}

// INT4_G64 step (two groups) from a weight stage and an x slot in pair order
// (sg_rewrite_i4).  The MMA's k slots 2t, 2t+1 of a 16-k window carry k = t
// and t + 4 of its first 8-k block, slots 2t+8, 2t+9 the same of the second,
// in A and in B alike: a lane's A pair is one shift, one LOP3 and one bf16
// subtract of a word of the row, its B registers one 8-byte word pair.
template <int NT>
__device__ __forceinline__ void sg_consume_i4p(const uint8_t *stage, const uint8_t *xs, int lane,
                                               float (&yacc)[2][NT][4])
{
    constexpr int kXR = sg_xrow(3);
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *xl = xs + g * kXR + 8 * t;
    const uint32_t sh = 4u * (uint32_t)t;
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
        float acc[2][NT][4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int ks = 4 * grp + s;  // 16-k window within the stage: bytes 8 ks .. 8 ks + 7 of a row
            uint2 b[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) b[nt] = *reinterpret_cast<const uint2 *>(xl + 8 * nt * kXR + 32 * ks);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t a[2][2];  // [row g / g+8][block 0 / 1 of the window]
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(stage + (16 * tt + 8 * r + g) * kI4sRowStride + 8 * ks);
                    a[r][0] = i4_pair4_bf16(w.x, sh);
                    a[r][1] = i4_pair4_bf16(w.y, sh);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (s == 0)
                        hmma0(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                    else
                        hmma(acc[tt][nt], a[0][0], a[1][0], a[0][1], a[1][1], b[nt].x, b[nt].y);
                }
            }
        }
        sg_scale<3, NT>(stage, g, grp, acc, yacc);
    }
}

// ---------------------------------------------------------------------------
// weight copies of one consumer warp
// ---------------------------------------------------------------------------

// The copies of one 32-row block.  Q1_0_g128: lane L copies the 16-byte half
// L%2 of rows L/2 and L/2 + 16; INT4_G64: the 16-byte column L%4 of rows
// L/4 + {0, 8, 16, 24}; both: the scale pair of row L.  Rows past N copy
// nothing (zero fill).
// KF > 0: K fixed at compile time, so the copies' row stride is an
// immediate offset.
template <int FMT, int KF = 0>
struct SgCopy {
    static constexpr int kCopies = FMT == 1 ? 2 : 4;
    static constexpr unsigned kStride = KF > 0 ? (unsigned)((FMT == 1 ? 16 : 8) * (FMT == 1 ? KF / 8 : KF / 2)) : 0u;
    static constexpr unsigned kDstStride = FMT == 1 ? 16 * kSmRowStride : 8 * kI4sRowStride;
    const uint8_t *src = nullptr;  // copy 0's bytes of step 0; copy c reads c * stride bytes further
    const uint16_t *scale = nullptr;
    unsigned stride = 0, ok = 0;   // ok bit c: copy c's row < N; bit kCopies: the scale row

    __device__ __forceinline__ void set(const uint8_t *bits, const uint16_t *scales, int blk, int N, int K, int lane)
    {
        const int rowbytes = FMT == 1 ? K / 8 : K / 2, G = FMT == 1 ? K / 128 : K / 64;
        const int r0 = blk * 32 + (FMT == 1 ? (lane >> 1) : (lane >> 2));
        stride = (unsigned)((FMT == 1 ? 16 : 8) * rowbytes);
        ok = 0;
#pragma unroll
        for (int c = 0; c < kCopies; ++c) ok |= (r0 + (FMT == 1 ? 16 : 8) * c < N ? 1u : 0u) << c;
        src = bits + (size_t)r0 * rowbytes + (lane & (FMT == 1 ? 1 : 3)) * 16;
        const int srow = blk * 32 + lane;
        ok |= (srow < N ? 1u : 0u) << kCopies;
        scale = scales + (size_t)srow * G;
    }

    // copies of step s of the block into the stage at shared address st
    __device__ __forceinline__ void issue(unsigned st, int s, const void *dummy) const
    {
        const int lane = threadIdx.x & 31;
        const unsigned dst0 = FMT == 1 ? (unsigned)((lane >> 1) * kSmRowStride + (lane & 1) * 16)
                                       : (unsigned)((lane >> 2) * kI4sRowStride + (lane & 3) * 16);
#pragma unroll
        for (int c = 0; c < kCopies; ++c) {
            const bool v = (ok >> c) & 1u;
            const unsigned cs = KF > 0 ? kStride * c : stride * c;
            sm_cp16(st + dst0 + kDstStride * c, v ? src + cs + s * SgFmt<FMT>::kStepBytes : dummy, v);
        }
        const bool sv = (ok >> kCopies) & 1u;
        sm_cp4(st + SgFmt<FMT>::kStageW + lane * 4, sv ? scale + 2 * s : dummy, sv);
    }
};

// ---------------------------------------------------------------------------
// the producer warp
// ---------------------------------------------------------------------------

// Producer task (Q1_0_g128): output chunk q (0..3) of a 32-k unit, from the
// unit's 64 raw bytes at `src` (natural order), to `dst`.  Chunk q =
// P[4q .. 4q+3], P[i] = {x[i], x[i+16]}: words 2q, 2q+1 of the low half and
// the same words 8 later, i.e. 16-byte chunks q/2 and q/2 + 2 of the unit.
__device__ __forceinline__ void sg_rewrite(const uint8_t *src, uint8_t *dst, int q)
{
    const uint4 L = *reinterpret_cast<const uint4 *>(src + 16 * (q >> 1));
    const uint4 H = *reinterpret_cast<const uint4 *>(src + 16 * (q >> 1) + 32);
    const uint32_t l0 = (q & 1) ? L.z : L.x, l1 = (q & 1) ? L.w : L.y;
    const uint32_t h0 = (q & 1) ? H.z : H.x, h1 = (q & 1) ? H.w : H.y;
    *reinterpret_cast<uint4 *>(dst) =
        make_uint4(prmt(l0, h0, 0x5410u), prmt(l0, h0, 0x7632u), prmt(l1, h1, 0x5410u), prmt(l1, h1, 0x7632u));
}

// Producer task (INT4_G64): one 16-k window of one row, from its 32 raw
// bytes at `src` (natural order) to `dst` in pair order: the eight bf16
// pairs {x[8b + j], x[8b + j + 4]} (block b = 0, 1 of the window, j = 0..3)
// as words in the order (b=0 j=0, b=1 j=0, b=0 j=1, b=1 j=1, ...), so that a
// lane's two B registers of the window are one 8-byte word pair.
__device__ __forceinline__ void sg_rewrite_i4(const uint8_t *src, uint8_t *dst)
{
    const uint4 A = *reinterpret_cast<const uint4 *>(src);       // x0x1 x2x3 x4x5 x6x7
    const uint4 B = *reinterpret_cast<const uint4 *>(src + 16);  // x8x9 ... x14x15
    *reinterpret_cast<uint4 *>(dst) = make_uint4(prmt(A.x, A.z, 0x5410u), prmt(B.x, B.z, 0x5410u),
                                                 prmt(A.x, A.z, 0x7632u), prmt(B.x, B.z, 0x7632u));
    *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(prmt(A.y, A.w, 0x5410u), prmt(B.y, B.w, 0x5410u),
                                                      prmt(A.y, A.w, 0x7632u), prmt(B.y, B.w, 0x7632u));
}

// Fill x-ring slot u % SLOTS with step s0 + u % ncycle of x, u = 0 .. total-1.
// DIRECT: tensor copies straight into the slot, boxes of all M rows and
// sg_xrow(3) / 2 k (one per INT4_G64 step, one per 128-k half of a
// Q1_0_g128 step, the halves in two regions), natural order.  Otherwise raw
// slices of one step each, rewritten once into the consumers' order
// (Q1_0_g128: {x[k], x[k+16]} pairs; INT4_G64: {x[k], x[k+4]} pairs).
// Called by every lane of the producer warp; returns when done or when a
// wait ran out.
template <int FMT, int NT, int SLOTS, int RAW, bool DIRECT>
__device__ __forceinline__ void sg_produce(const CUtensorMap *xmap, uint8_t *raw, uint8_t *xring, uint64_t *full,
                                           uint64_t *empty, uint64_t *rawbar, int M, int total, int s0, int ncycle,
                                           int lane)
{
    constexpr int kXR = sg_xrow(FMT);
    constexpr int kXSlot = 8 * NT * kXR;
    pdl_wait_primary();  // x is produced by earlier kernels
    if (DIRECT) {
        constexpr int kBoxes = FMT == 1 ? 2 : 1;
        constexpr int kRow = sg_xrow(3);  // bytes of a box row
        if (lane == 0) {
            const unsigned bytes = (unsigned)(kBoxes * M * kRow);
            for (int u = 0; u < total; ++u) {
                const int sl = u % SLOTS;
                if (u >= SLOTS && !sg_wait(empty + sl, ((u / SLOTS) - 1) & 1)) break;
                mbar_arrive_expect_tx(full + sl, bytes);
                const int k0 = (s0 + u % ncycle) * SgFmt<FMT>::kStepK;
#pragma unroll
                for (int h = 0; h < kBoxes; ++h)
                    tma_load_2d(xring + sl * kXSlot + h * (8 * NT * kRow), xmap, k0 + h * kI4sStepK, 0, full + sl);
            }
        }
        return;
    }
    // raw slices by tensor copy, rewritten once into the x ring
    constexpr int kStepK = SgFmt<FMT>::kStepK;
    const int rawslot = M * kStepK * 2;
    auto copy_raw = [&](int v) {  // lane 0: step v of the sequence into raw slot v % RAW
        if (v >= total) return;
        uint64_t *bar = rawbar + v % RAW;
        mbar_arrive_expect_tx(bar, (unsigned)rawslot);
        tma_load_2d(raw + (v % RAW) * rawslot, xmap, (s0 + v % ncycle) * kStepK, 0, bar);
    };
    if (lane == 0)
        for (int v = 0; v < RAW; ++v) copy_raw(v);
    // Q1_0_g128: task T = (unit item T/4 = (row n, unit c), output chunk
    // T%4); a quarter warp covers two adjacent units: 128 contiguous bytes
    // each way.  INT4_G64: task T = (row T/8, 16-k window T%8).
    constexpr int kUnitsStep = kSmStepK / 32;
    const int tasks = FMT == 1 ? M * kUnitsStep * 4 : M * (kI4sStepK / 16);
    constexpr int kUn = 4;
    for (int u = 0; u < total; ++u) {
        const int sl = u % SLOTS, rs = u % RAW;
        bool ok = u < SLOTS || sg_wait(empty + sl, ((u / SLOTS) - 1) & 1);
        ok = ok && sg_wait(rawbar + rs, (u / RAW) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const uint8_t *rsrc = raw + rs * rawslot;
        uint8_t *xdst = xring + sl * kXSlot;
        for (int base = 0; base < tasks; base += 32 * kUn) {
#pragma unroll
            for (int i = 0; i < kUn; ++i) {
                const int T = base + 32 * i + lane;
                if (T < tasks) {
                    if (FMT == 1) {
                        const int item = T >> 2, n = item / kUnitsStep, c = item - n * kUnitsStep;
                        sg_rewrite(rsrc + n * kSmStepK * 2 + 64 * c, xdst + n * kXR + 64 * c + 16 * (T & 3), T & 3);
                    } else {
                        const int n = T >> 3, c = T & 7;
                        sg_rewrite_i4(rsrc + n * kI4sStepK * 2 + 32 * c, xdst + n * kXR + 32 * c);
                    }
                }
            }
        }
        mbar_arrive(full + sl);
        // the raw slot's reads are done: it may be refilled (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) copy_raw(u + RAW);
    }
}

// Shared-memory setup of both kernels: x-ring rows M .. 8 NT - 1 stay zero,
// the barriers (full: the producer's 32 rewriting lanes when there is a raw
// ring, else its one copying thread; empty: the nc consumer warps), the sign
// multipliers.  Ends with a CTA barrier.
template <int FMT, int NT, int SLOTS, int RAW>
__device__ __forceinline__ void sg_setup(uint8_t *xring, uint64_t *full, uint64_t *empty, uint64_t *rawbar,
                                         uint32_t (*multab)[4], int M, int nc)
{
    // rows of kR bytes: an x slot is kRegions regions of 8 NT rows
    constexpr bool kDirectQ1 = FMT == 1 && RAW == 0;
    constexpr int kR = kDirectQ1 ? sg_xrow(3) : sg_xrow(FMT);
    constexpr int kRegions = kDirectQ1 ? 2 : 1;
    const int zrows = 8 * NT - M;
    const int per_slot = kRegions * zrows * (kR / 16);
    for (int i = threadIdx.x; i < SLOTS * per_slot; i += blockDim.x) {
        const int sl = i / per_slot, rem = i - sl * per_slot;
        const int reg = rem / (zrows * (kR / 16)), rem2 = rem - reg * zrows * (kR / 16);
        const int row = M + rem2 / (kR / 16), col = rem2 % (kR / 16);
        *reinterpret_cast<uint4 *>(xring + (sl * kRegions + reg) * 8 * NT * kR + row * kR + 16 * col) =
            make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x < 16) multab[threadIdx.x >> 2][threadIdx.x & 3] = 1u << (15 - 4 * (threadIdx.x >> 2) - (threadIdx.x & 3));
    if (threadIdx.x == 0) {
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(full + s, RAW > 0 ? 32 : 1);
            mbar_init(empty + s, (unsigned)nc);
        }
        for (int s = 0; s < RAW; ++s) mbar_init(rawbar + s, 1);
        mbar_fence_init();
    }
    __syncthreads();
}

// x [M][K] bf16 as a 2-D tensor whose box is the M rows of one step of k
// (into the raw ring) or of 128 k plus 16 (direct copies, the x ring's row
// stride), rows dense in shared memory; k past K reads as zero.
static bool sg_xmap(CUtensorMap *map, int fmt, bool direct, const uint16_t *x, int M, int K)
{
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)(direct ? sg_xrow(3) / 2 : fmt == 1 ? kSmStepK : kI4sStepK), (cuuint32_t)M};
    const cuuint32_t estride[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// ---------------------------------------------------------------------------
// single matrix: cluster split-K
// ---------------------------------------------------------------------------

constexpr int kSmWarps = 4;                 // consumer warps per CTA
constexpr int kSmRows = kSmWarps * 32;      // rows per CTA
constexpr int kSmThreads = (kSmWarps + 1) * 32;
constexpr int kSmSlots = 4;                 // x ring depth, in steps
constexpr int kSmWStages = 3;               // weight ring depth per warp, in steps
constexpr int kSmMaxCluster = 8;
// CTAs per SM the register budget allows: three (128 registers per thread),
// two for the INT4_G64 instances with three or four batch tiles (170)
__host__ __device__ constexpr int sm_min_blocks(int fmt, int NT) { return fmt == 3 && NT >= 3 ? 2 : 3; }

constexpr int kSmMaxR = 8;                  // matrices of one launch

struct SmParams {
    const uint8_t *bits[kSmMaxR];
    const uint16_t *scales[kSmMaxR];
    float *y[kSmMaxR];
    int M, N, K;
    int nsteps;  // K / step
    int L;       // steps per K-slice
    int blocks;  // 128-row blocks per matrix
    int push;    // split-K partial sums pushed to their owner before one cluster barrier
};

template <int FMT, int NT>
__global__ void __launch_bounds__(kSmThreads, sm_min_blocks(FMT, NT)) k_smallm(const __grid_constant__ CUtensorMap xmap,
                                                                           const __grid_constant__ SmParams p)
{
    constexpr int kSB = SgFmt<FMT>::kStageBytes;
    constexpr int kXSlot = 8 * NT * sg_xrow(FMT);
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bars[2 * kSmSlots];
    __shared__ uint32_t multab[4][4];
    uint64_t *full = bars, *empty = bars + kSmSlots;
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = blockIdx.x, nsl = gridDim.x;
    const int mat = blockIdx.y / p.blocks, rb = blockIdx.y - mat * p.blocks;
    const uint8_t *bits = p.bits[mat];
    float *yout = p.y[mat];
    const int s_lo = slice * p.L, s_hi = min(p.nsteps, s_lo + p.L);
    const int ns = max(0, s_hi - s_lo);  // steps of this CTA
    // x arrives by direct tensor copies (no raw ring): a CTA has few steps
    // and four consumer warps, too few to hide a rewrite of every slot
    uint8_t *xring = smem;
    uint8_t *wring0 = xring + sg_xring_bytes(FMT, kSmSlots, NT);
    float *part = reinterpret_cast<float *>(wring0 + (size_t)kSmWarps * kSmWStages * kSB);
    sg_setup<FMT, NT, kSmSlots, 0>(xring, full, empty, nullptr, multab, p.M, kSmWarps);

    if (warp == kSmWarps) {
        sg_produce<FMT, NT, kSmSlots, 1, true>(&xmap, nullptr, xring, full, empty, nullptr, p.M, ns, s_lo, max(ns, 1),
                                               lane);
    } else {
        const int blk = rb * kSmWarps + warp;
        const bool rows = blk * 32 < p.N;  // this warp has rows
        uint8_t *wring = wring0 + (size_t)warp * kSmWStages * kSB;
        const unsigned wr_s = (unsigned)__cvta_generic_to_shared(wring);
        uint32_t mul[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mul[i] = multab[lane & 3][i];
        SgCopy<FMT> cp;
        if (rows) cp.set(bits, p.scales[mat], blk, p.N, p.K, lane);
        int cs = 0, cstage = 0;  // next step to copy, its stage
        auto issue_next = [&]() {
            if (rows && cs < ns) cp.issue(wr_s + cstage * kSB, s_lo + cs, bits);
            sm_commit();
            ++cs;
            cstage = cstage + 1 == kSmWStages ? 0 : cstage + 1;
        };
#pragma unroll
        for (int t = 0; t < kSmWStages - 1; ++t) issue_next();
        pdl_wait_primary();  // y was last read by earlier kernels

        float yacc[2][NT][4];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
        int sl = 0, stage = 0;
        unsigned phase = 0;
        for (int u = 0; u < ns; ++u) {
            issue_next();
            if (!__all_sync(0xffffffffu, sg_wait(full + sl, phase))) break;
            sm_wait<kSmWStages - 1>();  // this lane's copies of step u landed
            __syncwarp();               // ... and every lane's
            if (rows) {
                if (FMT == 1)
                    sg_consume_q1n<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, mul, yacc);
                else
                    sg_consume_i4<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, yacc);
            }
            __syncwarp();  // every lane has read the slot and the stage
            if (lane == 0) mbar_arrive(empty + sl);
            if (++sl == kSmSlots) {
                sl = 0;
                phase ^= 1u;
            }
            stage = stage + 1 == kSmWStages ? 0 : stage + 1;
        }
        sm_wait<0>();
        // partial sums of this CTA: part[m][row]; lane (g, t) holds rows 16 tt + g (+8), vectors 8 nt + 2t (+1)
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = 8 * nt + 2 * t + (j & 1);
                    const int row = warp * 32 + 16 * tt + g + 8 * (j >> 1);
                    if (m < p.M) part[m * kSmRows + row] = yacc[tt][nt][j];
                }
    }

    if (nsl == 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < p.M * kSmRows; i += blockDim.x) {
            const int m = i / kSmRows, row = rb * kSmRows + (i - m * kSmRows);
            if (row < p.N) yout[(size_t)m * p.N + row] = part[i];
        }
        return;
    }
    // rank q owns entries [q*per, (q+1)*per) of part and adds them up over
    // all ranks, in rank order.
    const int tot = p.M * kSmRows, per = (tot + nsl - 1) / nsl;
    if (p.push) {
        // every slice pushes its partial sums of q's share into rank q's
        // recv[slice] before one cluster barrier (release / acquire); nothing
        // reads another CTA's shared memory after it, so each CTA may then
        // finish on its own
        float *recv = part + p.M * kSmRows;
        __syncthreads();  // part[] is complete
        for (int q = 0; q < nsl; ++q)
            for (int j = threadIdx.x; j < per && q * per + j < tot; j += blockDim.x)
                sm_st_peer(recv + slice * per + j, (unsigned)q, part[q * per + j]);
        sm_cluster_sync();
        for (int j = threadIdx.x; j < per && slice * per + j < tot; j += blockDim.x) {
            float sum = 0.f;
            for (int q = 0; q < nsl; ++q) sum += recv[q * per + j];
            const int i = slice * per + j, m = i / kSmRows, row = rb * kSmRows + (i - m * kSmRows);
            if (row < p.N) yout[(size_t)m * p.N + row] = sum;
        }
        return;
    }
    // otherwise (the receive buffer would cost residency) rank q reads the
    // peers' part[] after one barrier, and a second keeps it alive until all
    // ranks have read it
    sm_cluster_sync();
    for (int i = slice * per + threadIdx.x; i < min(tot, (slice + 1) * per); i += blockDim.x) {
        float v[kSmMaxCluster];
#pragma unroll
        for (int q = 0; q < kSmMaxCluster; ++q) v[q] = q < nsl ? sm_ld_peer(part + i, (unsigned)q) : 0.f;
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < kSmMaxCluster; ++q) sum += v[q];
        const int m = i / kSmRows, row = rb * kSmRows + (i - m * kSmRows);
        if (row < p.N) yout[(size_t)m * p.N + row] = sum;
    }
    sm_cluster_sync();
}

struct SmPlan {
    int nsteps, L, S, blocks, NT;
    bool push;
    size_t smem;
    bool ok;
};

// fmt: 1 = Q1_0_g128 (256 k per step), 3 = INT4_G64 (128 k per step); R
// matrices of one launch (blocks counts the row blocks of all of them)
static SmPlan sm_plan(int fmt, int M, int N, int K, int sms, int R = 1)
{
    SmPlan P = {};
    const int stepk = fmt == 1 ? kSmStepK : kI4sStepK, maxm = fmt == 1 ? kSmMaxM : kI4sMaxM;
    P.NT = (M + 7) / 8;
    P.nsteps = K / stepk;
    P.blocks = (N + kSmRows - 1) / kSmRows * R;
    if (M < 2 || M > maxm || N < 1 || K % stepk != 0 || P.nsteps < 1 || R < 1 || R > kSmMaxR) return P;
    const size_t ring = (size_t)kSmWarps * kSmWStages * (fmt == 1 ? kSmStageBytes : kI4sStageBytes);
    // the partial sums; with push, the peers' pushed partial sums after them
    // (up to S - 1 entries more).  Pushing was measured faster up to M = 8
    // (Q1_0_g128 5120x5120: 7.7 -> 7.2 us) and slower above (INT4_G64
    // 11008x4096 M=32: 23.5 -> 26.6 us, about 4096 remote stores per CTA), so
    // it is taken for M <= 8, where it also costs no residency
    const size_t base = 128 /*alignment*/ + sg_xring_bytes(fmt, kSmSlots, P.NT) + ring + (size_t)M * kSmRows * 4;
    const size_t with_recv = base + ((size_t)M * kSmRows + kSmMaxCluster) * 4;
    // CTAs resident per SM (shared memory, with 1 KB reserved per CTA, and registers)
    auto resident_at = [&](size_t smem) {
        return (int)std::max<size_t>(1, std::min<size_t>(sm_min_blocks(fmt, P.NT), (228 * 1024) / (smem + 1024)));
    };
    P.push = M <= 8 && with_recv <= (size_t)kSmMaxSmem && resident_at(with_recv) >= resident_at(base);
    P.smem = P.push ? with_recv : base;
    const int resident = resident_at(P.smem);
    // K slices: as many as keep every CTA resident in one wave
    P.S = (int)std::min<long long>(std::min(kSmMaxCluster, P.nsteps),
                                   std::max<long long>(1, (long long)resident * sms / P.blocks));
    P.L = (P.nsteps + P.S - 1) / P.S;
    P.S = (P.nsteps + P.L - 1) / P.L;
    P.ok = P.smem <= (size_t)kSmMaxSmem && P.blocks < 65536;
    return P;
}

bool q1sm_supported(int M, int N, int K) { return sm_plan(1, M, N, K, sm_num_sms()).ok; }
bool i4sm_supported(int M, int N, int K) { return sm_plan(3, M, N, K, sm_num_sms()).ok; }

// R <= kSmMaxR matrices of one shape that read one x, one launch
static lowbit_status sm_launch(int fmt, const uint8_t *const *bits, const uint16_t *const *scales, const uint16_t *x,
                               float *const *y, int R, int M, int N, int K, cudaStream_t st)
{
    const SmPlan P = sm_plan(fmt, M, N, K, sm_num_sms(), R);
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap xmap;
    if (!sg_xmap(&xmap, fmt, true, x, M, K)) return LOWBIT_ERR_CUDA;
    SmParams p = {};
    for (int r = 0; r < R; ++r) {
        p.bits[r] = bits[r];
        p.scales[r] = scales[r];
        p.y[r] = y[r];
    }
    p.M = M;
    p.N = N;
    p.K = K;
    p.nsteps = P.nsteps;
    p.L = P.L;
    p.blocks = P.blocks / R;
    p.push = P.push ? 1 : 0;
    void (*kern)(const CUtensorMap, const SmParams);
    if (fmt == 1)
        kern = P.NT == 1 ? k_smallm<1, 1> : k_smallm<1, 2>;
    else
        kern = P.NT == 1 ? k_smallm<3, 1> : P.NT == 2 ? k_smallm<3, 2> : P.NT == 3 ? k_smallm<3, 3> : k_smallm<3, 4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.S, P.blocks);
    cfg.blockDim = dim3(kSmThreads);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = P.S;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, xmap, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q1sm_launch(const uint8_t *bits, const uint16_t *scales, const uint16_t *x, float *y, int M, int N,
                          int K, cudaStream_t st)
{
    return sm_launch(1, &bits, &scales, x, &y, 1, M, N, K, st);
}

lowbit_status i4sm_launch(const uint8_t *q, const uint16_t *scales, const uint16_t *x, float *y, int M, int N, int K,
                          cudaStream_t st)
{
    return sm_launch(3, &q, &scales, x, &y, 1, M, N, K, st);
}

// R matrices in launches of up to kSmMaxR
lowbit_status smr_launch(int fmt, const uint8_t *const *bits, const uint16_t *const *scales, const uint16_t *x,
                         float *const *y, int R, int M, int N, int K, cudaStream_t st)
{
    for (int r0 = 0; r0 < R; r0 += kSmMaxR) {
        const lowbit_status s =
            sm_launch(fmt, bits + r0, scales + r0, x, y + r0, std::min(kSmMaxR, R - r0), M, N, K, st);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

// ---------------------------------------------------------------------------
// grouped persistent form: R matrices of one shape that read one x (M >= 2)
// ---------------------------------------------------------------------------

constexpr int kSgMaxGroup = 256;
constexpr int kSgMaxWarps = 15;  // consumer warps (16 warps with the producer: 128 registers each)
constexpr int kSgMinWarps = 8;
// consumer warps an instance may have: 11 for the INT4_G64 instances with
// three or four batch tiles (12 warps: 170 registers each), else kSgMaxWarps
__host__ __device__ constexpr int sg_max_warps(int fmt, int NT) { return fmt == 3 && NT >= 3 ? 11 : kSgMaxWarps; }
// Ring depths (compile-time knobs; the defaults are the measured best).
#ifndef LOWBIT_SG_SLOTS
#define LOWBIT_SG_SLOTS 6
#endif
#ifndef LOWBIT_SG_RAW
#define LOWBIT_SG_RAW 3
#endif
#ifndef LOWBIT_SG_WSTAGES
#define LOWBIT_SG_WSTAGES 3
#endif
constexpr int kSgSlots = LOWBIT_SG_SLOTS;      // x ring depth, in steps
constexpr int kSgRaw = LOWBIT_SG_RAW;          // raw ring depth (Q1_0_g128), in steps
constexpr int kSgWStages = LOWBIT_SG_WSTAGES;  // weight ring depth per warp, in steps

struct SmGroup {
    const uint8_t *bits[kSgMaxGroup];
    const uint16_t *scales[kSgMaxGroup];
    float *y[kSgMaxGroup];
};

struct SmGParams {
    int M, N, K, nsteps, blocksN, nblocks, rounds;
};

template <int FMT, int NT, int KF = 0>
__global__ void __launch_bounds__((sg_max_warps(FMT, NT) + 1) * 32, 1) k_smallm_grp(const __grid_constant__ SmGroup grp,
                                                                 const __grid_constant__ CUtensorMap xmap,
                                                                 const SmGParams q)
{
    constexpr int kSB = SgFmt<FMT>::kStageBytes;
    constexpr int kXSlot = 8 * NT * sg_xrow(FMT);
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bars[2 * kSgSlots + kSgRaw];  // full[s], empty[s], raw[s]
    __shared__ uint32_t multab[4][4];
    uint64_t *full = bars, *empty = bars + kSgSlots, *rawbar = bars + 2 * kSgSlots;
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x >> 5) - 1;
    const int total = q.rounds * q.nsteps;  // (round, step) sequence of every warp
    uint8_t *raw = smem;
    uint8_t *xring = raw + sg_raw_bytes(FMT, kSgRaw, q.M);
    sg_setup<FMT, NT, kSgSlots, kSgRaw>(xring, full, empty, rawbar, multab, q.M, nw);

    if (warp == nw) {
        sg_produce<FMT, NT, kSgSlots, kSgRaw, false>(&xmap, raw, xring, full, empty, rawbar, q.M, total, 0, q.nsteps,
                                                     lane);
        return;
    }

    // ---- consumers
    uint8_t *wring = xring + sg_xring_bytes(FMT, kSgSlots, NT) + (size_t)warp * kSgWStages * kSB;
    const unsigned wr_s = (unsigned)__cvta_generic_to_shared(wring);
    uint32_t mul[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mul[i] = multab[lane & 3][i];

    // copy cursor: the (round, step) whose weights go out next
    SgCopy<FMT, KF> cp;
    int cj = 0, cs = 0, cstage = 0;
    bool clive = false;
    auto set_round = [&](int j) {
        cj = j;
        cs = 0;
        const int b = (j * (int)gridDim.x + (int)blockIdx.x) * nw + warp;
        clive = j < q.rounds && b < q.nblocks;
        if (!clive) return;
        const int r = b / q.blocksN, blk = b - r * q.blocksN;
        cp.set(grp.bits[r], grp.scales[r], blk, q.N, q.K, lane);
    };
    auto issue_next = [&]() {  // one commit group per call, empty past the end
        if (clive) cp.issue(wr_s + cstage * kSB, cs, grp.bits[0]);
        sm_commit();
        cstage = cstage + 1 == kSgWStages ? 0 : cstage + 1;
        if (++cs == q.nsteps) set_round(cj + 1);
    };
    set_round(0);
#pragma unroll
    for (int t = 0; t < kSgWStages - 1; ++t) issue_next();
    pdl_wait_primary();  // y was last read by earlier kernels

    float yacc[2][NT][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
    const int g = lane >> 2, t4 = lane & 3;
    int sl = 0, stage = 0, s = 0;
    unsigned phase = 0;
    int b = blockIdx.x * nw + warp;  // block of the current round
    for (int u = 0; u < total; ++u) {
        issue_next();
        if (!__all_sync(0xffffffffu, sg_wait(full + sl, phase))) break;
        sm_wait<kSgWStages - 1>();  // this lane's copies of step u landed
        __syncwarp();               // ... and every lane's
        if (b < q.nblocks) {
            if (FMT == 1)
                sg_consume_q1<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, mul, yacc);
            else
                sg_consume_i4p<NT>(wring + stage * kSB, xring + sl * kXSlot, lane, yacc);
        }
        __syncwarp();  // every lane has read the slot and the stage
        if (lane == 0) mbar_arrive(empty + sl);
        if (++sl == kSgSlots) {
            sl = 0;
            phase ^= 1u;
        }
        stage = stage + 1 == kSgWStages ? 0 : stage + 1;
        if (++s == q.nsteps) {
            if (b < q.nblocks) {
                const int r = b / q.blocksN, blk = b - r * q.blocksN;
                float *y = grp.y[r];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int m = 8 * nt + 2 * t4 + (e & 1);
                            const int row = blk * 32 + 16 * tt + g + 8 * (e >> 1);
                            if (m < q.M && row < q.N) y[(size_t)m * q.N + row] = yacc[tt][nt][e];
                        }
            }
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    yacc[tt][nt][0] = yacc[tt][nt][1] = yacc[tt][nt][2] = yacc[tt][nt][3] = 0.f;
            s = 0;
            b += (int)gridDim.x * nw;
        }
    }
    sm_wait<0>();
}

struct SgPlan {
    int nsteps, blocksN, nblocks, warps, rounds, NT;
    size_t smem;
    bool ok;
};

// Consumer warps per CTA: as many as fit (<= kSgMaxWarps), then the count in
// [kSgMinWarps, max] whose rounds come out fullest (ties: more warps).
static SgPlan sg_plan(int fmt, int R, int M, int N, int K, int sms)
{
    SgPlan P = {};
    const int stepk = fmt == 1 ? kSmStepK : kI4sStepK, maxm = fmt == 1 ? kSmMaxM : kI4sMaxM;
    if (R < 1 || R > kSgMaxGroup || M < 2 || M > maxm || N < 1 || K % stepk != 0 || K < stepk) return P;
    P.NT = (M + 7) / 8;
    P.nsteps = K / stepk;
    P.blocksN = (N + 31) / 32;
    P.nblocks = R * P.blocksN;
    const size_t xring = 128 /*alignment*/ + sg_raw_bytes(fmt, kSgRaw, M) + sg_xring_bytes(fmt, kSgSlots, P.NT);
    const size_t per_warp = (size_t)kSgWStages * (fmt == 1 ? kSmStageBytes : kI4sStageBytes);
    if (xring + kSgMinWarps * per_warp > (size_t)kSmMaxSmem) return P;
    const int fit = (int)std::min<size_t>(sg_max_warps(fmt, P.NT), ((size_t)kSmMaxSmem - xring) / per_warp);
    double best = -1.0;
    for (int w = fit; w >= kSgMinWarps; --w) {
        if ((long long)P.nblocks < (long long)sms * w) continue;  // at least one full round
        const int rounds = (int)((P.nblocks + (long long)sms * w - 1) / ((long long)sms * w));
        const double eff = (double)P.nblocks / ((double)rounds * sms * w);
        if (eff > best + 1e-9) {
            best = eff;
            P.warps = w;
            P.rounds = rounds;
        }
    }
    P.smem = xring + (size_t)P.warps * per_warp;
    P.ok = P.warps >= kSgMinWarps;
    return P;
}

bool smg_supported(int fmt, int R, int M, int N, int K) { return sg_plan(fmt, R, M, N, K, sm_num_sms()).ok; }

lowbit_status smg_launch(int fmt, const uint8_t *const *bits, const uint16_t *const *scales, const uint16_t *x,
                         float *const *y, int R, int M, int N, int K, cudaStream_t st)
{
    const int sms = sm_num_sms();
    const SgPlan P = sg_plan(fmt, R, M, N, K, sms);
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap xmap;
    if (!sg_xmap(&xmap, fmt, false, x, M, K)) return LOWBIT_ERR_CUDA;
    static SmGroup grp;  // large: kept off the stack
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int r = 0; r < R; ++r) {
        grp.bits[r] = bits[r];
        grp.scales[r] = scales[r];
        grp.y[r] = y[r];
    }
    SmGParams q = {};
    q.M = M;
    q.N = N;
    q.K = K;
    q.nsteps = P.nsteps;
    q.blocksN = P.blocksN;
    q.nblocks = P.nblocks;
    q.rounds = P.rounds;
    void (*kern)(const SmGroup, const CUtensorMap, const SmGParams);
    if (fmt == 1)
        kern = P.NT == 1     ? k_smallm_grp<1, 1>
               : K == 5120  ? k_smallm_grp<1, 2, 5120>
               : K == 17408 ? k_smallm_grp<1, 2, 17408>
                            : k_smallm_grp<1, 2>;
    else
        kern = P.NT == 1 ? k_smallm_grp<3, 1>
             : P.NT == 2 ? k_smallm_grp<3, 2>
             : P.NT == 3 ? k_smallm_grp<3, 3>
             : K == 4096 ? k_smallm_grp<3, 4, 4096>
                         : k_smallm_grp<3, 4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3((P.warps + 1) * 32);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, grp, xmap, q);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// Read and clear the fault flag of the current device.
int smg_fault_flag()
{
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_sg_fault, sizeof(v)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_sg_fault, &zero, sizeof(zero));
    return v != 0;
}

}  // namespace lowbit
