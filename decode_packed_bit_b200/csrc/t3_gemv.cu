// t3_gemv.cu -- ternary weights with an FP16 scale per 128 (base-3 bytes):
// packer, unpacker and the matrix-vector product.
//
// Format ("Bonsai-27B-gguf technical white paper digest": the ternary 27B
// model is 5.9 GB where the 1.125-bit one is 3.79 GB, i.e. 1.75 bits per
// weight; the page gives no layout, this is the library's reading): w in
// {-1, 0, +1}, t = w + 1; the 128 trits of a group of one row are packed five
// per byte in base 3 -- byte j < 25 of the group holds k = 5j .. 5j+4 as
// sum_i t_i 3^i, byte 25 holds k = 125..127 -- so a group is 26 bytes; one
// FP16 scale per group.  Row n: bytes [n][26 K/128], scales [n][K/128].
//     y[m][n] = sum_g d[n][g] * sum_{k in g} w[n][k] * x[m][k].
//
// The product (k_t3_m1, M = 1, K % 1024 == 0): a warp takes 32 rows, lane l
// reads row l, so every value of x a step needs is the same for the whole
// warp and is read from shared memory once per warp (a broadcast).  x is
// rewritten once per CTA, per 128-group, as exact integers: X_k = round(x_k
// 2^(22 - E_g)) with 2^(E_g - 2) <= max|x_g| < 2^(E_g - 1), so |X| < 2^21,
// split into three signed bytes X = L0 + 256 L1 + 65536 L2.  A packed byte's
// first four trits come from a table (byte -> four trit bytes; one copy per
// lane, so the lookups never share a bank), the fifth from floor(b / 81) =
// (b * 203) >> 14 computed for two bytes at once in 16-bit lanes.  dp4a
// (unsigned trits x signed limbs) sums t X exactly in int32 per group; the
// epilogue per group adds d * 2^(E - 22) * (sum t X - sum X), since w = t - 1.
// Integer-exact up to the 22-bit rounding of x and the fp32 epilogue.
#include <algorithm>

#include "common.cuh"

namespace lowbit {

constexpr int kT3GroupBytes = 26;
constexpr int kT3UnitGroups = 8;                       // 1024 k per step
constexpr int kT3UnitBytes = kT3UnitGroups * kT3GroupBytes;   // 208 = 13 x 16
constexpr int kT3StepRows = 32;
constexpr int kT3StageW = kT3StepRows * kT3UnitBytes;  // rows 208 bytes apart: 13 r mod 8 is a permutation,
                                                      // so a quarter-warp's 16-byte reads use every bank once
constexpr int kT3StageBytes = kT3StageW + kT3StepRows * 16;   // + eight fp16 scales per row
constexpr int kT3LutBytes = 256 * 32 * 4;             // byte -> trits 0..3, one copy per lane
constexpr int kT3MaxSmem = 226 * 1024;
constexpr int kT3MaxGroup = 256;
constexpr int kT3MinExp = -96;

struct T3Group {
    const uint8_t *w[kT3MaxGroup];
    const uint16_t *s[kT3MaxGroup];
    float *y[kT3MaxGroup];
};

struct T3Params {
    const uint16_t *x;
    int R, N, K;
    int blocksN;       // 32-row blocks per matrix
    int cells;         // R * blocksN
    int slices;        // K slices per cell (partial sums added with atomics when > 1)
    int units;         // 1024-k steps per row
    int stages;
    int tab_off, tabB_off, gtab_off, ring_off;   // shared-memory offsets
};

// digit i of b in base 3 (any byte value: floor(b / 3^i) mod 3)
__host__ __device__ __forceinline__ int t3_digit(int b, int i)
{
    for (int j = 0; j < i; ++j) b /= 3;
    return b % 3;
}

// ---------------------------------------------------------------------------
// pack / unpack: one thread per packed byte
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) k_pack_t3(const int8_t *__restrict__ codes, uint8_t *__restrict__ packed,
                                                 int64_t rows, int64_t cols)
{
    const int64_t rb = 26 * (cols / 128);
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * rb) return;
    const int64_t r = i / rb, p = i - r * rb, g = p / 26, j = p - g * 26;
    const int8_t *c = codes + r * cols + 128 * g + 5 * j;
    const int n = j < 25 ? 5 : 3;
    int v = 0, pw = 1;
    for (int t = 0; t < n; ++t) {
        const int w = max(-1, min(1, (int)c[t]));   // codes outside {-1, 0, 1} are clamped
        v += (w + 1) * pw;
        pw *= 3;
    }
    packed[i] = (uint8_t)v;
}

__global__ void __launch_bounds__(256) k_unpack_t3(const uint8_t *__restrict__ packed, int8_t *__restrict__ codes,
                                                   int64_t rows, int64_t cols)
{
    const int64_t rb = 26 * (cols / 128);
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * rb) return;
    const int64_t r = i / rb, p = i - r * rb, g = p / 26, j = p - g * 26;
    int8_t *c = codes + r * cols + 128 * g + 5 * j;
    const int n = j < 25 ? 5 : 3;
    const int b = packed[i];
    for (int t = 0; t < n; ++t) c[t] = (int8_t)(t3_digit(b, t) - 1);
}

lowbit_status t3_pack_launch(const int8_t *codes, int64_t rows, int64_t cols, uint8_t *packed, cudaStream_t st)
{
    const int64_t n = rows * 26 * (cols / 128);
    if (n == 0) return LOWBIT_OK;
    k_pack_t3<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(codes, packed, rows, cols);
    return launch_status();
}

lowbit_status t3_unpack_launch(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *codes, cudaStream_t st)
{
    const int64_t n = rows * 26 * (cols / 128);
    if (n == 0) return LOWBIT_OK;
    k_unpack_t3<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(packed, codes, rows, cols);
    return launch_status();
}

// ---------------------------------------------------------------------------
// the streaming product, M = 1
// ---------------------------------------------------------------------------

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// floor(b / 81) of each byte of w (bytes below 243): the fifth trit.  In
// 16-bit lanes b * 203 < 2^16, and (b * 203) >> 14 = floor(b / 81) for every
// b < 243.
__device__ __forceinline__ uint32_t t3_fifth_trits(uint32_t w)
{
    const uint32_t e = prmt(w, 0u, 0x4240u);   // bytes 0 and 2 in 16-bit lanes
    const uint32_t o = prmt(w, 0u, 0x4341u);   // bytes 1 and 3
    const uint32_t te = ((e * 203u) >> 14) & 0x00030003u;
    const uint32_t to = ((o * 203u) >> 14) & 0x00030003u;
    return prmt(te, to, 0x6240u);
}

__device__ __forceinline__ float t3_pow2(int e) { return __int_as_float((e + 127) << 23); }

// The x tables of one CTA (M = 1).  Group g: E_g, c_g = 2^(E_g - 22), SX_g =
// sum_k X_k.  Byte position p = 26 g + j of a row covers k = 128 g + 5 j + i:
// tabA[p] = {L0, L1, L2} of slots i = 0..3 (one byte each), tabB[p / 4] byte
// p % 4 = {L0, L1, L2} of slot 4.  Slots past the group (j = 25, i = 3, 4)
// hold 0.
__device__ void t3_build_tables(const uint16_t *__restrict__ x, int K, uint4 *tabA, uint4 *tabB, float2 *gtab)
{
    const int G = K >> 7, lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int *Eg = reinterpret_cast<int *>(gtab + G);
    for (int g = warp; g < G; g += nw) {
        float v[4], m = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[q] = bf16_bits_to_float(x[128 * g + 32 * q + lane]);
            m = fmaxf(m, fabsf(v[q]));
        }
        m = warp_max_nonneg(m);
        const int e8 = (int)((__float_as_uint(m) >> 23) & 0xFFu);
        const int E = max(e8 == 0 ? kT3MinExp : e8 - 125, kT3MinExp);   // 2^(E-2) <= m < 2^(E-1)
        int s = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) s += __float2int_rn(v[q] * t3_pow2(22 - E));
        s = warp_sum_int(s);
        if (lane == 0) {
            gtab[g] = make_float2(t3_pow2(E - 22), __int_as_float(s));
            Eg[g] = E;
        }
    }
    __syncthreads();
    const int P = 26 * G;
    uint8_t *tb = reinterpret_cast<uint8_t *>(tabB);
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int g = p / 26, j = p - 26 * g, E = Eg[g];
        uint32_t l[3][5] = {};
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            if (j < 25 || i < 3) {
                const int X = __float2int_rn(bf16_bits_to_float(x[128 * g + 5 * j + i]) * t3_pow2(22 - E));
                const int l0 = (int)(int8_t)(X & 0xFF);
                const int r = (X - l0) >> 8;
                const int l1 = (int)(int8_t)(r & 0xFF);
                const int l2 = (r - l1) >> 8;   // |X| < 2^21 keeps it in [-32, 32]
                l[0][i] = (uint32_t)(uint8_t)l0;
                l[1][i] = (uint32_t)(uint8_t)l1;
                l[2][i] = (uint32_t)(uint8_t)l2;
            }
        }
        uint32_t a[3];
#pragma unroll
        for (int t = 0; t < 3; ++t) a[t] = l[t][0] | (l[t][1] << 8) | (l[t][2] << 16) | (l[t][3] << 24);
        tabA[p] = make_uint4(a[0], a[1], a[2], 0u);
#pragma unroll
        for (int t = 0; t < 3; ++t) tb[16 * (p >> 2) + 4 * t + (p & 3)] = (uint8_t)l[t][4];
        if ((p & 3) == 0) tb[16 * (p >> 2) + 12] = tb[16 * (p >> 2) + 13] = tb[16 * (p >> 2) + 14] =
            tb[16 * (p >> 2) + 15] = 0;
    }
}

__device__ __forceinline__ void t3_cp16(unsigned dst, const void *src, bool ok)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0) : "memory");
}
__device__ __forceinline__ void t3_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void t3_wait(int n)
{
    // the ring depth is a launch parameter: wait for all but n groups (n <= 2)
    if (n >= 2)
        asm volatile("cp.async.wait_group 2;" ::: "memory");
    else if (n == 1)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Lane l's contribution of one byte of its row: trits 0..3 from the table,
// limbs of the byte's position from tabA.
__device__ __forceinline__ void t3_byte(uint32_t b, const uint32_t *lut_lane, const uint4 &ta, int (&acc)[3])
{
    const uint32_t t = lut_lane[b << 5];
    acc[0] = dp4a_us(t, ta.x, acc[0]);
    acc[1] = dp4a_us(t, ta.y, acc[1]);
    acc[2] = dp4a_us(t, ta.z, acc[2]);
}

#ifndef LOWBIT_T3_MAX_WARPS
#define LOWBIT_T3_MAX_WARPS 12
#endif
constexpr int kT3MaxWarps = LOWBIT_T3_MAX_WARPS;

__global__ void __launch_bounds__(kT3MaxWarps * 32, 1) k_t3_m1(const __grid_constant__ T3Group grp, const T3Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    const uint4 *tabA = reinterpret_cast<const uint4 *>(smem + p.tab_off);
    const uint4 *tabB = reinterpret_cast<const uint4 *>(smem + p.tabB_off);
    const float2 *gtab = reinterpret_cast<const float2 *>(smem + p.gtab_off);
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int S = p.stages;
    uint8_t *ring = smem + p.ring_off + (size_t)warp * S * kT3StageBytes;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);
    const size_t rowbytes = (size_t)26 * (p.K >> 7);
    const int G = p.K >> 7;
    const int upc = p.units / p.slices;          // units per work item
    // 32-bit item indices (the planner keeps cells * slices below 2^31): a
    // 64-bit division per step is a long software routine
    const int items = p.cells * p.slices;
    const int gw = blockIdx.x * nw + warp, gstride = gridDim.x * nw;

    // issue side: step s of this warp's items, in order
    int is_item = gw;
    int is_u = 0, is_slot = 0;
    auto issue_next = [&]() {
        if (is_item < items) {
            const int cell = is_item / p.slices, sl = is_item - cell * p.slices;
            const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
            const int u = sl * upc + is_u;
            const unsigned st = ring_s + is_slot * kT3StageBytes;
#pragma unroll
            for (int i = 0; i < 13; ++i) {
                const int q = i * 32 + lane, row = q / 13, col = q - 13 * row;
                const int n = blk * kT3StepRows + row;
                const bool ok = n < p.N;
                t3_cp16(st + row * kT3UnitBytes + col * 16,
                        ok ? grp.w[r] + (size_t)n * rowbytes + (size_t)u * kT3UnitBytes + col * 16 : grp.w[r], ok);
            }
            const int n = blk * kT3StepRows + lane;
            const bool ok = n < p.N;
            t3_cp16(st + kT3StageW + lane * 16, ok ? grp.s[r] + (size_t)n * G + 8 * u : grp.s[r], ok);
            if (++is_u == upc) {
                is_u = 0;
                is_item += gstride;
            }
        }
        t3_commit();
        is_slot = is_slot + 1 == S ? 0 : is_slot + 1;
    };
    for (int t = 0; t < S - 1; ++t) issue_next();

    // the byte table and the x tables
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const int b = i >> 5;
        lut[i] = (uint32_t)t3_digit(b, 0) | ((uint32_t)t3_digit(b, 1) << 8) | ((uint32_t)t3_digit(b, 2) << 16) |
                 ((uint32_t)t3_digit(b, 3) << 24);
    }
    pdl_wait_primary();   // x and the outputs follow stream order from here
    t3_build_tables(p.x, p.K, reinterpret_cast<uint4 *>(smem + p.tab_off), reinterpret_cast<uint4 *>(smem + p.tabB_off),
                    reinterpret_cast<float2 *>(smem + p.gtab_off));
    __syncthreads();

    const uint32_t *lut_lane = lut + lane;
    int slot = 0;
    for (int item = gw; item < items; item += gstride) {
        const int cell = item / p.slices, sl = item - cell * p.slices;
        const int r = cell / p.blocksN, blk = cell - r * p.blocksN;
        float yacc = 0.f;
        for (int uu = 0; uu < upc; ++uu) {
            const int u = sl * upc + uu;
            issue_next();
            t3_wait(S - 1);
            __syncwarp();
            const uint8_t *st = ring + slot * kT3StageBytes;
            // this lane's row: 8 fp16 scales, then one group pair (52 bytes)
            // at a time from the 16-word window that holds it
            const uint8_t *row = st + lane * kT3UnitBytes;
            const uint4 sc4 = *reinterpret_cast<const uint4 *>(st + kT3StageW + lane * 16);
            const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
            const int p0 = u * kT3UnitBytes;    // first byte position of the unit in the row
#pragma unroll
            for (int q = 0; q < 4; ++q) {       // group pairs 2q, 2q + 1
                constexpr int kBase[4] = {0, 12, 24, 36};   // 16-byte aligned window of words 13q .. 13q+12
                uint32_t wv[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + 4 * kBase[q] + 16 * c);
                    wv[4 * c] = v.x;
                    wv[4 * c + 1] = v.y;
                    wv[4 * c + 2] = v.z;
                    wv[4 * c + 3] = v.w;
                }
                const int off = 13 * q - kBase[q];
                int accA[3] = {0, 0, 0}, accB[3] = {0, 0, 0};
#pragma unroll
                for (int w = 0; w < 13; ++w) {
                    const uint32_t word = wv[off + w];
                    const int pw = p0 + 52 * q + 4 * w;           // position of the word's first byte
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 ta = tabA[pw + i];
                        const uint32_t b = (word >> (8 * i)) & 0xFFu;
                        if (4 * w + i < 26)
                            t3_byte(b, lut_lane, ta, accA);
                        else
                            t3_byte(b, lut_lane, ta, accB);
                    }
                    const uint32_t f = t3_fifth_trits(word);
                    const uint4 tb = tabB[pw >> 2];
                    if (w < 6) {
                        accA[0] = dp4a_us(f, tb.x, accA[0]);
                        accA[1] = dp4a_us(f, tb.y, accA[1]);
                        accA[2] = dp4a_us(f, tb.z, accA[2]);
                    } else if (w > 6) {
                        accB[0] = dp4a_us(f, tb.x, accB[0]);
                        accB[1] = dp4a_us(f, tb.y, accB[1]);
                        accB[2] = dp4a_us(f, tb.z, accB[2]);
                    } else {   // bytes 24, 25 end group 2q, bytes 26, 27 start group 2q + 1
                        const uint32_t fa = f & 0x0000FFFFu, fb = f & 0xFFFF0000u;
                        accA[0] = dp4a_us(fa, tb.x, accA[0]);
                        accA[1] = dp4a_us(fa, tb.y, accA[1]);
                        accA[2] = dp4a_us(fa, tb.z, accA[2]);
                        accB[0] = dp4a_us(fb, tb.x, accB[0]);
                        accB[1] = dp4a_us(fb, tb.y, accB[1]);
                        accB[2] = dp4a_us(fb, tb.z, accB[2]);
                    }
                }
                // sum t X = acc0 + 256 acc1 + 65536 acc2 < 2^30 in magnitude; minus sum X
                const int g0 = 8 * u + 2 * q;
                const float2 ga = gtab[g0], gb = gtab[g0 + 1];
                const int va = accA[0] + 256 * accA[1] + 65536 * accA[2] - __float_as_int(ga.y);
                const int vb = accB[0] + 256 * accB[1] + 65536 * accB[2] - __float_as_int(gb.y);
                const uint32_t sp = scw[q];
                const float da = f16_bits_to_float((uint16_t)(sp & 0xFFFFu));
                const float db = f16_bits_to_float((uint16_t)(sp >> 16));
                yacc = fmaf(da * ga.x, (float)va, yacc);
                yacc = fmaf(db * gb.x, (float)vb, yacc);
            }
            __syncwarp();   // every lane is done with the stage before it is refilled
            slot = slot + 1 == S ? 0 : slot + 1;
        }
        const int n = blk * kT3StepRows + lane;
        if (n < p.N) {
            if (p.slices == 1)
                grp.y[r][n] = yacc;
            else
                atomicAdd(grp.y[r] + n, yacc);
        }
    }
    t3_wait(0);
}

// ---------------------------------------------------------------------------
// any shape (K % 128 == 0, 1 <= M <= 16): one warp per output row, plain
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) k_t3_gemv_simt(const uint8_t *__restrict__ w, const uint16_t *__restrict__ s,
                                                      const uint16_t *__restrict__ x, float *__restrict__ y, int M,
                                                      int N, int K)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    pdl_wait_primary();
    if (n >= N) return;
    const int P = 26 * (K >> 7);
    const uint8_t *row = w + (size_t)n * P;
    for (int m = 0; m < M; ++m) {
        const uint16_t *xm = x + (size_t)m * K;
        float acc = 0.f;
        for (int pos = lane; pos < P; pos += 32) {
            const int g = pos / 26, j = pos - 26 * g;
            int b = row[pos];
            float part = 0.f;
            const int cnt = j < 25 ? 5 : 3;
            for (int i = 0; i < cnt; ++i) {
                const int t = b % 3;
                b /= 3;
                part += (float)(t - 1) * bf16_bits_to_float(xm[128 * g + 5 * j + i]);
            }
            acc = fmaf(f16_bits_to_float(s[(size_t)n * (K >> 7) + g]), part, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) y[(size_t)m * N + n] = acc;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static int t3_num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

struct T3Plan {
    bool ok;
    int warps, stages, slices, grid;
    size_t smem;
    int tab_off, tabB_off, gtab_off, ring_off;
};

// The streaming kernel: M = 1, K % 1024 == 0; shared memory holds the byte
// table, the x tables (about 17 bytes per k) and every warp's ring.
static T3Plan t3_plan(int R, int N, int K, int sms)
{
    T3Plan P = {};
    if (K % 1024 != 0 || K <= 0 || N <= 0 || R < 1 || R > kT3MaxGroup) return P;
    const int G = K / 128, Pn = 26 * G;
    P.tab_off = kT3LutBytes;
    P.tabB_off = P.tab_off + 16 * Pn;
    P.gtab_off = P.tabB_off + 16 * (Pn / 4);
    P.ring_off = (int)align256((size_t)P.gtab_off + 12u * G);
    const size_t left = P.ring_off < kT3MaxSmem ? kT3MaxSmem - P.ring_off : 0;
    // as many warps as fit (at most kT3MaxWarps), each with three stages if
    // they fit, else two
    for (int w = kT3MaxWarps; w >= 4 && !P.ok; --w)
        for (int st = 3; st >= 2; --st)
            if ((size_t)w * st * kT3StageBytes <= left) {
                P.warps = w;
                P.stages = st;
                P.ok = true;
                break;
            }
    if (!P.ok) return P;
    P.smem = (size_t)P.ring_off + (size_t)P.warps * P.stages * kT3StageBytes;
    const long long cells = (long long)R * ((N + kT3StepRows - 1) / kT3StepRows);
    const long long warps_total = (long long)sms * P.warps;
    // split K when there are too few cells to give every warp two
    int S = 1;
    while (cells * S < 2 * warps_total && S * 2 <= K / 1024 && (K / 1024) % (S * 2) == 0) S *= 2;
    P.slices = S;
    P.grid = (int)std::min<long long>(sms, (cells * S + P.warps - 1) / P.warps);
    if (cells * S >= (1LL << 31)) P.ok = false;  // the kernel indexes items with 32-bit ints
    return P;
}

bool t3_fast_supported(int R, int N, int K) { return t3_plan(R, N, K, t3_num_sms()).ok; }

lowbit_status t3_group_launch(const uint8_t *const *w, const uint16_t *const *s, const uint16_t *x, float *const *y,
                              int R, int N, int K, cudaStream_t st)
{
    const T3Plan P = t3_plan(R, N, K, t3_num_sms());
    if (!P.ok) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    T3Group grp;
    for (int r = 0; r < R; ++r) {
        grp.w[r] = w[r];
        grp.s[r] = s[r];
        grp.y[r] = y[r];
    }
    T3Params p = {};
    p.x = x;
    p.R = R;
    p.N = N;
    p.K = K;
    p.blocksN = (N + kT3StepRows - 1) / kT3StepRows;
    p.cells = R * p.blocksN;
    p.slices = P.slices;
    p.units = K / 1024;
    p.stages = P.stages;
    p.tab_off = P.tab_off;
    p.tabB_off = P.tabB_off;
    p.gtab_off = P.gtab_off;
    p.ring_off = P.ring_off;
    if (P.slices > 1)
        for (int r = 0; r < R; ++r)   // partial sums are added into zeroed outputs
            if (cudaMemsetAsync(y[r], 0, (size_t)N * sizeof(float), st) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (cudaFuncSetAttribute(k_t3_m1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    cudaError_t e = launch_pdl(k_t3_m1, dim3(P.grid), dim3(P.warps * 32), P.smem, st, grp, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status t3_simt_launch(const uint8_t *w, const uint16_t *s, const uint16_t *x, float *y, int M, int N, int K,
                             cudaStream_t st)
{
    cudaError_t e = launch_pdl(k_t3_gemv_simt, dim3((N + 7) / 8), dim3(256), 0, st, w, s, x, y, M, N, K);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace lowbit
