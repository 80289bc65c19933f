// q2_mlp.cu -- the Z80-style 2-bit integer MLP, all layers fused in one kernel.
//
// "Show HN: Z80-uLM, a conversational AI that fits in 40KB":
//   - weights {-2,-1,0,+1} stored as codes 0..3, four per byte, lowest field
//     first (the "unpack 2-bit weight" listing: and 03h / sub 2 / rrca rrca);
//   - 16-bit two's-complement accumulation (the MULADD listing);
//   - an arithmetic shift right by 2 after every layer (the sra h / rr l
//     listing);
//   - ReLU between hidden layers; one output neuron per character, argmax.
//
// A 16-bit register that wraps after every add holds, at the end, the exact
// sum reduced mod 2^16 (reduction mod 2^16 is a ring homomorphism), so each
// dot product is summed exactly in int32 (|w| <= 2, |a| <= 2^15, width <=
// 1024 keeps it below 2^27) and wrapped once.  Everything is integer: the
// result is bit-exact for every input.
//
// Layout: one CTA runs the whole network for kVecs input vectors.  The packed
// weights of every layer are staged once into shared memory as bytes; the
// activations of the CTA's vectors ping-pong between two shared buffers, so
// no intermediate layer output ever leaves the SM.
#include <algorithm>

#include "common.cuh"

namespace lowbit {

constexpr int kQ2MaxLayers = 8;
constexpr int kQ2MaxDim = 1024;
constexpr int kQ2MaxWeightBytes = 96 * 1024;
constexpr int kVecs = 8;

struct Q2Net {
    const uint8_t *w[kQ2MaxLayers];
    int dims[kQ2MaxLayers + 1];
    int woff[kQ2MaxLayers];  // byte offset of layer l in shared memory
    int n_layers;
    int wbytes;              // total packed bytes, multiple of 16
};

__device__ __forceinline__ int q2_code_to_weight(uint32_t byte, int field)
{
    return (int)((byte >> (2 * field)) & 3u) - 2;
}

__global__ void __launch_bounds__(256) k_q2_mlp(Q2Net net, const int16_t *__restrict__ x, int batch,
                                               int16_t *__restrict__ logits, int32_t *__restrict__ argmax)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *wsm = smem;                                              // packed weights
    int16_t *act0 = reinterpret_cast<int16_t *>(smem + net.wbytes);   // [kVecs][kQ2MaxDim]
    int16_t *act1 = act0 + kVecs * kQ2MaxDim;

    pdl_launch_dependents();
    pdl_wait_primary();

    // stage all layers' packed weights (byte copies: a layer's size need not be
    // a multiple of 4)
    for (int l = 0; l < net.n_layers; ++l) {
        const int nbytes = net.dims[l + 1] * (net.dims[l] / 4);
        const uint8_t *src = net.w[l];
        uint8_t *dst = wsm + net.woff[l];
        for (int i = threadIdx.x; i < nbytes; i += blockDim.x) dst[i] = src[i];
    }
    const int v0 = blockIdx.x * kVecs;
    const int nv = min(kVecs, batch - v0);
    const int d0 = net.dims[0];
    for (int i = threadIdx.x; i < kVecs * d0; i += blockDim.x) {
        const int v = i / d0, c = i % d0;
        act0[v * kQ2MaxDim + c] = v < nv ? x[(int64_t)(v0 + v) * d0 + c] : (int16_t)0;
    }
    __syncthreads();

    int16_t *cur = act0, *nxt = act1;
    for (int l = 0; l < net.n_layers; ++l) {
        const int din = net.dims[l], dout = net.dims[l + 1];
        const bool hidden = l < net.n_layers - 1;
        const uint8_t *wl = wsm + net.woff[l];
        const int rowb = din / 4;
        // one thread per (output neuron, vector) pair
        for (int p = threadIdx.x; p < dout * kVecs; p += blockDim.x) {
            const int o = p / kVecs, v = p % kVecs;
            const uint8_t *wr = wl + o * rowb;
            const int16_t *a = cur + v * kQ2MaxDim;
            int32_t acc = 0;
            for (int j = 0; j < rowb; ++j) {
                const uint32_t byte = wr[j];
#pragma unroll
                for (int f = 0; f < 4; ++f) acc += q2_code_to_weight(byte, f) * (int32_t)a[4 * j + f];
            }
            const int16_t wrapped = (int16_t)(uint16_t)(uint32_t)acc;  // mod 2^16
            int16_t z = (int16_t)(wrapped >> 2);                       // arithmetic shift
            if (hidden && z < 0) z = 0;
            nxt[v * kQ2MaxDim + o] = z;
        }
        __syncthreads();
        int16_t *t = cur; cur = nxt; nxt = t;
    }

    const int dl = net.dims[net.n_layers];
    for (int i = threadIdx.x; i < nv * dl; i += blockDim.x) {
        const int v = i / dl, c = i % dl;
        logits[(int64_t)(v0 + v) * dl + c] = cur[v * kQ2MaxDim + c];
    }
    if (argmax != nullptr && threadIdx.x < nv) {
        const int16_t *a = cur + threadIdx.x * kQ2MaxDim;
        int best = 0;
        for (int c = 1; c < dl; ++c)
            if (a[c] > a[best]) best = c;   // strict: the lowest index wins ties
        argmax[v0 + threadIdx.x] = best;
    }
}

// ---------------------------------------------------------------------------
// the same network on the integer tensor cores (layer widths <= 256)
// ---------------------------------------------------------------------------
//
// Persistent CTAs expand every layer's codes once into signed bytes (c - 2)
// in shared memory, row-major, rows padded to 16 and inputs to 32 with zero
// weights.  Vectors go 32 at a time (four 8-column MMA tiles).  An int16
// activation a is held as two byte limbs, lo = a & 0xFF (unsigned) and hi =
// a >> 8 (signed), so a = lo + 256 hi; a layer is two mma.sync m16n8k32 per
// 32 inputs (s8 x u8 for lo, s8 x s8 for hi) and acc = D_lo + 256 D_hi is the
// exact int32 sum (|acc| < 2^27).  The epilogue wraps it to int16, shifts
// right by 2, applies ReLU between hidden layers and writes the next layer's
// limbs; nothing leaves the SM until the logits.

constexpr int kQ2tVecs = 32;        // vectors per tile (4 MMA columns tiles)
constexpr int kQ2tMaxDim = 256;
constexpr int kQ2tPad = 16;         // row padding (bytes): conflict-free fragment reads
constexpr int kQ2tThreads = 256;

struct Q2TNet {
    const uint8_t *w[kQ2MaxLayers];
    int dims[kQ2MaxLayers + 1];
    int rows[kQ2MaxLayers];   // dims[l+1] rounded up to 16
    int cols[kQ2MaxLayers];   // dims[l] rounded up to 32
    int woff[kQ2MaxLayers];   // byte offset of layer l's expanded weights
    int wbytes;
    int n_layers;
};

__device__ __forceinline__ void imma_s8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void imma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kAStride = kQ2tMaxDim + kQ2tPad;

// Activation limb row of vector v: [buffer 2][limb 2][vector 32][kAStride].
__device__ __forceinline__ uint8_t *q2t_limb(uint8_t *abuf, int buf, int l, int v)
{
    return abuf + ((size_t)(buf * 2 + l) * kQ2tVecs + v) * kAStride;
}

// Expand every layer's codes once into signed bytes (c - 2) in shared
// memory; padding rows and columns are 0.  Ends with a CTA barrier.
__device__ __forceinline__ void q2t_expand_weights(const Q2TNet &net, int8_t *wsm)
{
    for (int i = threadIdx.x; i < net.wbytes / 16; i += kQ2tThreads)
        reinterpret_cast<uint4 *>(wsm)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int l = 0; l < net.n_layers; ++l) {
        const int din = net.dims[l], dout = net.dims[l + 1], rowb = din / 4, cols = net.cols[l] + kQ2tPad;
        int8_t *dst = wsm + net.woff[l];
        if (rowb % 4 == 0) {
            // one 32-bit word of codes (16 weights) per thread and step, four loads in flight
            const int wpr = rowb / 4, nw = dout * wpr;
            for (int i0 = threadIdx.x; i0 < nw; i0 += 4 * kQ2tThreads) {
                uint32_t word[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * kQ2tThreads;
                    const int o = i / wpr, j = i - o * wpr;
                    word[u] = i < nw ? reinterpret_cast<const uint32_t *>(net.w[l] + (size_t)o * rowb)[j] : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * kQ2tThreads;
                    if (i >= nw) break;
                    const int o = i / wpr, j = i - o * wpr;
                    uint32_t out[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {  // packed byte b: weights 16 j + 4 b .. + 3
                        const uint32_t byte = (word[u] >> (8 * b)) & 0xFFu;
                        uint32_t v = 0;
#pragma unroll
                        for (int f = 0; f < 4; ++f) v |= (uint32_t)(uint8_t)(int8_t)q2_code_to_weight(byte, f) << (8 * f);
                        out[b] = v;
                    }
                    *reinterpret_cast<uint4 *>(dst + (size_t)o * cols + 16 * j) = make_uint4(out[0], out[1], out[2], out[3]);
                }
            }
        } else {
            for (int i = threadIdx.x; i < dout * din; i += kQ2tThreads) {
                const int o = i / din, k = i - o * din;
                dst[(size_t)o * cols + k] = (int8_t)q2_code_to_weight(net.w[l][(size_t)o * rowb + k / 4], k & 3);
            }
        }
    }
    __syncthreads();
}

// Every layer for 32 vectors.  The input limbs (columns past dims[0] zero)
// are read from `in`, laid out as one buffer ([limb 2][vector 32][kAStride]):
// buffer 0 of abuf, or a buffer of the caller's that the layers never write.
// The layers alternate between abuf's buffers 1 and 0.  Returns the buffer
// whose first bytes hold the int16 logits, vector v's at [v * kAStride + o].
// Ends with a CTA barrier.
__device__ __forceinline__ int q2t_forward(const Q2TNet &net, const int8_t *wsm, uint8_t *abuf, const uint8_t *in)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    int cur = 0;
    for (int l = 0; l < net.n_layers; ++l) {
        const bool hidden = l < net.n_layers - 1;
        const int mts = net.rows[l] / 16, kcs = net.cols[l] / 32, wcols = net.cols[l] + kQ2tPad;
        const int8_t *wl = wsm + net.woff[l];
        // (16-row tile, 8-vector tile) pairs, round-robin over the warps
        for (int pr = warp; pr < mts * (kQ2tVecs / 8); pr += kQ2tThreads / 32) {
            const int mt = pr / (kQ2tVecs / 8), nt = pr - mt * (kQ2tVecs / 8);
            int dlo[4] = {0, 0, 0, 0}, dhi[4] = {0, 0, 0, 0};
            const int8_t *wa = wl + (size_t)(mt * 16 + g) * wcols + 4 * t;
            const uint8_t *blo = (l == 0 ? in + (size_t)(nt * 8 + g) * kAStride : q2t_limb(abuf, cur, 0, nt * 8 + g)) + 4 * t;
            const uint8_t *bhi =
                (l == 0 ? in + (size_t)(kQ2tVecs + nt * 8 + g) * kAStride : q2t_limb(abuf, cur, 1, nt * 8 + g)) + 4 * t;
            for (int kc = 0; kc < kcs; ++kc) {
                const int k0 = 32 * kc;
                const uint32_t a0 = *reinterpret_cast<const uint32_t *>(wa + k0);
                const uint32_t a1 = *reinterpret_cast<const uint32_t *>(wa + 8 * wcols + k0);
                const uint32_t a2 = *reinterpret_cast<const uint32_t *>(wa + k0 + 16);
                const uint32_t a3 = *reinterpret_cast<const uint32_t *>(wa + 8 * wcols + k0 + 16);
                imma_s8u8(dlo, a0, a1, a2, a3, *reinterpret_cast<const uint32_t *>(blo + k0),
                          *reinterpret_cast<const uint32_t *>(blo + k0 + 16));
                imma_s8s8(dhi, a0, a1, a2, a3, *reinterpret_cast<const uint32_t *>(bhi + k0),
                          *reinterpret_cast<const uint32_t *>(bhi + k0 + 16));
            }
            // d[j]: row mt*16 + g + 8 (j >> 1), vector nt*8 + 2t + (j & 1)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int acc = dlo[j] + 256 * dhi[j];                         // exact: |acc| < 2^27
                const int16_t wrapped = (int16_t)(uint16_t)(uint32_t)acc;      // mod 2^16
                int16_t z = (int16_t)(wrapped >> 2);                           // arithmetic shift
                if (hidden && z < 0) z = 0;
                const int o = mt * 16 + g + 8 * (j >> 1), v = nt * 8 + 2 * t + (j & 1);
                if (hidden) {
                    q2t_limb(abuf, cur ^ 1, 0, v)[o] = (uint8_t)(z & 0xFF);
                    q2t_limb(abuf, cur ^ 1, 1, v)[o] = (uint8_t)(int8_t)(z >> 8);
                } else if (o < net.dims[l + 1]) {
                    // logits as int16: vector v's row spans both limb regions of the buffer
                    reinterpret_cast<int16_t *>(q2t_limb(abuf, cur ^ 1, 0, 0))[v * kAStride + o] = z;
                }
            }
        }
        __syncthreads();
        cur ^= 1;
    }
    return cur;
}

// Smallest index of the largest of n int16 values.
__device__ __forceinline__ int q2t_argmax(const int16_t *a, int n)
{
    int best = 0;
    for (int c = 1; c < n; ++c)
        if (a[c] > a[best]) best = c;  // strict: the lowest index wins ties
    return best;
}

__global__ void __launch_bounds__(kQ2tThreads) k_q2_mlp_tc(const Q2TNet net, const int16_t *__restrict__ x,
                                                           int batch, int16_t *__restrict__ logits,
                                                           int32_t *__restrict__ argmax)
{
    extern __shared__ __align__(16) uint8_t smem[];
    int8_t *wsm = reinterpret_cast<int8_t *>(smem);
    uint8_t *abuf = smem + net.wbytes;

    pdl_launch_dependents();
    pdl_wait_primary();
    q2t_expand_weights(net, wsm);

    const int ntiles = (batch + kQ2tVecs - 1) / kQ2tVecs;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int v0 = tile * kQ2tVecs, nv = min(kQ2tVecs, batch - v0);
        const int d0 = net.dims[0];
        // input limbs (zeros past the batch and past the input width)
        for (int i = threadIdx.x; i < kQ2tVecs * net.cols[0]; i += kQ2tThreads) {
            const int v = i / net.cols[0], k = i - v * net.cols[0];
            const int a = (v < nv && k < d0) ? (int)x[(int64_t)(v0 + v) * d0 + k] : 0;
            q2t_limb(abuf, 0, 0, v)[k] = (uint8_t)(a & 0xFF);
            q2t_limb(abuf, 0, 1, v)[k] = (uint8_t)(int8_t)(a >> 8);
        }
        __syncthreads();
        const int cur = q2t_forward(net, wsm, abuf, q2t_limb(abuf, 0, 0, 0));
        // logits (int16, in the last buffer) and argmax
        const int dl = net.dims[net.n_layers];
        const int16_t *lg = reinterpret_cast<const int16_t *>(q2t_limb(abuf, cur, 0, 0));
        for (int i = threadIdx.x; i < nv * dl; i += kQ2tThreads) {
            const int v = i / dl, c = i - v * dl;
            logits[(int64_t)(v0 + v) * dl + c] = lg[v * kAStride + c];
        }
        if (argmax != nullptr && threadIdx.x < nv) argmax[v0 + threadIdx.x] = q2t_argmax(lg + threadIdx.x * kAStride, dl);
        __syncthreads();  // the buffers are reused by the next tile
    }
}

// ---------------------------------------------------------------------------
// the autoregressive reply loop of "Show HN: Z80-uLM" (architecture and
// feature lists): 128 query + 128 context trigram buckets in, one output per
// character, one character per step.  The context buckets hold the trigram
// encoding of the reply so far (the library's reading; the page names the
// loop, not its state), and the character-set byte 0 ends a reply.
// ---------------------------------------------------------------------------
//
// A CTA keeps 32 conversations on the SM for their whole reply: their bucket
// vectors (int16 [32][256]) and the network's input limbs stay in shared
// memory, each step runs the network on all 32 (q2t_forward; the layers never
// write the input limbs), eight threads per conversation take its argmax, and
// one of them writes the character and updates the context buckets, and the
// limbs of the buckets that changed, in place.  Appending
// a letter c to a word whose last two characters are a, b (a = ' ' at the
// word start) changes three trigrams of the padded word: "ab " leaves, "abc"
// and "bc " arrive; a letter after a space starts a word " c "; a space
// changes nothing.  So the buckets after t characters equal the encoding of
// the t-character reply, which is what the definition re-encodes each step.

constexpr int kZ80MaxReply = 250;  // replies stay under the encoder's 255-character word limit
constexpr int kZ80Buckets = 128;

struct Z80Params {
    const uint8_t *queries;  // [batch][qlen]
    uint8_t *reply;          // [batch][max_new]
    int32_t *reply_len;      // [batch]
    int batch, qlen, max_new, nchars;
    uint8_t charset[kQ2tMaxDim];
};

__device__ __forceinline__ uint32_t z80_lower(uint32_t c) { return (c >= 'A' && c <= 'Z') ? c - 'A' + 'a' : c; }

// FNV-1a (32-bit) of three bytes, reduced to one of the 128 buckets.
__device__ __forceinline__ int z80_bucket(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t h = 2166136261u;
    h = (h ^ a) * 16777619u;
    h = (h ^ b) * 16777619u;
    h = (h ^ c) * 16777619u;
    return (int)(h & (kZ80Buckets - 1));
}

// Trigram buckets of one text (one thread): words are the runs between
// spaces, lower-cased, padded with one space on each side, at most 255
// characters kept per word; every 3-byte window adds 32 to its bucket.
__device__ void z80_encode(const uint8_t *__restrict__ text, int n, int16_t *buckets)
{
    for (int i = 0; i < kZ80Buckets; ++i) buckets[i] = 0;
    int i = 0;
    while (i < n) {
        while (i < n && text[i] == ' ') ++i;
        uint32_t x = 0, y = ' ';
        int len = 0;
        while (i < n && text[i] != ' ') {
            if (len < 255) {
                const uint32_t c = z80_lower(text[i]);
                if (len > 0) buckets[z80_bucket(x, y, c)] += 32;
                x = y;
                y = c;
                ++len;
            }
            ++i;
        }
        if (len == 0) break;
        buckets[z80_bucket(x, y, ' ')] += 32;
    }
}

__global__ void __launch_bounds__(kQ2tThreads) k_z80_generate(const Q2TNet net, const Z80Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    int8_t *wsm = reinterpret_cast<int8_t *>(smem);
    uint8_t *abuf = smem + net.wbytes;
    uint8_t *inb = abuf + 4 * kQ2tVecs * kAStride;                 // input limbs: [limb 2][vector 32][kAStride]
    int16_t *bk = reinterpret_cast<int16_t *>(inb + 2 * kQ2tVecs * kAStride);  // [32][256]: query, context
    __shared__ int s_len[kQ2tVecs];

    pdl_launch_dependents();
    pdl_wait_primary();
    q2t_expand_weights(net, wsm);

    const int ntiles = (p.batch + kQ2tVecs - 1) / kQ2tVecs;
    const int dl = net.dims[net.n_layers];
    // conversation v of a tile belongs to the 8 threads 8v .. 8v+7; thread 8v
    // keeps its state (the last two characters of the reply, lower-cased, ' '
    // before the first; whether it goes on)
    const int v = threadIdx.x >> 3, part = threadIdx.x & 7;
    const bool owner = part == 0;
    auto set_input = [&](int u, int k, int val) {   // bucket k of conversation u -> its two limbs
        inb[(size_t)u * kAStride + k] = (uint8_t)(val & 0xFF);
        inb[(size_t)(kQ2tVecs + u) * kAStride + k] = (uint8_t)(int8_t)(val >> 8);
    };
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int v0 = tile * kQ2tVecs, nv = min(kQ2tVecs, p.batch - v0);
        uint32_t a = ' ', b = ' ';
        bool live = false;
        if (owner) {
            int16_t *row = bk + v * 2 * kZ80Buckets;
            if (v < nv) {
                const uint8_t *q = p.queries + (int64_t)(v0 + v) * p.qlen;
                int n = 0;
                while (n < p.qlen && q[n] != 0) ++n;   // the query ends at its first 0 byte
                z80_encode(q, n, row);
                live = true;
            } else {
                for (int i = 0; i < kZ80Buckets; ++i) row[i] = 0;
            }
            for (int i = 0; i < kZ80Buckets; ++i) row[kZ80Buckets + i] = 0;  // empty reply
            s_len[v] = 0;
        }
        __syncthreads();
        // the input limbs once per tile; afterwards only changed buckets are rewritten
        for (int i = threadIdx.x; i < kQ2tVecs * 2 * kZ80Buckets; i += kQ2tThreads) set_input(i >> 8, i & 255, bk[i]);
        __syncthreads();
        for (int t = 0; t < p.max_new; ++t) {
            const int cur = q2t_forward(net, wsm, abuf, inb);
            const int16_t *lg = reinterpret_cast<const int16_t *>(q2t_limb(abuf, cur, 0, 0)) + v * kAStride;
            // argmax: each of the 8 threads scans every 8th logit, then the
            // largest value wins, the lowest index among equals
            int best = part < dl ? part : 0;
            int bv = part < dl ? lg[best] : -32768 - 1;
            for (int c = part + 8; c < dl; c += 8)
                if (lg[c] > bv) {
                    bv = lg[c];
                    best = c;
                }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) {
                const int ov = __shfl_xor_sync(0xffffffffu, bv, o), oc = __shfl_xor_sync(0xffffffffu, best, o);
                if (ov > bv || (ov == bv && oc < best)) {
                    bv = ov;
                    best = oc;
                }
            }
            if (owner && live) {
                const uint32_t ch = p.charset[best];
                if (ch == 0) {
                    live = false;                          // end of reply
                } else {
                    p.reply[(int64_t)(v0 + v) * p.max_new + t] = (uint8_t)ch;
                    s_len[v] = t + 1;
                    int16_t *ctx = bk + v * 2 * kZ80Buckets + kZ80Buckets;
                    const uint32_t c = z80_lower(ch);
                    auto bump = [&](int k, int d) {
                        ctx[k] += d;
                        set_input(v, kZ80Buckets + k, ctx[k]);
                    };
                    if (c != ' ') {
                        if (b == ' ') {
                            bump(z80_bucket(' ', c, ' '), 32);   // a new word " c "
                        } else {
                            bump(z80_bucket(a, b, ' '), -32);    // "ab " leaves
                            bump(z80_bucket(a, b, c), 32);       // "abc" and "bc " arrive
                            bump(z80_bucket(b, c, ' '), 32);
                        }
                    }
                    a = b;
                    b = c;
                }
            }
            // every thread has read the logits; stop when no reply of the tile goes on
            if (!__syncthreads_or(owner && live)) break;
        }
        if (owner && v < nv) {
            const int len = s_len[v];
            p.reply_len[v0 + v] = len;
            uint8_t *r = p.reply + (int64_t)(v0 + v) * p.max_new;
            for (int i = len; i < p.max_new; ++i) r[i] = 0;
        }
        __syncthreads();  // shared state is reused by the next tile
    }
}

// Network description for the tensor-core kernels (all widths <= 256);
// false when a width is larger.
static bool q2t_describe(const uint8_t *const *w_packed, const int32_t *dims, int n_layers, Q2TNet &tn)
{
    tn = Q2TNet{};
    tn.n_layers = n_layers;
    bool fits = true;
    int toff = 0;
    for (int l = 0; l <= n_layers; ++l) {
        tn.dims[l] = dims[l];
        fits = fits && dims[l] <= kQ2tMaxDim;
    }
    for (int l = 0; l < n_layers && fits; ++l) {
        tn.w[l] = w_packed[l];
        tn.rows[l] = (dims[l + 1] + 15) / 16 * 16;
        tn.cols[l] = (dims[l] + 31) / 32 * 32;
        tn.woff[l] = toff;
        toff += tn.rows[l] * (tn.cols[l] + kQ2tPad);
    }
    tn.wbytes = (toff + 15) & ~15;
    return fits;
}

static int num_sms_q2()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

constexpr size_t kZ80MaxSmem = 226u * 1024u;

size_t z80_smem_bytes(const int32_t *dims, int n_layers)
{
    Q2TNet tn;
    const uint8_t *none[kQ2MaxLayers] = {};
    if (n_layers < 1 || n_layers > kQ2MaxLayers || !q2t_describe(none, dims, n_layers, tn)) return 0;
    return (size_t)tn.wbytes + 6u * kQ2tVecs * kAStride + (size_t)kQ2tVecs * 2 * kZ80Buckets * 2;
}

lowbit_status z80_generate_launch(const uint8_t *const *w_packed, const int32_t *dims, int n_layers,
                                  const uint8_t *queries, int batch, int qlen, const uint8_t *charset, int max_new,
                                  uint8_t *reply, int32_t *reply_len, cudaStream_t st)
{
    Q2TNet tn;
    if (!q2t_describe(w_packed, dims, n_layers, tn)) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    const size_t smem = z80_smem_bytes(dims, n_layers);
    if (smem == 0 || smem > kZ80MaxSmem) return LOWBIT_ERR_UNSUPPORTED_SHAPE;
    Z80Params p = {};
    p.queries = queries;
    p.reply = reply;
    p.reply_len = reply_len;
    p.batch = batch;
    p.qlen = qlen;
    p.max_new = max_new;
    p.nchars = dims[n_layers];
    for (int i = 0; i < dims[n_layers]; ++i) p.charset[i] = charset[i];
    if (cudaFuncSetAttribute(k_z80_generate, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kZ80MaxSmem) !=
        cudaSuccess)
        return LOWBIT_ERR_CUDA;
    const int tiles = (batch + kQ2tVecs - 1) / kQ2tVecs;
    dim3 grid(std::min(tiles, num_sms_q2())), block(kQ2tThreads);
    cudaError_t e = launch_pdl(k_z80_generate, grid, block, smem, st, tn, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

lowbit_status q2_mlp_launch(const uint8_t *const *w_packed, const int32_t *dims, int n_layers,
                            const int16_t *x, int batch, int16_t *logits, int32_t *argmax,
                            cudaStream_t st)
{
    Q2Net net = {};
    net.n_layers = n_layers;
    int off = 0;
    for (int l = 0; l <= n_layers; ++l) net.dims[l] = dims[l];
    for (int l = 0; l < n_layers; ++l) {
        net.w[l] = w_packed[l];
        net.woff[l] = off;
        off += ((dims[l + 1] * (dims[l] / 4)) + 15) & ~15;
    }
    net.wbytes = off;
    if (batch == 0) return LOWBIT_OK;
    {
        Q2TNet tn;
        const bool fits = q2t_describe(w_packed, dims, n_layers, tn);
        const size_t tsmem = (size_t)tn.wbytes + 4u * kQ2tVecs * kAStride;
        if (fits && tsmem <= 200u * 1024u) {
            if (cudaFuncSetAttribute(k_q2_mlp_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) !=
                cudaSuccess)
                return LOWBIT_ERR_CUDA;
            int per_sm = 1;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_q2_mlp_tc, kQ2tThreads, tsmem) != cudaSuccess ||
                per_sm < 1)
                per_sm = 1;
            const int tiles = (batch + kQ2tVecs - 1) / kQ2tVecs;
            dim3 tgrid(std::min(tiles, per_sm * num_sms_q2())), tblock(kQ2tThreads);  // persistent: every CTA resident
            cudaError_t e = launch_pdl(k_q2_mlp_tc, tgrid, tblock, tsmem, st, tn, x, batch, logits, argmax);
            return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
        }
    }
    const size_t smem = (size_t)off + 2u * kVecs * kQ2MaxDim * sizeof(int16_t);
    // per-device function attribute, always set to the same (largest) value so
    // concurrent callers never shrink it under each other
    const int smem_max = kQ2MaxWeightBytes + 2 * kVecs * kQ2MaxDim * (int)sizeof(int16_t);
    if (cudaFuncSetAttribute(k_q2_mlp, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    dim3 grid((batch + kVecs - 1) / kVecs), block(256);
    cudaError_t e = launch_pdl(k_q2_mlp, grid, block, smem, st, net, x, batch, logits, argmax);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

int q2_weight_bytes_padded(const int32_t *dims, int n_layers)
{
    int off = 0;
    for (int l = 0; l < n_layers; ++l) off += ((dims[l + 1] * (dims[l] / 4)) + 15) & ~15;
    return off;
}

}  // namespace lowbit
