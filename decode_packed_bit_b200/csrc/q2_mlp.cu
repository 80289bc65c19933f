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
