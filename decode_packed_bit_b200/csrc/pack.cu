// pack.cu -- packers and unpackers of the three weight formats.
//
// Layouts (see include/lowbit.h): one row is packed along its columns, the
// lowest column in the lowest bits of each byte.
//   Q1_0_g128: 8 sign codes per byte, code of column c at bit c%8.
//   Q2:        4 codes per byte, code of column c at bits 2*(c%4)..+1
//              ("Show HN: Z80-uLM": the unpack listing takes the bottom two
//              bits first and rotates the next field down).
//   INT4_G64:  2 nibbles per byte, even column in the low nibble.
// One thread produces one packed byte (pack) or consumes one (unpack); the
// codes of one byte are one aligned 8/4/2-byte word, so the loads and stores
// are single vector accesses.
#include "common.cuh"

namespace lowbit {

__global__ void __launch_bounds__(256) k_pack_q1(const uint2 *__restrict__ codes,
                                                 uint8_t *__restrict__ packed, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    uint2 c = codes[i];
    // gather bit 0 of each of the 8 code bytes into one byte
    uint32_t lo = c.x & 0x01010101u, hi = c.y & 0x01010101u;
    uint32_t b = (lo | (lo >> 7) | (lo >> 14) | (lo >> 21)) & 0xFu;
    b |= ((hi | (hi >> 7) | (hi >> 14) | (hi >> 21)) & 0xFu) << 4;
    packed[i] = (uint8_t)b;
}

__global__ void __launch_bounds__(256) k_unpack_q1(const uint8_t *__restrict__ packed,
                                                   uint2 *__restrict__ codes, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    uint32_t b = packed[i];
    uint32_t lo = ((b & 1u) | ((b & 2u) << 7) | ((b & 4u) << 14) | ((b & 8u) << 21));
    uint32_t hi = (((b >> 4) & 1u) | (((b >> 4) & 2u) << 7) | (((b >> 4) & 4u) << 14) |
                   (((b >> 4) & 8u) << 21));
    codes[i] = make_uint2(lo, hi);
}

__global__ void __launch_bounds__(256) k_pack_q2(const uint32_t *__restrict__ codes,
                                                 uint8_t *__restrict__ packed, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    uint32_t c = codes[i] & 0x03030303u;
    packed[i] = (uint8_t)((c | (c >> 6) | (c >> 12) | (c >> 18)) & 0xFFu);
}

__global__ void __launch_bounds__(256) k_unpack_q2(const uint8_t *__restrict__ packed,
                                                   uint32_t *__restrict__ codes, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    uint32_t b = packed[i];
    codes[i] = (b & 3u) | (((b >> 2) & 3u) << 8) | (((b >> 4) & 3u) << 16) | (((b >> 6) & 3u) << 24);
}

__global__ void __launch_bounds__(256) k_pack_int4(const uint16_t *__restrict__ codes,
                                                   uint8_t *__restrict__ packed, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    uint32_t c = codes[i];  // low byte = even column, high byte = odd column
    packed[i] = (uint8_t)((c & 0xFu) | ((c >> 4) & 0xF0u));
}

__global__ void __launch_bounds__(256) k_unpack_int4(const uint8_t *__restrict__ packed,
                                                     uint16_t *__restrict__ codes, int64_t nbytes)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    int32_t b = packed[i];
    // sign-extend each nibble to an int8: shift it to the top of an int32 and
    // shift back arithmetically
    int32_t lo = (b << 28) >> 28, hi = (b << 24) >> 28;
    codes[i] = (uint16_t)((lo & 0xFF) | ((hi & 0xFF) << 8));
}

lowbit_status pack_launch(lowbit_format fmt, const int8_t *codes, int64_t rows, int64_t cols,
                          uint8_t *packed, cudaStream_t st)
{
    int per = fmt == LOWBIT_FMT_Q1_G128 ? 8 : fmt == LOWBIT_FMT_Q2 ? 4 : 2;
    int64_t nbytes = rows * (cols / per);
    if (nbytes == 0) return LOWBIT_OK;
    int64_t blocks = (nbytes + 255) / 256;
    if (fmt == LOWBIT_FMT_Q1_G128)
        k_pack_q1<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint2 *>(codes), packed, nbytes);
    else if (fmt == LOWBIT_FMT_Q2)
        k_pack_q2<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint32_t *>(codes), packed, nbytes);
    else
        k_pack_int4<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint16_t *>(codes), packed, nbytes);
    return launch_status();
}

lowbit_status unpack_launch(lowbit_format fmt, const uint8_t *packed, int64_t rows, int64_t cols,
                            int8_t *codes, cudaStream_t st)
{
    int per = fmt == LOWBIT_FMT_Q1_G128 ? 8 : fmt == LOWBIT_FMT_Q2 ? 4 : 2;
    int64_t nbytes = rows * (cols / per);
    if (nbytes == 0) return LOWBIT_OK;
    int64_t blocks = (nbytes + 255) / 256;
    if (fmt == LOWBIT_FMT_Q1_G128)
        k_unpack_q1<<<(unsigned)blocks, 256, 0, st>>>(packed, reinterpret_cast<uint2 *>(codes), nbytes);
    else if (fmt == LOWBIT_FMT_Q2)
        k_unpack_q2<<<(unsigned)blocks, 256, 0, st>>>(packed, reinterpret_cast<uint32_t *>(codes), nbytes);
    else
        k_unpack_int4<<<(unsigned)blocks, 256, 0, st>>>(packed, reinterpret_cast<uint16_t *>(codes), nbytes);
    return launch_status();
}

}  // namespace lowbit
