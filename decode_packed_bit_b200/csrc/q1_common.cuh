// q1_common.cuh -- what the Q1_0_g128 M = 1 tensor-core kernels share: the
// group of weight matrices one launch multiplies with the same activation,
// and the entry points of the two implementations.
#pragma once

#include "common.cuh"

namespace lowbit {

constexpr int kQ1MaxGroup = 256;  // matrices per grouped launch

// Pointers of the R matrices of a group, passed by value as a kernel
// argument (6 KiB).
struct Q1Group {
    const uint8_t *bits[kQ1MaxGroup];
    const uint16_t *scales[kQ1MaxGroup];
    float *y[kQ1MaxGroup];
};

// tcgen05 implementation (q1_gemv_tc.cu), for K a multiple of 1024.
bool q1tc_supported(int R, int N, int K);
size_t q1tc_act_bytes(int K);
size_t q1tc_xcopy_off(int K);
lowbit_status q1tc_prepare_launch(const uint16_t *x, int K, void *act, cudaStream_t st);
lowbit_status q1tc_gemv_launch(const uint8_t *const *bits, const uint16_t *const *scales, const void *act,
                               float *const *y, int R, int N, int K, cudaStream_t st);
int q1tc_fault_flag();

}  // namespace lowbit
