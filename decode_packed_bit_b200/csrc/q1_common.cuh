// q1_common.cuh -- what the Q1_0_g128 M = 1 tensor-core kernels share: the
// group of weight matrices one launch multiplies with the same activation.
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


}  // namespace lowbit
