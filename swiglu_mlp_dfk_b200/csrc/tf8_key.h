// tf8_key.h -- lookup of the FP8 tensor-core kernels.
#pragma once

namespace dfk {
// Pointer to the __global__ function, or nullptr if that combination is not compiled.
const void *tf8_find_kernel(int nmat, bool norm);
// E4M3-MMA kernel (fused gate/up: nmat 2; GEMV: nmat 1) and its prep kernel.
const void *tf8mma_find_kernel(int nmat);
const void *tf8mma_prep_fn();
}  // namespace dfk
