// tf8_key.h -- lookup of the FP8 tensor-core kernels.
#pragma once

namespace dfk {
// Pointer to the __global__ function, or nullptr if that combination is not compiled.
const void *tf8_find_kernel(int nmat, bool norm);
// E4M3-MMA kernel (fused gate/up: nmat 2; GEMV: nmat 1) and the prep kernel.
// ibp = 0: terms from the prep kernel; ibp > 0: terms derived inside the
// kernel for ibp token slots, it terms each ((4, 4), (8, 2), (8, 4), (16, 2)).
const void *tf8mma_find_kernel(int nmat, int ibp, int it);
const void *tf8mma_prep_fn();
}  // namespace dfk
