// tf8_key.h -- lookup of the FP8 tensor-core kernels.
#pragma once

namespace dfk {
// Pointer to the __global__ function, or nullptr if that combination is not compiled.
const void *tf8_find_kernel(int nmat, bool norm);
}  // namespace dfk
