// tc_key.h -- lookup of the compiled tensor-core kernel instantiations.
#pragma once

namespace dfk {
// __global__ function for (matrices, RMSNorm prologue, weight layout 0 row /
// 1 column / 2 interleaved, sub-tiles), or nullptr.
const void *tc_find_kernel(int nmat, int norm, int wl, int mt);
}  // namespace dfk
