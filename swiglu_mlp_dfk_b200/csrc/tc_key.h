// tc_key.h -- lookup of the compiled tensor-core kernel instantiations.
#pragma once

namespace dfk {
// __global__ function for (matrices, RMSNorm prologue, interleaved, sub-tiles), or nullptr.
const void *tc_find_kernel(int nmat, int norm, int il, int mt);
}  // namespace dfk
