// tc_key.h -- lookup of the compiled tensor-core kernel instantiations.
#pragma once

namespace dfk {
// __global__ function for (matrices, RMSNorm mode 0 none / 1 in kernel /
// 2 prepared, weight layout 0 row / 1 column / 2 interleaved, sub-tiles), or
// nullptr.
const void *tc_find_kernel(int nmat, int norm, int wl, int mt);
// The prep kernel of RMSNorm mode 2.
const void *tc_norm_prep_fn();
}  // namespace dfk
