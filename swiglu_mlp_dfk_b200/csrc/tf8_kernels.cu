// FP8 tensor-core kernel instantiations: fused gate/up (with and without the
// RMSNorm prologue) and the GEMV (down projection).
#include "tf8_engine.cuh"
#include "tf8_key.h"

namespace dfk {
const void *tf8_find_kernel(int nmat, bool norm) {
  if (nmat == 2 && norm) return reinterpret_cast<const void *>(&tf8_gemv_kernel<2, true>);
  if (nmat == 2) return reinterpret_cast<const void *>(&tf8_gemv_kernel<2, false>);
  if (nmat == 1 && !norm) return reinterpret_cast<const void *>(&tf8_gemv_kernel<1, false>);
  return nullptr;
}
}  // namespace dfk
