// E4M3-MMA FP8 kernel instantiations and the activation-term prep kernel.
#define DFK_TF8MMA_KERNELS
#include "tf8mma_engine.cuh"
#include "tf8_key.h"

namespace dfk {
const void *tf8mma_find_kernel(int nmat) {
  if (nmat == 2) return reinterpret_cast<const void *>(&tf8mma_kernel<2>);
  if (nmat == 1) return reinterpret_cast<const void *>(&tf8mma_kernel<1>);
  return nullptr;
}
const void *tf8mma_prep_fn() { return reinterpret_cast<const void *>(&tf8mma_prep_kernel); }
}  // namespace dfk
