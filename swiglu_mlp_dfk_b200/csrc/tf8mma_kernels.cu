// E4M3-MMA FP8 kernel instantiations and the activation-term prep kernel.
#define DFK_TF8MMA_KERNELS
#include "tf8mma_engine.cuh"
#include "tf8_key.h"

namespace dfk {
#define DFK_TM8(NM, BP, T) reinterpret_cast<const void *>(&tf8mma_kernel<NM, BP, T>)
const void *tf8mma_find_kernel(int nmat, int ibp, int it) {
  if (nmat != 1 && nmat != 2) return nullptr;
  const bool two = nmat == 2;
  if (ibp == 0) return two ? DFK_TM8(2, 0, 0) : DFK_TM8(1, 0, 0);
  if (ibp == 4 && it == 4) return two ? DFK_TM8(2, 4, 4) : DFK_TM8(1, 4, 4);
  if (ibp == 8 && it == 2) return two ? DFK_TM8(2, 8, 2) : DFK_TM8(1, 8, 2);
  if (ibp == 8 && it == 4) return two ? DFK_TM8(2, 8, 4) : DFK_TM8(1, 8, 4);
  if (ibp == 16 && it == 2) return two ? DFK_TM8(2, 16, 2) : DFK_TM8(1, 16, 2);
  return nullptr;
}
#undef DFK_TM8
const void *tf8mma_prep_fn() { return reinterpret_cast<const void *>(&tf8mma_prep_kernel); }
}  // namespace dfk
