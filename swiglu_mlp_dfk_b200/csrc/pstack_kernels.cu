// Instantiation of the persistent decode-step kernel (pstack_engine.cuh).
#define DFK_PSTACK_KERNELS
#include "pstack_engine.cuh"

namespace dfk {

const void *pstack_fn() { return reinterpret_cast<const void *>(&pstack_kernel); }

}  // namespace dfk
