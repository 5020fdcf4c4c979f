// GEMV with FP8 E4M3 weights (down projection), k split 1 and 2.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_fp8_gemv_a(int key) {
  switch (key) {
    DFK_CC_JB8(1, 1, 1, 0)
    DFK_CC_JB8(1, 1, 0, 0)
    DFK_CC_JB8(1, 2, 1, 0)
    DFK_CC_JB8(1, 2, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
