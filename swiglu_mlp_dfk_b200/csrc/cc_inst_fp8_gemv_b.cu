// GEMV with FP8 E4M3 weights (down projection), k split 4 and 8.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_fp8_gemv_b(int key) {
  switch (key) {
    DFK_CC_JB8(1, 4, 1, 0)
    DFK_CC_JB8(1, 4, 0, 0)
    DFK_CC_JB8(1, 8, 1, 0)
    DFK_CC_JB8(1, 8, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
