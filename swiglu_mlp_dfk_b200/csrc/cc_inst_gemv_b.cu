// Plain GEMV (down projection, unfused baseline), k split 4 and 8.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_gemv_b(int key) {
  switch (key) {
    DFK_CC_JB(0, 1, 4, 1, 0)
    DFK_CC_JB(0, 1, 4, 0, 0)
    DFK_CC_JB(0, 1, 8, 1, 0)
    DFK_CC_JB(0, 1, 8, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
