// Plain GEMV (down projection, unfused baseline), k split 1 and 2.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_gemv_a(int key) {
  switch (key) {
    DFK_CC_JB(0, 1, 1, 1, 0)
    DFK_CC_JB(0, 1, 1, 0, 0)
    DFK_CC_JB(0, 1, 2, 1, 0)
    DFK_CC_JB(0, 1, 2, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
