// Fused gate/up, row-major weights [F][D] x2.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_row(int key) {
  switch (key) {
    DFK_CC_JB(0, 2, 1, 1, 0)
    DFK_CC_JB(0, 2, 1, 1, 1)
    DFK_CC_JB(0, 2, 1, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
