// Fused gate/up, gate/up-interleaved weights [F][2][D].
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_il(int key) {
  switch (key) {
    DFK_CC_JB(2, 2, 1, 1, 0)
    DFK_CC_JB(2, 2, 1, 1, 1)
    DFK_CC_JB(2, 2, 1, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
