// Fused gate/up with FP8 E4M3 weights [F][D] x2 and per-row scales.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_fp8_gate_up(int key) {
  switch (key) {
    DFK_CC_JB8(2, 1, 1, 0)
    DFK_CC_JB8(2, 1, 1, 1)
    DFK_CC_JB8(2, 1, 0, 0)
    default: return nullptr;
  }
}
}  // namespace dfk
