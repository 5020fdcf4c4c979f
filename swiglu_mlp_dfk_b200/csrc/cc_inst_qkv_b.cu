// GEMV with the RMSNorm prologue (packed QKV projection), k split 4 and 8.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_qkv_b(int key) {
  switch (key) {
    DFK_CC_JB(0, 1, 4, 1, 1)
    DFK_CC_JB(0, 1, 8, 1, 1)
    default: return nullptr;
  }
}
}  // namespace dfk
