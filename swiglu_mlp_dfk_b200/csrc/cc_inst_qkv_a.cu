// GEMV with the RMSNorm prologue (packed QKV projection), k split 1 and 2.
#include "cc_inst.cuh"
namespace dfk {
const void *cc_lookup_qkv_a(int key) {
  switch (key) {
    DFK_CC_JB(0, 1, 1, 1, 1)
    DFK_CC_JB(0, 1, 2, 1, 1)
    default: return nullptr;
  }
}
}  // namespace dfk
