// Instantiations of the tensor-core engine: fused gate/up (with and without
// the RMSNorm prologue, row-major or interleaved weights) and the plain GEMV
// of the down projection, each with one or two 128-row sub-tiles per CTA.
#include "tc_engine.cuh"
#include "tc_key.h"

namespace dfk {

const void *tc_find_kernel(int nmat, int norm, int il, int mt) {
#define DFK_TC_ENTRY(NM, NO, IL_, MT_)                                                    \
  if (nmat == NM && norm == NO && il == IL_ && mt == MT_)                                 \
    return reinterpret_cast<const void *>(&tc_gemv_kernel<NM, (NO) != 0, (IL_) != 0, MT_>);
  DFK_TC_ENTRY(2, 0, 0, 1)
  DFK_TC_ENTRY(2, 0, 0, 2)
  DFK_TC_ENTRY(2, 1, 0, 1)
  DFK_TC_ENTRY(2, 1, 0, 2)
  DFK_TC_ENTRY(2, 0, 1, 1)
  DFK_TC_ENTRY(2, 0, 1, 2)
  DFK_TC_ENTRY(2, 1, 1, 1)
  DFK_TC_ENTRY(2, 1, 1, 2)
  DFK_TC_ENTRY(1, 0, 0, 1)
  DFK_TC_ENTRY(1, 0, 0, 2)
#undef DFK_TC_ENTRY
  return nullptr;
}

}  // namespace dfk
