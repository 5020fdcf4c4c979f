// Instantiations of the tensor-core engine: fused gate/up (without the
// RMSNorm prologue, with it transformed in the kernel, or with it prepared by
// the prep kernel; row-major, interleaved or column-major weights) and
// the GEMV (down projection; with the RMSNorm prologue, the packed QKV
// projection), with one or two 128-row sub-tiles per CTA (one for
// column-major).
#define DFK_TC_KERNELS
#include "tc_engine.cuh"
#include "tc_key.h"

namespace dfk {

const void *tc_find_kernel(int nmat, int norm, int wl, int mt) {
#define DFK_TC_ENTRY(NM, NO, WL_, MT_)                                          \
  if (nmat == NM && norm == NO && wl == WL_ && mt == MT_)                       \
    return reinterpret_cast<const void *>(&tc_gemv_kernel<NM, NO, WL_, MT_>);
  DFK_TC_ENTRY(2, 0, 0, 1)
  DFK_TC_ENTRY(2, 0, 0, 2)
  DFK_TC_ENTRY(2, 1, 0, 1)
  DFK_TC_ENTRY(2, 1, 0, 2)
  DFK_TC_ENTRY(2, 0, 2, 1)
  DFK_TC_ENTRY(2, 0, 2, 2)
  DFK_TC_ENTRY(2, 1, 2, 1)
  DFK_TC_ENTRY(2, 1, 2, 2)
  DFK_TC_ENTRY(2, 0, 1, 1)
  DFK_TC_ENTRY(2, 1, 1, 1)
  DFK_TC_ENTRY(2, 2, 0, 1)
  DFK_TC_ENTRY(2, 2, 0, 2)
  DFK_TC_ENTRY(2, 2, 2, 1)
  DFK_TC_ENTRY(2, 2, 2, 2)
  DFK_TC_ENTRY(2, 2, 1, 1)
  DFK_TC_ENTRY(1, 0, 0, 1)
  DFK_TC_ENTRY(1, 0, 0, 2)
  DFK_TC_ENTRY(1, 1, 0, 1)
  DFK_TC_ENTRY(1, 1, 0, 2)
  DFK_TC_ENTRY(1, 2, 0, 1)
  DFK_TC_ENTRY(1, 2, 0, 2)
#undef DFK_TC_ENTRY
  return nullptr;
}

const void *tc_norm_prep_fn() { return reinterpret_cast<const void *>(&tc_norm_prep_kernel); }

}  // namespace dfk
