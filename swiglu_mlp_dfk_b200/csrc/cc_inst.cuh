// cc_inst.cuh -- instantiation helpers for the CUDA-core engine.  Each
// cc_inst_*.cu file instantiates a slice of the template space (so the
// slices compile in parallel) and exposes a lookup by key.
#pragma once
#include "cc_engine.cuh"
#include "cc_key.h"

#define DFK_CC_CASE(L, NM, J, BT, KS, XF, NO)                                   \
  case DFK_CC_KEY(L, NM, J, BT, KS, XF, NO, 0):                                 \
    return reinterpret_cast<const void *>(                                      \
        &dfk::cc_gemv_kernel<L, NM, J, BT, KS, (XF) != 0, (NO) != 0, false>);    \
  case DFK_CC_KEY(L, NM, J, BT, KS, XF, NO, 1):                                 \
    return reinterpret_cast<const void *>(                                      \
        &dfk::cc_gemv_kernel<L, NM, J, BT, KS, (XF) != 0, (NO) != 0, true>);

// every (j_per_thread, token_tile) pair compiled
#define DFK_CC_JB(L, NM, KS, XF, NO)                                                 \
  DFK_CC_CASE(L, NM, 4, 1, KS, XF, NO) DFK_CC_CASE(L, NM, 4, 2, KS, XF, NO)          \
  DFK_CC_CASE(L, NM, 4, 4, KS, XF, NO) DFK_CC_CASE(L, NM, 2, 1, KS, XF, NO)          \
  DFK_CC_CASE(L, NM, 2, 2, KS, XF, NO) DFK_CC_CASE(L, NM, 2, 4, KS, XF, NO)          \
  DFK_CC_CASE(L, NM, 2, 8, KS, XF, NO)

// FP8 E4M3 weights (row-major only)
#define DFK_CC_CASE8(NM, J, BT, KS, XF, NO)                                            \
  case DFK_CC_KEY(0, NM, J, BT, KS, XF, NO, 0) | DFK_CC_KEY_W8:                        \
    return reinterpret_cast<const void *>(                                             \
        &dfk::cc_gemv_kernel<0, NM, J, BT, KS, (XF) != 0, (NO) != 0, false, true>);     \
  case DFK_CC_KEY(0, NM, J, BT, KS, XF, NO, 1) | DFK_CC_KEY_W8:                        \
    return reinterpret_cast<const void *>(                                             \
        &dfk::cc_gemv_kernel<0, NM, J, BT, KS, (XF) != 0, (NO) != 0, true, true>);

#define DFK_CC_JB8(NM, KS, XF, NO)                                                \
  DFK_CC_CASE8(NM, 4, 1, KS, XF, NO) DFK_CC_CASE8(NM, 4, 2, KS, XF, NO)            \
  DFK_CC_CASE8(NM, 4, 4, KS, XF, NO) DFK_CC_CASE8(NM, 2, 1, KS, XF, NO)            \
  DFK_CC_CASE8(NM, 2, 2, KS, XF, NO) DFK_CC_CASE8(NM, 2, 4, KS, XF, NO)            \
  DFK_CC_CASE8(NM, 2, 8, KS, XF, NO)
