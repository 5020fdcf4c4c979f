// cc_key.h -- key of one compiled CUDA-core engine instantiation.
#pragma once

// layout (2 bits) | matrices (2) | j per thread (4) | token tile (4) |
// k split (4) | fp32 activations (1) | RMSNorm prologue (1) | paired FMA (1) |
// FP8 E4M3 weights (1)
#define DFK_CC_KEY(L, NM, J, BT, KS, XF, NO, PR)                                 \
  ((L) | ((NM) << 2) | ((J) << 4) | ((BT) << 8) | ((KS) << 12) | ((XF) << 16) | \
   ((NO) << 17) | ((PR) << 18))
#define DFK_CC_KEY_W8 (1 << 19)

namespace dfk {
// Pointer to the __global__ function for a key, or nullptr if not compiled.
const void *cc_find_kernel(int key);
const void *cc_lookup_row(int key);
const void *cc_lookup_col(int key);
const void *cc_lookup_il(int key);
const void *cc_lookup_gemv_a(int key);
const void *cc_lookup_gemv_b(int key);
const void *cc_lookup_fp8_gate_up(int key);
const void *cc_lookup_fp8_gemv_a(int key);
const void *cc_lookup_fp8_gemv_b(int key);
const void *cc_lookup_qkv_a(int key);
const void *cc_lookup_qkv_b(int key);
}  // namespace dfk
