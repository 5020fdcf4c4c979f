// elementwise.cu -- the small kernels of the unfused baseline and of the
// decode stack: standalone RMSNorm, SiLU, multiply, per-row RMS rescale.
//
// The unfused baseline is the data flow the fusion removes ("Optimizing QKV
// Projection with Operator Fusion", section "The Why of Operator Fusion":
// every intermediate is written to HBM and read back by the next kernel).
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>

#include "launch_util.h"
#include "ptx.cuh"

namespace dfk {

// One warp per row.  The sum of squares uses the same fixed order as the
// fused gate/up prologue: lane l accumulates k = 8 l + e + 256 c (c, then e
// ascending), then a xor butterfly over the 32 lanes -- so r_b is the same
// fp32 value.  Unlike the fused prologue (which keeps xn in fp32), this
// kernel stores xn in HBM and therefore rounds it to bf16.
__global__ void rmsnorm_rows_kernel(const uint16_t *__restrict__ x,
                                    const uint16_t *__restrict__ gamma, float eps,
                                    uint16_t *__restrict__ out, int B, int D) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (row >= B) return;
  const uint16_t *xr = x + static_cast<size_t>(row) * D;
  float ss = 0.f;
  for (int k = 8 * lane; k < D; k += 256) {
    const uint4 v = ld_nc_v4(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float f0 = bf16_lo(w[i]), f1 = bf16_hi(w[i]);
      ss = fmaf(f0, f0, ss);
      ss = fmaf(f1, f1, ss);
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  const float r = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
  uint16_t *orow = out + static_cast<size_t>(row) * D;
  for (int k = 8 * lane; k < D; k += 256) {
    const uint4 v = ld_nc_v4(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t g[4] = {0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u};  // 1.0 pairs
    if (gamma) {
      const uint4 gv = ld_nc_v4(gamma + k);
      g[0] = gv.x; g[1] = gv.y; g[2] = gv.z; g[3] = gv.w;
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = f32_to_bf16_bits((bf16_lo(w[i]) * r) * bf16_lo(g[i]));
      const uint32_t hi = f32_to_bf16_bits((bf16_hi(w[i]) * r) * bf16_hi(g[i]));
      o[i] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(orow + k) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__global__ void silu_kernel(const uint16_t *__restrict__ a, uint16_t *__restrict__ out,
                            long long n) {
  pdl_wait();
  pdl_launch_dependents();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float v = __uint_as_float(static_cast<uint32_t>(a[i]) << 16);
    out[i] = f32_to_bf16_bits(v / (1.0f + expf(-v)));
  }
}

__global__ void mul_kernel(const uint16_t *__restrict__ a, const uint16_t *__restrict__ b,
                           uint16_t *__restrict__ out, long long n) {
  pdl_wait();
  pdl_launch_dependents();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float va = __uint_as_float(static_cast<uint32_t>(a[i]) << 16);
    const float vb = __uint_as_float(static_cast<uint32_t>(b[i]) << 16);
    out[i] = f32_to_bf16_bits(va * vb);
  }
}

}  // namespace dfk

namespace dfk {

cudaError_t launch_rmsnorm_rows(const void *x, const void *gamma, float eps, void *out, int B,
                                int D, cudaStream_t s, bool pdl) {
  const int warps = 8;
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  const uint16_t *gp = static_cast<const uint16_t *>(gamma);
  uint16_t *op = static_cast<uint16_t *>(out);
  void *args[] = {&xp, &gp, &eps, &op, &B, &D};
  return launch_kernel(reinterpret_cast<const void *>(&rmsnorm_rows_kernel),
                       dim3((B + warps - 1) / warps), dim3(32 * warps), 0, s, pdl, args);
}

static unsigned ew_blocks(long long n) {
  long long b = (n + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

cudaError_t launch_silu(const void *a, void *out, long long n, cudaStream_t s, bool pdl) {
  const uint16_t *ap = static_cast<const uint16_t *>(a);
  uint16_t *op = static_cast<uint16_t *>(out);
  void *args[] = {&ap, &op, &n};
  return launch_kernel(reinterpret_cast<const void *>(&silu_kernel), dim3(ew_blocks(n)),
                       dim3(256), 0, s, pdl, args);
}

cudaError_t launch_mul(const void *a, const void *b, void *out, long long n, cudaStream_t s,
                       bool pdl) {
  const uint16_t *ap = static_cast<const uint16_t *>(a);
  const uint16_t *bp = static_cast<const uint16_t *>(b);
  uint16_t *op = static_cast<uint16_t *>(out);
  void *args[] = {&ap, &bp, &op, &n};
  return launch_kernel(reinterpret_cast<const void *>(&mul_kernel), dim3(ew_blocks(n)),
                       dim3(256), 0, s, pdl, args);
}

// Device copy of `n16` 16-byte chunks, used by the host-memory entry point
// to move x into and y out of pinned host buffers that the device addresses
// directly (in place of copy-engine transfers, so the copies take part in
// programmatic dependent launch).  WAIT_FIRST: the source is the previous
// kernel's output (wait before reading); otherwise the loads are issued
// first and only the stores wait for the previous kernel.
template <bool WAIT_FIRST>
__global__ void copy16_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                              size_t n16) {
  if (WAIT_FIRST) pdl_wait();
  pdl_launch_dependents();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint4 v[4];
  for (; i < n16; i += 4 * stride) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * stride < n16) v[u] = src[i + u * stride];
    if (!WAIT_FIRST) pdl_wait();
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * stride < n16) dst[i + u * stride] = v[u];
  }
  if (!WAIT_FIRST) pdl_wait();  // threads without work still order after the previous kernel
}

cudaError_t launch_copy16(const void *src, void *dst, size_t bytes, bool wait_first,
                          cudaStream_t s, bool pdl) {
  const size_t n16 = bytes / 16;
  if (n16 == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>(148, (n16 + threads - 1) / threads));
  const uint4 *a = static_cast<const uint4 *>(src);
  uint4 *b = static_cast<uint4 *>(dst);
  size_t n = n16;
  void *args[] = {&a, &b, &n};
  return launch_kernel(wait_first ? reinterpret_cast<const void *>(&copy16_kernel<true>)
                                  : reinterpret_cast<const void *>(&copy16_kernel<false>),
                       dim3(blocks), dim3(threads), 0, s, pdl, args);
}

}  // namespace dfk
