// launch_util.h -- kernel launch with optional programmatic dependent launch.
#pragma once
#include <cuda_runtime.h>

namespace dfk {

// Launch `fn` (a __global__ function) with the given geometry.  With `pdl`
// the launch may begin while the previous kernel in the stream finishes;
// kernels here call griddepcontrol.wait before touching data that the
// previous kernel writes, so this only overlaps their prologues.
inline cudaError_t launch_kernel(const void *fn, dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, bool pdl, void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// elementwise.cu
cudaError_t launch_rmsnorm_rows(const void *x, const void *gamma, float eps, void *out, int B,
                                int D, cudaStream_t s, bool pdl);
cudaError_t launch_silu(const void *a, void *out, long long n, cudaStream_t s, bool pdl);
cudaError_t launch_mul(const void *a, const void *b, void *out, long long n, cudaStream_t s,
                       bool pdl);

}  // namespace dfk
