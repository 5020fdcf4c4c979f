// launch_util.h -- kernel launch with optional programmatic dependent launch.
#pragma once
#include <cuda_runtime.h>

namespace dfk {

// Launch `fn` (a __global__ function) with the given geometry.  With `pdl`
// the launch may begin while the previous kernel in the stream finishes;
// kernels here call griddepcontrol.wait before touching data that the
// previous kernel writes, so this only overlaps their prologues.
// `cluster_x` > 1 groups that many consecutive blocks along x into a
// thread-block cluster (portable sizes: at most 8).
// `cooperative`: every block of the grid is resident at once (the launch
// fails otherwise); for grids whose blocks wait on one another.
inline cudaError_t launch_kernel(const void *fn, dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, bool pdl, void **args,
                                 unsigned cluster_x = 1, bool cooperative = false) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  unsigned n = 0;
  if (cooperative) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// elementwise.cu
cudaError_t launch_rmsnorm_rows(const void *x, const void *gamma, float eps, void *out, int B,
                                int D, cudaStream_t s, bool pdl);
cudaError_t launch_silu(const void *a, void *out, long long n, cudaStream_t s, bool pdl);
cudaError_t launch_mul(const void *a, const void *b, void *out, long long n, cudaStream_t s,
                       bool pdl);
cudaError_t launch_copy16(const void *src, void *dst, size_t bytes, bool wait_first,
                          cudaStream_t s, bool pdl);
// selftest.cu
cudaError_t launch_wait_selftest(unsigned *err, unsigned long long *elapsed_ns, cudaStream_t s);

}  // namespace dfk
