// noalloc.cu -- the down projection for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc when they run the MLP: a serving
// runtime that reserves all device memory for its own pool up front, code
// that runs inside CUDA stream capture (allocation calls are not permitted
// while a stream is being captured), or a host that lends this library a
// device it does not own.  The ordinary split-K down projection keeps its
// partial sums in a workspace that the library allocates on first use; this
// entry point runs the same kernel on a fixed-size scratch array that is part
// of the library image instead (a static __device__ array, resident on every
// device that loads the library until the process exits) and calls no
// allocating routine.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <map>
#include <mutex>

#include "dfk.h"

namespace dfk {
int down_proj_with_scratch(const void *h, const void *w_down, void *y, int B, int d_model,
                           int d_ff, float *part, size_t part_capacity, unsigned *counters,
                           size_t counter_capacity, bool clear_counters, cudaStream_t s);
}  // namespace dfk

namespace {

// Partial sums: at most (#SMs) x 64 tokens x 128 rows of fp32 (4.85 MB on a
// 148-SM B200); counters: one per row block.
constexpr size_t kPartBytes = static_cast<size_t>(6) << 20;  // 6 MiB
constexpr size_t kCounterBytes = 4096;                       // 1024 row blocks

}  // namespace

static __device__ __align__(256) unsigned char g_dfk_static_scratch[kPartBytes + kCounterBytes];

namespace {

std::mutex g_static_mu;
std::map<int, unsigned char *> g_static_addr;  // device -> device address of the array

// Device address of the array on the current device.  Host code cannot use
// the array's name as a device pointer; the address is looked up once per
// device with that device current.
int static_scratch(unsigned char **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DFK_ERR_ARCH;
  }
  std::lock_guard<std::mutex> lk(g_static_mu);
  auto it = g_static_addr.find(dev);
  if (it != g_static_addr.end()) {
    *out = it->second;
    return DFK_OK;
  }
  void *ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_dfk_static_scratch);
  if (e != cudaSuccess || !ptr) {
    cudaGetLastError();
    return DFK_ERR_CUDA;
  }
  g_static_addr[dev] = static_cast<unsigned char *>(ptr);
  *out = static_cast<unsigned char *>(ptr);
  return DFK_OK;
}

}  // namespace

extern "C" int dfk_down_proj_static_scratch(const void *h, const void *w_down, void *y, int B,
                                            int d_model, int d_ff, void *stream) {
  if (B == 0) return DFK_OK;
  unsigned char *base = nullptr;
  int rc = static_scratch(&base);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned *counters = reinterpret_cast<unsigned *>(base + kPartBytes);
  // the arrival counters must start at zero (the array keeps the last call's
  // contents): cleared on the stream once the arguments have been accepted
  return dfk::down_proj_with_scratch(h, w_down, y, B, d_model, d_ff,
                                     reinterpret_cast<float *>(base), kPartBytes, counters,
                                     kCounterBytes, /*clear_counters=*/true, s);
}
