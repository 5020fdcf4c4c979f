// tp.cu -- tensor-parallel MLP: the reduction dimension of the down
// projection (d_ff) is sharded over the ranks of a group, one GPU each, and
// the all-reduce of the partial outputs is fused into the down-projection
// kernel's epilogue over peer memory ("Deep Kernel Fusion for Transformers",
// abstract: the kernel stays adaptable to inference configurations; the
// shard boundaries follow the gate/up pairs, so the fused gate/up needs no
// communication at all).
//
// Each rank owns one device buffer (tp_internal.h) and maps every peer's
// buffer through CUDA IPC.  The host side here only allocates, maps and
// validates; the exchange itself runs in the kernel.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <tuple>

#include "dfk.h"
#include "tp_internal.h"

struct dfk_tp_group {
  int world = 0, rank = 0, bmax = 0, d_model = 0, dev = -1;
  void *own = nullptr;                    // this rank's buffer (cudaMalloc)
  void *buf[dfk::TP_MAX_RANKS] = {};      // every rank's buffer in this process
  bool opened[dfk::TP_MAX_RANKS] = {};    // IPC mappings to close
  bool connected = false;
};

namespace {

int tp_fail(int status, const char *msg) { return dfk::report_error(status, msg); }

int cuda_status(cudaError_t e) {
  cudaGetLastError();
  return dfk::report_error(DFK_ERR_CUDA, cudaGetErrorString(e));
}

// The emulated groups: all ranks' buffers on one device, one allocation
// per (device, world, d_model), grown for the token capacity.
struct Emu {
  void *base = nullptr;
  int bmax = 0;
};
std::mutex g_emu_mu;
std::map<std::tuple<int, int, int>, Emu> g_emu;

}  // namespace

extern "C" {

int dfk_tp_group_create(int world, int rank, int max_B, int d_model, dfk_tp_group **out,
                        void *handle) {
  if (!out || !handle) return tp_fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  *out = nullptr;
  if (world < 1 || world > dfk::TP_MAX_RANKS || rank < 0 || rank >= world)
    return tp_fail(DFK_ERR_INVALID_ARG, "world must be 1..8 and 0 <= rank < world");
  if (max_B < 1 || max_B > 64 || d_model <= 0 || d_model % 8)
    return tp_fail(DFK_ERR_UNSUPPORTED_SHAPE, "need 1 <= max_B <= 64 and d_model % 8 == 0");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e) return cuda_status(e);
  const dfk::TpLayout L = dfk::tp_layout(world, max_B, d_model);
  void *p = nullptr;
  if ((e = cudaMalloc(&p, L.total))) return cuda_status(e);
  if ((e = cudaMemset(p, 0, L.total)) || (e = cudaDeviceSynchronize())) {
    cudaFree(p);
    return cuda_status(e);
  }
  cudaIpcMemHandle_t h;
  if (world > 1 && (e = cudaIpcGetMemHandle(&h, p))) {
    cudaFree(p);
    return cuda_status(e);
  }
  if (world == 1) std::memset(&h, 0, sizeof h);
  dfk_tp_group *g = new (std::nothrow) dfk_tp_group;
  if (!g) {
    cudaFree(p);
    return tp_fail(DFK_ERR_CUDA, "out of host memory");
  }
  g->world = world;
  g->rank = rank;
  g->bmax = max_B;
  g->d_model = d_model;
  g->dev = dev;
  g->own = p;
  g->buf[rank] = p;
  std::memcpy(handle, &h, sizeof h);
  *out = g;
  return DFK_OK;
}

int dfk_tp_group_connect(dfk_tp_group *g, const void *handles) {
  if (!g || (!handles && g->world > 1)) return tp_fail(DFK_ERR_INVALID_ARG, "null pointer");
  if (g->connected) return DFK_OK;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != g->dev) return tp_fail(DFK_ERR_INVALID_ARG, "the group's device is not current");
  const char *hb = static_cast<const char *>(handles);
  for (int r = 0; r < g->world; ++r) {
    if (r == g->rank) continue;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, hb + static_cast<size_t>(r) * sizeof h, sizeof h);
    void *p = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e) {
      for (int q = 0; q < r; ++q)
        if (g->opened[q]) {
          cudaIpcCloseMemHandle(g->buf[q]);
          g->opened[q] = false;
          g->buf[q] = nullptr;
        }
      return cuda_status(e);
    }
    g->buf[r] = p;
    g->opened[r] = true;
  }
  g->connected = true;
  return DFK_OK;
}

int dfk_tp_down_proj_allreduce(dfk_tp_group *g, const void *h, const void *w_down_shard,
                               void *y, int B, int d_model, int d_ff_shard, void *stream) {
  if (!g) return tp_fail(DFK_ERR_INVALID_ARG, "group is NULL");
  if (!g->connected) return tp_fail(DFK_ERR_INVALID_ARG, "group is not connected");
  if (d_model != g->d_model)
    return tp_fail(DFK_ERR_UNSUPPORTED_SHAPE, "d_model differs from the group's");
  dfk::TpLaunch a{};
  a.world = g->world;
  a.rank0 = g->rank;
  a.ranks_here = 1;
  a.h = h;
  a.w = w_down_shard;
  a.y = y;
  a.B = B;
  a.d_model = d_model;
  a.d_ff_shard = d_ff_shard;
  a.bmax = g->bmax;
  for (int r = 0; r < g->world; ++r) a.buf[r] = g->buf[r];
  a.ctl = g->own;
  a.cooperative = false;
  return dfk::launch_tp_down(a, static_cast<cudaStream_t>(stream));
}

int dfk_tp_group_destroy(dfk_tp_group *g) {
  if (!g) return DFK_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(g->dev);
  cudaDeviceSynchronize();
  for (int r = 0; r < g->world; ++r)
    if (g->opened[r]) cudaIpcCloseMemHandle(g->buf[r]);
  cudaFree(g->own);
  cudaGetLastError();
  if (prev >= 0) cudaSetDevice(prev);
  delete g;
  return DFK_OK;
}

int dfk_tp_down_proj_allreduce_emulated(int world, const void *h_all, const void *w_all,
                                        void *y_all, int B, int d_model, int d_ff_shard,
                                        void *stream) {
  if (world < 1 || world > dfk::TP_MAX_RANKS)
    return tp_fail(DFK_ERR_INVALID_ARG, "world must be 1..8");
  if (B < 0 || B > 64 || d_model <= 0 || d_model % 8)
    return tp_fail(DFK_ERR_UNSUPPORTED_SHAPE, "need 0 <= B <= 64 and d_model % 8 == 0");
  if (B == 0) return DFK_OK;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dfk::TpLayout L = dfk::tp_layout(world, 64, d_model);
  void *base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_emu_mu);
    Emu &em = g_emu[std::make_tuple(dev, world, d_model)];
    if (!em.base) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        return tp_fail(DFK_ERR_NO_VARIANT, "make one emulated call before stream capture");
      }
      if ((e = cudaMalloc(&em.base, L.total * world))) return cuda_status(e);
      if ((e = cudaMemset(em.base, 0, L.total * world)) || (e = cudaDeviceSynchronize())) {
        cudaFree(em.base);
        em.base = nullptr;
        return cuda_status(e);
      }
      em.bmax = 64;
    }
    base = em.base;
  }
  dfk::TpLaunch a{};
  a.world = world;
  a.rank0 = 0;
  a.ranks_here = world;
  a.h = h_all;
  a.w = w_all;
  a.y = y_all;
  a.B = B;
  a.d_model = d_model;
  a.d_ff_shard = d_ff_shard;
  a.bmax = 64;
  for (int r = 0; r < world; ++r) a.buf[r] = static_cast<char *>(base) + L.total * r;
  a.ctl = base;  // one grid: one call counter
  a.cooperative = true;
  return dfk::launch_tp_down(a, s);
}

}  // extern "C"
