// dfk_api.cu -- the C ABI of libdfk.so: argument validation, work
// partitioning, TMA descriptor cache, the profiler-driven variant scheduler
// and the launches.  Declarations and argument contracts: include/dfk.h.
//
// Scheduler ("Deep Kernel Fusion for Transformer Decoding", episode
// description: profiler-driven runtime scheduling across row-major and
// column-major kernel variants; "Deep Kernel Fusion for Transformers",
// abstract: the fused kernel is paired with a kernel scheduler): on the
// first call for a (device, op, B, d_model, d_ff, layout) the candidate
// variants are timed with CUDA events on the caller's stream (L2 flushed,
// then a short burst of back-to-back launches per sample), and the fastest
// is cached.  During stream capture
// nothing is timed: a cached winner or the heuristic default is used.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "cc_engine.cuh"
#include "cc_key.h"
#include "dfk.h"
#include "launch_util.h"
#include "tc_engine.cuh"
#include "tc_key.h"
#include "tf8_engine.cuh"
#include "tf8_key.h"
#include "tf8mma_engine.cuh"
#include "tp_internal.h"
#include "pstack_engine.cuh"

// Device status block: word 0 = error bits (bit 0 = a pipeline wait in some
// kernel gave up, bit 1 = a bounds check of the checked build failed),
// word 1 = the site of the first failed bounds check, words 2-3 = the
// pipeline-wait limit in ns (0 = default).
__device__ __align__(16) unsigned g_dfk_err[dfk::STATUS_WORDS];

namespace dfk {

// ---------------------------------------------------------------- errors

static thread_local std::string t_last_error;

static int fail(int status, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

static int cuda_fail(cudaError_t e, const char *what) {
  return fail(DFK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool env_flag(const char *name, bool dflt) {
  const char *v = getenv(name);
  if (!v || !*v) return dflt;
  return !(v[0] == '0' || v[0] == 'n' || v[0] == 'N' || v[0] == 'f' || v[0] == 'F');
}

static int env_int(const char *name, int dflt) {
  const char *v = getenv(name);
  if (!v || !*v) return dflt;
  return atoi(v);
}

static void log_msg(const char *fmt, ...) {
  if (!env_flag("DFK_LOG", false)) return;
  va_list ap;
  va_start(ap, fmt);
  fprintf(stderr, "[dfk] ");
  vfprintf(stderr, fmt, ap);
  fprintf(stderr, "\n");
  va_end(ap);
}

// ---------------------------------------------------------------- kernels table

const void *cc_find_kernel(int key) {
  const void *f = nullptr;
  if ((f = cc_lookup_row(key))) return f;
  if ((f = cc_lookup_col(key))) return f;
  if ((f = cc_lookup_il(key))) return f;
  if ((f = cc_lookup_gemv_a(key))) return f;
  if ((f = cc_lookup_gemv_b(key))) return f;
  if ((f = cc_lookup_fp8_gate_up(key))) return f;
  if ((f = cc_lookup_fp8_gemv_a(key))) return f;
  if ((f = cc_lookup_fp8_gemv_b(key))) return f;
  if ((f = cc_lookup_qkv_a(key))) return f;
  if ((f = cc_lookup_qkv_b(key))) return f;
  return nullptr;
}

// ---------------------------------------------------------------- devices

struct DeviceState {
  bool init = false;
  int sms = 0;
  int major = 0, minor = 0;
  int smem_optin = 0;
  int l2_bytes = 0;
  unsigned *err = nullptr;
};

static std::mutex g_mu;
static std::map<int, DeviceState> g_dev;

static int current_device(DeviceState **out, int *dev_out = nullptr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(DFK_ERR_ARCH, "no CUDA device: %s", cudaGetErrorString(e));
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &st = g_dev[dev];
  if (!st.init) {
    if ((e = cudaDeviceGetAttribute(&st.major, cudaDevAttrComputeCapabilityMajor, dev)) ||
        (e = cudaDeviceGetAttribute(&st.minor, cudaDevAttrComputeCapabilityMinor, dev)) ||
        (e = cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev)) ||
        (e = cudaDeviceGetAttribute(&st.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                    dev)) ||
        (e = cudaDeviceGetAttribute(&st.l2_bytes, cudaDevAttrL2CacheSize, dev))) {
      cudaGetLastError();
      return fail(DFK_ERR_ARCH, "device query failed: %s", cudaGetErrorString(e));
    }
    if (st.major != 10)
      return fail(DFK_ERR_ARCH, "device %d is sm_%d%d; this library runs on sm_100 only", dev,
                  st.major, st.minor);
    if ((e = cudaGetSymbolAddress(reinterpret_cast<void **>(&st.err), g_dfk_err))) {
      cudaGetLastError();
      return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    }
    st.init = true;
  }
  *out = &st;
  if (dev_out) *dev_out = dev;
  return DFK_OK;
}

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn g_encode = nullptr;

static int get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return DFK_OK;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    cudaGetLastError();
    return fail(DFK_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  }
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return DFK_OK;
}

// key: pointer, rank, dims[3], strides[2], box[3], swizzle, element type
using MapKey = std::tuple<uintptr_t, int, uint64_t, uint64_t, uint64_t, uint64_t, uint64_t,
                          uint32_t, uint32_t, uint32_t, int, int>;
static std::map<MapKey, CUtensorMap> g_maps;

// Tensor map of rank 2 or 3 (bf16 elements, or bytes for FP8 weights):
// dims[0] contiguous elements, strides in bytes for dims 1.., box extents,
// 128-byte swizzle or none, zero fill outside the tensor.
static int tensor_map(const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
                      const uint32_t *box, bool sw128, CUtensorMap *out,
                      CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  int rc = get_encoder();
  if (rc) return rc;
  MapKey key{reinterpret_cast<uintptr_t>(ptr), rank, dims[0], dims[1], rank > 2 ? dims[2] : 0,
             strides[0], rank > 2 ? strides[1] : 0, box[0], box[1], rank > 2 ? box[2] : 0,
             sw128 ? 1 : 0, static_cast<int>(dt)};
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return DFK_OK;
    }
  }
  CUtensorMap m;
  cuuint64_t d[3] = {dims[0], dims[1], rank > 2 ? dims[2] : 1};
  cuuint64_t st[2] = {strides[0], rank > 2 ? strides[1] : 0};
  cuuint32_t bx[3] = {box[0], box[1], rank > 2 ? box[2] : 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(&m, dt, static_cast<cuuint32_t>(rank),
                        const_cast<void *>(ptr), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(DFK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d), rank %d dims %llu x %llu "
                "box %u x %u", static_cast<int>(r), rank, static_cast<unsigned long long>(d[0]),
                static_cast<unsigned long long>(d[1]), bx[0], bx[1]);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps[key] = m;
  *out = m;
  return DFK_OK;
}

// 2-D tensor map: `inner` elements per row, `outer` rows, `pitch` bytes
// between rows, box of box_inner x box_outer.
static int tensor_map_2d(const void *ptr, uint64_t inner, uint64_t outer, uint64_t pitch,
                         uint32_t box_inner, uint32_t box_outer, CUtensorMap *out,
                         bool sw128 = false,
                         CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {pitch};
  const uint32_t box[2] = {box_inner, box_outer};
  return tensor_map(ptr, 2, dims, strides, box, sw128, out, dt);
}

// ---------------------------------------------------------------- variants

enum { CLS_GATE_UP = 0, CLS_GEMV = 1 };

struct VDef {
  int id;
  int cls;
  int family;
  int jpt, bt, ksplit, nt;
  int nbank;  // tensor core: independent TMEM accumulator banks per output
  int pair;   // CUDA core: FMAs issued in pairs (fma.rn.f32x2)
  int full;   // tensor core: CTAs own full 128-row M tiles (fewer CTAs than SMs)
  int e4m3mma;  // tensor core, FP8 weights only: E4M3 MMA on the codes (kind::f8f6f4)
};

static const int kJB[][2] = {{4, 1}, {4, 2}, {4, 4}, {2, 1}, {2, 2}, {2, 4}, {2, 8}};

static const std::vector<VDef> &variants() {
  static std::vector<VDef> v = [] {
    std::vector<VDef> t;
    int id = 1;
    for (int pr : {0, 1})
      for (int nt : {1, 2, 4})
        for (auto &jb : kJB)
          t.push_back({id++, CLS_GATE_UP, DFK_FAMILY_CUDA_CORE, jb[0], jb[1], 1, nt, 1, pr, 0});
    for (int pr : {0, 1})
      for (int nt : {1, 2, 4})
        for (int ks : {1, 2, 4, 8})
          for (auto &jb : kJB)
            t.push_back({id++, CLS_GEMV, DFK_FAMILY_CUDA_CORE, jb[0], jb[1], ks, nt, 1, pr, 0});
    // tensor-core family: token tile chosen from B at launch (16 / 32 / 64)
    // gate/up: rows spread over every SM, or full 128-row tiles
    for (int fu : {0, 1})
      for (int nt : {1, 2})
        t.push_back({id++, CLS_GATE_UP, DFK_FAMILY_TENSOR_CORE, 0, 64, 1, nt, 1, 0, fu});
    // GEMV: k-split = reduction slices across CTAs (split-K with a workspace)
    for (int ks : {1, 2, 4})
      for (int nt : {1, 2, 4, 8})
        t.push_back({id++, CLS_GEMV, DFK_FAMILY_TENSOR_CORE, 0, 64, ks, nt, 1, 0, 0});
    // FP8 weights only: the E4M3 MMA on the codes (activations as E4M3 terms)
    t.push_back({id++, CLS_GATE_UP, DFK_FAMILY_TENSOR_CORE, 0, 64, 1, 1, 1, 0, 0, 1});
    for (int ks : {1, 2, 4})
      t.push_back({id++, CLS_GEMV, DFK_FAMILY_TENSOR_CORE, 0, 64, ks, 1, 1, 0, 0, 1});
    // ... with two 128-wide k tiles per ring stage
    t.push_back({id++, CLS_GATE_UP, DFK_FAMILY_TENSOR_CORE, 0, 64, 1, 2, 1, 0, 0, 1});
    for (int ks : {1, 2, 4})
      t.push_back({id++, CLS_GEMV, DFK_FAMILY_TENSOR_CORE, 0, 64, ks, 2, 1, 0, 0, 1});
    // GEMV in full 128-row tiles (every MMA row used), k split 0 = as many
    // slices as fill the SMs: ceil(N / 128) row blocks x floor(SMs / blocks)
    for (int nt : {1, 2, 4, 8})
      t.push_back({id++, CLS_GEMV, DFK_FAMILY_TENSOR_CORE, 0, 64, 0, nt, 1, 0, 1, 0});
    // FP8 weights, up to 16 tokens: the E4M3 MMA with the activation terms
    // derived inside the kernel (no prep kernel)
    for (int nt : {1, 2}) {
      t.push_back({id++, CLS_GATE_UP, DFK_FAMILY_TENSOR_CORE, 0, 64, 1, nt, 1, 0, 0, 2});
      for (int ks : {1, 2, 4})
        t.push_back({id++, CLS_GEMV, DFK_FAMILY_TENSOR_CORE, 0, 64, ks, nt, 1, 0, 0, 2});
    }
    return t;
  }();
  return v;
}

// Variants that can run FP8 weights: CUDA-core ones, and tensor-core ones with
// one k tile per stage whose rows are spread over the SMs.
static bool fp8_capable(const VDef &d) {
  return d.family == DFK_FAMILY_CUDA_CORE || (d.nt == 1 && d.full == 0) || d.e4m3mma;
}

// Variants that can run bf16 weights: all but the E4M3-MMA ones.
static bool bf16_capable(const VDef &d) { return d.e4m3mma == 0; }

static const VDef *find_variant(int id) {
  for (const VDef &d : variants())
    if (d.id == id) return &d;
  return nullptr;
}

static int next_pow2(int b) {
  int p = 1;
  while (p < b) p <<= 1;
  return p;
}

// Token tile a variant family uses for batch B (largest compiled tile for
// its j-per-thread: 4 tokens with 4 rows per thread, 8 with 2).
static int bt_for(int B, int jpt) { return std::min(next_pow2(std::max(B, 1)), jpt == 4 ? 4 : 8); }

// ---------------------------------------------------------------- CUDA-core plan

struct CcPlan {
  const void *fn = nullptr;
  int grid = 0, block = 0;
  size_t smem = 0;
  int r_lo = 0;
  bool xf32 = true;
  CcParams p{};
};

static int ceil_div(int a, int b) { return (a + b - 1) / b; }
static int round_up(int a, int b) { return ceil_div(a, b) * b; }

// L2 bytes (over the whole grid) that a weight-streaming kernel prefetches
// ahead of its shared-memory ring while it waits on the previous kernel; a
// fraction of the 126 MB L2, so the boxes are still there when loaded.
static constexpr long long kPrefetchBytes = 48LL << 20;

// Where the prefetch pays (measured on the 8B shapes, back-to-back calls):
// a bf16 single-matrix GEMV whose weights are at least twice the budget (the
// down projection, 117 MB: 0.5-2 us saved at 1-64 tokens).  It was neutral
// to harmful where the budget covers most of the weights (packed QKV, 50 MB;
// FP8 down, 59 MB: up to 2 us lost) and on the fused gate/up (up to 1.5 us
// lost: the deeper per-CTA sweep is already covered by the ring).
static bool prefetch_pays(int nmat, bool w8, int N, int K) {
  return nmat == 1 && !w8 && 2LL * N * K >= 2 * kPrefetchBytes;
}

// Partition N output rows over the SMs and size the shared-memory ring.
static bool plan_cc(int layout, int nmat, bool norm, bool w8, const VDef &v, int B, int K,
                    int N, const DeviceState &ds, CcPlan *pl, std::string *why) {
  // FP8 weights: 128 codes per 128-byte tile row; the TMA box is at most 256
  // elements wide, so at most two tiles per stage
  const int tk = w8 ? 2 * TILE_K : TILE_K;
  if (w8 && (layout != LAYOUT_ROW || v.nt > 2)) {
    if (why) *why = "FP8 weights: row-major, at most two tiles per stage";
    return false;
  }
  const int g = (layout == LAYOUT_COL) ? 8 : 4;
  const int U = ceil_div(N, g);
  const int smem_cap = std::min(ds.smem_optin, 232448);
  for (int mult = 1; mult <= 16; mult *= 2) {
    const int P = std::min(U, ds.sms * mult);
    const int ubase = U / P, uextra = U % P;
    const int r_hi = (ubase + (uextra ? 1 : 0)) * g;
    const int r_lo = ubase * g;
    if (r_hi > 256) continue;  // TMA box limit
    const int nq = r_hi / v.jpt;
    const int tpt = (layout == LAYOUT_COL) ? 256 * ceil_div(nq, 32) : round_up(8 * nq, 32);
    const int ncons = v.ksplit * tpt;
    // consumers, the producer warp and (RMSNorm) the warp that computes r_b
    const int nthreads = ncons + 32 + (norm ? 32 : 0);
    if (nthreads > CC_MAX_THREADS) continue;
    const int nT = ceil_div(K, tk);
    const int nsteps = ceil_div(nT, v.ksplit * v.nt);
    const int kpad = nsteps * v.ksplit * v.nt * tk;
    const int stage_bytes = v.ksplit * nmat * r_hi * TILE_K * 2 * v.nt;
    const int red_bytes = v.ksplit * (layout == LAYOUT_COL ? NSLOT : 1) * nmat * v.bt * r_hi * 4;
    const int bar_bytes = 256;
    int best_s = 0, best_region = 0;
    bool best_xf32 = true;
    // normalised activations are kept in fp32: only the fp32 store is allowed then
    for (int xf = 1; xf >= (norm ? 1 : 0); --xf) {
      const int xs_bytes = v.bt * kpad * (xf ? 4 : 2);
      const int g_bytes = 0;  // (gamma is multiplied in as x is loaded)
      const int region = round_up(std::max(xs_bytes + g_bytes, red_bytes), 128);
      const int avail = smem_cap - region - bar_bytes;
      const int S = avail > 0 ? std::min(8, avail / stage_bytes) : 0;
      if (xf && S >= 4) { best_s = S; best_region = region; best_xf32 = true; break; }
      if (S > best_s) { best_s = S; best_region = region; best_xf32 = xf != 0; }
    }
    if (best_s < 2) {
      if (why) *why = "shared memory too small for two ring stages";
      continue;
    }
    const int key = DFK_CC_KEY(layout, nmat, v.jpt, v.bt, v.ksplit, best_xf32 ? 1 : 0,
                               norm ? 1 : 0, v.pair ? 1 : 0) | (w8 ? DFK_CC_KEY_W8 : 0);
    const void *fn = cc_find_kernel(key);
    if (!fn) {
      if (why) *why = "variant not compiled for this layout";
      return false;
    }
    pl->fn = fn;
    pl->grid = P;
    pl->block = nthreads;
    pl->r_lo = r_lo;
    pl->xf32 = best_xf32;
    CcParams &p = pl->p;
    p = CcParams{};
    p.K = K;
    p.N = N;
    p.B = B;
    p.nt = v.nt;
    p.nsteps = nsteps;
    p.kpad = kpad;
    p.granule = g;
    p.ubase = ubase;
    p.uextra = uextra;
    p.r_hi = r_hi;
    p.stages = best_s;
    p.stage_bytes = stage_bytes;
    p.npass = ceil_div(B, v.bt);
    p.tpt = tpt;
    p.xs_off = best_s * stage_bytes;
    p.g_off = p.xs_off + v.bt * kpad * (best_xf32 ? 4 : 2);
    p.bar_off = p.xs_off + best_region;
    // single-matrix GEMV: L2 prefetch of the steps after the ring fill
    p.pf_steps = !prefetch_pays(nmat, w8, N, K)
                     ? 0
                     : static_cast<int>(std::max(0LL, std::min<long long>(
                                 p.npass * nsteps - best_s,
                                 kPrefetchBytes / P / stage_bytes)));
    pl->smem = static_cast<size_t>(p.bar_off) + bar_bytes;
    return true;
  }
  if (why && why->empty()) *why = "no partition fits the thread / TMA-box limits";
  return false;
}

static std::mutex g_attr_mu;
static std::map<std::pair<int, const void *>, bool> g_attr_done;

static int ensure_smem_attr(int dev, const void *fn) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  auto k = std::make_pair(dev, fn);
  if (g_attr_done.count(k)) return DFK_OK;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaFuncSetAttribute");
  }
  g_attr_done[k] = true;
  return DFK_OK;
}

struct CcCall {
  int layout;      // LAYOUT_ROW / COL / IL
  int nmat;        // 2 fused gate/up, 1 plain GEMV
  bool norm;
  const void *x, *gamma;
  float eps;
  const void *w0, *w1;
  void *out;
  int B, K, N;
  bool w8 = false;               // FP8 E4M3 weights (row-major), per-row scales below
  const float *s0 = nullptr, *s1 = nullptr;
  void *outs[3] = {nullptr, nullptr, nullptr};  // packed QKV: q / k / v parts of the output
  int split[2] = {0, 0};                         // row ranges of the parts
};

static bool pdl_enabled() { return env_flag("DFK_PDL", true); }

static int launch_cc(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used) {
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  CcPlan pl;
  std::string why;
  if (!plan_cc(c.layout, c.nmat, c.norm, c.w8, v, c.B, c.K, c.N, *ds, &pl, &why))
    return fail(DFK_ERR_NO_VARIANT, "variant %d does not fit B=%d K=%d N=%d: %s", v.id, c.B,
                c.K, c.N, why.c_str());
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  CcMaps maps;
  memset(&maps, 0, sizeof maps);
  const int r_hi = pl.p.r_hi, r_lo = pl.r_lo > 0 ? pl.r_lo : pl.p.r_hi;
  const void *w[2] = {c.w0, c.w1};
  const uint32_t kbox = (c.w8 ? 2 * TILE_K : TILE_K) * v.nt;
  for (int m = 0; m < (c.layout == LAYOUT_IL ? 1 : c.nmat); ++m) {
    for (int lo = 0; lo < 2; ++lo) {
      const uint32_t r = lo ? r_lo : r_hi;
      if (c.w8)
        rc = tensor_map_2d(w[m], c.K, c.N, static_cast<uint64_t>(c.K), kbox, r,
                           &maps.m[m * 2 + lo], false, CU_TENSOR_MAP_DATA_TYPE_UINT8);
      else if (c.layout == LAYOUT_ROW)
        rc = tensor_map_2d(w[m], c.K, c.N, static_cast<uint64_t>(c.K) * 2, kbox, r,
                           &maps.m[m * 2 + lo]);
      else if (c.layout == LAYOUT_COL)
        rc = tensor_map_2d(w[m], c.N, c.K, static_cast<uint64_t>(c.N) * 2, r, kbox,
                           &maps.m[m * 2 + lo]);
      else
        rc = tensor_map_2d(w[m], c.K, 2ull * c.N, static_cast<uint64_t>(c.K) * 2, kbox, r,
                           &maps.m[m * 2 + lo]);
      if (rc) return rc;
    }
  }
  CcParams p = pl.p;
  p.x = static_cast<const uint16_t *>(c.x);
  p.gamma = static_cast<const uint16_t *>(c.gamma);
  p.out = static_cast<uint16_t *>(c.out);
  p.scale[0] = c.s0;
  p.scale[1] = c.s1;
  for (int i = 0; i < 3; ++i) p.outs[i] = static_cast<uint16_t *>(c.outs[i]);
  p.split[0] = c.split[0];
  p.split[1] = c.split[1];
  p.err = ds->err;
  p.eps = c.eps;
  void *args[] = {&maps, &p};
  cudaError_t e = launch_kernel(pl.fn, dim3(pl.grid), dim3(pl.block), pl.smem, s, pdl_enabled(),
                                args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "kernel launch");
  }
  if (stages_used) *stages_used = p.stages;
  return DFK_OK;
}

// ---------------------------------------------------------------- tensor-core plan

struct TcPlan {
  const void *fn = nullptr;
  int grid = 0;
  size_t smem = 0;
  int mt = 1;
  TcParams p{};
};

static int pow2_ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Dynamic shared memory of a kernel that follows its prep kernel (RMSNorm
// hi/lo rows, FP8 activation terms) in the stream.  The prep kernel's CTAs
// (one per token slot) become resident while the previous kernel runs and
// stay until their results are written; an SM holding one must still take a
// CTA of the main kernel, or that CTA starts its weight stream only after the
// prep CTA has left (up to 64 SMs late, one per token slot).  228 KB per SM,
// less 1 KB per resident CTA and the prep kernel's 1 KB static array, leaves
// 230,400 bytes.  (The prep kernels' register budgets are capped for the same
// reason.)
constexpr int SMEM_BESIDE_PREP = 233472 - 2 * 1024 - 1024;

// One CTA per SM over rows [j0, j0 + r) for the whole reduction; each
// 128-row MMA tile reads 128 rows from shared memory starting at its A
// tile, so the space behind the last A tile of the ring is kept readable.
// `prepped`: the RMSNorm activations come from the prep kernel (mode 2)
// instead of the in-kernel transform (mode 1).
static bool plan_tc(int layout, int nmat, bool norm, const VDef &v, int B, int K, int N,
                    const DeviceState &ds, TcPlan *pl, std::string *why, bool prepped = true) {
  if (v.e4m3mma) {
    if (why) *why = "E4M3-MMA variants run FP8 weights only";
    return false;
  }
  if (norm && nmat == 1 && v.ksplit != 1 && !prepped) {
    if (why) *why = "RMSNorm with split-K needs the prepared activations (r_b over all of K)";
    return false;
  }
  const bool colm = layout == LAYOUT_COL;
  const bool full = colm || v.full != 0;  // 128 rows per CTA
  if (colm && nmat != 2) {
    if (why) *why = "column-major tensor-core kernel is the fused gate/up only";
    return false;
  }
  if (B < 1 || B > 64) {
    if (why) *why = "tensor-core family needs 1 <= B <= 64";
    return false;
  }
  const int bn = B <= 16 ? 16 : (B <= 32 ? 32 : 64);
  const int cap = std::min(ds.smem_optin, (norm && prepped) ? SMEM_BESIDE_PREP : 232448);
  const int nt = v.nt;
  const int ntiles = ceil_div(K, TC_TILE_K);
  // GEMV in full tiles: k slices = SMs per row block (k split 0 = automatic)
  const int kslices = nmat != 1 ? 1
                      : (v.ksplit == 0 ? std::max(1, std::min({ntiles, SPLITK_MAX,
                                                               ds.sms / ceil_div(N, 128)}))
                                       : std::max(1, v.ksplit));
  if (kslices > SPLITK_MAX) {
    if (why) *why = "more than 8 k slices";
    return false;
  }
  if (kslices > 1 && (nmat != 1 || ntiles < kslices)) {
    if (why) *why = "split-K needs a single matrix and at least one k-tile per slice";
    return false;
  }
  for (int mult = 1; mult <= 8; mult *= 2) {
    // row blocks: one per CTA, or (split-K) one per kslices CTAs; column-major:
    // 128 columns per CTA (two full 64-column boxes)
    const int nblocks = full ? ceil_div(N, 128)
                             : (kslices > 1 ? std::min(N, ds.sms / kslices)
                                            : std::min(N, ds.sms * mult));
    if (nblocks < 1) break;
    const int P = nblocks * kslices;
    const int rbase = full ? 128 : N / nblocks, rextra = full ? 0 : N % nblocks;
    const int r_hi = rbase + (rextra ? 1 : 0);
    for (int mt = 1; mt <= (kslices > 1 || full ? 1 : 2); ++mt) {
      if (r_hi > 128 * mt) continue;
      if (mt == 2 && rbase < 2) continue;
      const int hmax = (r_hi + mt - 1) / mt;
      const int rc = full ? 128 : round_up(hmax, 8);
      const int a_bytes = nt * mt * nmat * rc * 128;
      const int xt_bytes = bn * 128 * (norm ? 2 : 1);  // hi rows (+ lo rows)
      const int x_bytes = nt * xt_bytes;
      const int stage = a_bytes + x_bytes;
      const int slack = std::max(0, 16384 - rc * 128 - x_bytes);
      const int nsteps = ceil_div(ceil_div(ntiles, kslices), nt);
      const int kpad = ceil_div(ntiles, nt) * nt * TC_TILE_K;
      const int g_bytes = (norm && !prepped) ? round_up(kpad * 2, 1024) : 0;
      const int fixed = 1024 /* alignment */ + slack + g_bytes + 1024 /* barriers */;
      const int S = std::min(8, (cap - fixed) / stage);
      if (S < 2) continue;
      // accumulator banks per output: the variant's count, as far as TMEM holds
      const int wn = norm ? 2 * bn : bn;  // MMA N: the tokens (hi rows, then lo rows)
      int nbank = std::max(1, v.nbank);
      while (nbank > 1 && mt * nmat * nbank * wn > 512) nbank >>= 1;
      const int cols = pow2_ceil(std::max(32, mt * nmat * nbank * wn));
      if (cols > 512) continue;
      const void *fn = tc_find_kernel(nmat, norm ? (prepped ? 2 : 1) : 0,
                                      layout == LAYOUT_IL ? 2 : (colm ? 1 : 0), mt);
      if (!fn) {
        if (why) *why = "tensor-core kernel not compiled for this case";
        return false;
      }
      pl->fn = fn;
      pl->grid = P;
      pl->mt = mt;
      TcParams &p = pl->p;
      p = TcParams{};
      p.B = B;
      p.K = K;
      p.N = N;
      p.nsteps = nsteps;
      p.nt = nt;
      p.rbase = rbase;
      p.rextra = rextra;
      p.hmax = hmax;
      p.rc = rc;
      p.bn = bn;
      p.stages = S;
      p.stage_bytes = stage;
      p.a_bytes = a_bytes;
      p.xt_bytes = xt_bytes;
      p.tmem_cols = cols;
      p.nbank = nbank;
      p.g_off = S * stage + slack;
      p.bar_off = p.g_off + g_bytes;
      p.ntiles = ntiles;
      p.kslices = kslices;
      p.nblocks = nblocks;
      p.full = full ? 1 : 0;
      // weight boxes prefetched into L2 ahead of the ring while the previous
      // kernel finishes, at most kPrefetchBytes over the grid
      const long long step_w = static_cast<long long>(nmat) * mt * nt * (full ? 128 : hmax) * 128;
      p.pf_steps = !prefetch_pays(nmat, false, N, K)
                       ? 0
                       : static_cast<int>(std::max(0LL, std::min<long long>(
                                   nsteps - S, kPrefetchBytes / P / step_w)));
      pl->smem = 1024 + static_cast<size_t>(p.bar_off) + 1024;
      return true;
    }
    if (kslices > 1 || full) break;  // these partitions do not depend on `mult`
  }
  if (why) *why = "no tensor-core partition fits shared memory";
  return false;
}

// ---- split-K workspace: one per (device, stream), grown on demand outside
// stream capture; the counter region is zeroed when allocated and every
// kernel leaves its counters at 0.
struct Workspace {
  void *base = nullptr;
  size_t bytes = 0;
};
static std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

static bool stream_capturing(cudaStream_t s);

static int get_workspace(int dev, cudaStream_t s, size_t part_bytes, size_t counter_bytes,
                         float **part, unsigned **counters) {
  const size_t part_round = (part_bytes + 255) & ~static_cast<size_t>(255);
  const size_t need = part_round + counter_bytes;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace &w = g_ws[std::make_pair(dev, s)];
  if (w.bytes < need) {
    if (stream_capturing(s))
      return fail(DFK_ERR_NO_VARIANT, "split-K workspace must be allocated before capture "
                  "(make one call of this shape on the stream first)");
    if (w.base) {
      cudaStreamSynchronize(s);
      cudaFree(w.base);
      w.base = nullptr;
      w.bytes = 0;
    }
    const size_t grow = std::max(need, static_cast<size_t>(8) << 20);
    cudaError_t e = cudaMalloc(&w.base, grow);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "cudaMalloc (split-K workspace)");
    }
    e = cudaMemsetAsync(w.base, 0, grow, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "zeroing the split-K workspace");
    }
    w.bytes = grow;
  }
  // counters at the end of the buffer: stable across shapes
  *part = static_cast<float *>(w.base);
  *counters = reinterpret_cast<unsigned *>(static_cast<char *>(w.base) + w.bytes - counter_bytes);
  if (part_round > w.bytes - counter_bytes) return fail(DFK_ERR_CUDA, "workspace layout");
  return DFK_OK;
}

static int get_term_buffer(int dev, cudaStream_t s, size_t bytes, void **out);

// Tensor-core RMSNorm from the prep kernel (mode 2): for the fused gate/up
// above 32 tokens (measured on the 8B layer: 66 -> 54 us at 64 tokens; at 16
// and 32 tokens the in-kernel transform is ~3 us faster, the prep latency not
// hidden), and always for the one-matrix GEMV (packed QKV), where it also
// allows split-K across CTAs (r_b over all of K).
static bool tc_prepared(const CcCall &c) { return c.norm && (c.B > 32 || c.nmat == 1); }

static int launch_tc(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used) {
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  // RMSNorm: prepared activations (tc_prepared) in the per-stream buffer; the
  // in-kernel transform when the buffer cannot be had (stream capture before
  // any call of this shape on the stream)
  void *xg = nullptr;
  bool prepped = false;
  size_t xg_bytes = 0;
  if (tc_prepared(c)) {
    const int bn = c.B <= 16 ? 16 : (c.B <= 32 ? 32 : 64);
    xg_bytes = static_cast<size_t>(ceil_div(c.K, TC_TILE_K)) * 2 * bn * TC_TILE_K * 2;
    rc = get_term_buffer(dev, s, xg_bytes + 64 * sizeof(float), &xg);
    if (rc == DFK_OK) prepped = true;
    else if (rc == DFK_ERR_NO_VARIANT && stream_capturing(s)) log_msg("RMSNorm prep buffer "
             "missing during capture: transforming in the kernel");
    else return rc;
    if (!prepped && c.nmat == 1 && v.ksplit != 1) {
      VDef whole = v;  // the in-kernel transform cannot split K
      whole.ksplit = 1;
      return launch_tc(c, whole, s, stages_used);
    }
  }
  TcPlan pl;
  std::string why;
  if (!plan_tc(c.layout, c.nmat, c.norm, v, c.B, c.K, c.N, *ds, &pl, &why, prepped))
    return fail(DFK_ERR_NO_VARIANT, "variant %d does not fit B=%d K=%d N=%d: %s", v.id, c.B,
                c.K, c.N, why.c_str());
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  TcMaps maps;
  memset(&maps, 0, sizeof maps);
  const int hmax = pl.p.hmax;
  for (int lo = 0; lo < 2; ++lo) {
    const uint32_t hgt = static_cast<uint32_t>(std::max(1, hmax - lo));
    if (c.layout == LAYOUT_COL) {
      // [K][N] weights: boxes of 64 columns x 64 k rows
      if ((rc = tensor_map_2d(c.w0, c.N, c.K, static_cast<uint64_t>(c.N) * 2, 64, TC_TILE_K,
                              &maps.wg[lo], true)) ||
          (rc = tensor_map_2d(c.w1, c.N, c.K, static_cast<uint64_t>(c.N) * 2, 64, TC_TILE_K,
                              &maps.wu[lo], true)))
        return rc;
    } else if (c.layout == LAYOUT_IL) {
      const uint64_t dims[3] = {static_cast<uint64_t>(c.K), 2, static_cast<uint64_t>(c.N)};
      const uint64_t strides[2] = {static_cast<uint64_t>(c.K) * 2,
                                   static_cast<uint64_t>(c.K) * 4};
      const uint32_t box[3] = {TC_TILE_K, 1, hgt};
      if ((rc = tensor_map(c.w0, 3, dims, strides, box, true, &maps.wg[lo]))) return rc;
    } else {
      if ((rc = tensor_map_2d(c.w0, c.K, c.N, static_cast<uint64_t>(c.K) * 2, TC_TILE_K, hgt,
                              &maps.wg[lo], true)))
        return rc;
      if (c.nmat == 2 &&
          (rc = tensor_map_2d(c.w1, c.K, c.N, static_cast<uint64_t>(c.K) * 2, TC_TILE_K, hgt,
                              &maps.wu[lo], true)))
        return rc;
    }
  }
  if (prepped) {
    // prepared rows: [ntiles][2 bn][64] bf16, one box of 2 bn rows per k tile
    if ((rc = tensor_map_2d(xg, TC_TILE_K, static_cast<uint64_t>(pl.p.ntiles) * 2 * pl.p.bn,
                            TC_TILE_K * 2, TC_TILE_K, 2 * pl.p.bn, &maps.x, true)))
      return rc;
  } else if ((rc = tensor_map_2d(c.x, c.K, c.B, static_cast<uint64_t>(c.K) * 2, TC_TILE_K,
                                 pl.p.bn, &maps.x, true))) {
    return rc;
  }
  TcParams p = pl.p;
  p.out = static_cast<uint16_t *>(c.out);
  p.gamma = static_cast<const uint16_t *>(c.gamma);
  p.rinv = prepped ? reinterpret_cast<const float *>(static_cast<char *>(xg) + xg_bytes)
                   : nullptr;
  for (int i = 0; i < 3; ++i) p.outs[i] = static_cast<uint16_t *>(c.outs[i]);
  p.split[0] = c.split[0];
  p.split[1] = c.split[1];
  p.err = ds->err;
  p.eps = c.eps;
  if (p.kslices > 1) {
    const size_t part_bytes =
        static_cast<size_t>(p.kslices) * p.nblocks * p.bn * 128 * sizeof(float);
    // counters: a fixed region sized for the largest partition (one per SM)
    const size_t counter_bytes = static_cast<size_t>(ds->sms) * 8 * sizeof(unsigned);
    if ((rc = get_workspace(dev, s, part_bytes, counter_bytes, &p.part, &p.counters))) {
      if (rc != DFK_ERR_NO_VARIANT || !stream_capturing(s)) return rc;
      // being captured on a stream without a workspace (none may be allocated
      // now): the same variant without the split
      VDef whole = v;
      whole.ksplit = 1;
      log_msg("split-K workspace missing during capture: launching without the split");
      return launch_tc(c, whole, s, stages_used);
    }
  }
  if (prepped) {
    TcPrepParams pp{};
    pp.x = static_cast<const uint16_t *>(c.x);
    pp.gamma = static_cast<const uint16_t *>(c.gamma);
    pp.xg = static_cast<uint16_t *>(xg);
    pp.rinv = const_cast<float *>(p.rinv);
    pp.B = c.B;
    pp.K = c.K;
    pp.bn = p.bn;
    pp.ntiles = p.ntiles;
    pp.eps = c.eps;
    pp.err = ds->err;
    void *pargs[] = {&pp};
    // one CTA per token slot
    cudaError_t e = launch_kernel(tc_norm_prep_fn(), dim3(p.bn), dim3(TC_PREP_THREADS), 0, s,
                                  pdl_enabled(), pargs);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "RMSNorm prep kernel launch");
    }
  }
  void *args[] = {&maps, &p};
  cudaError_t e = launch_kernel(pl.fn, dim3(pl.grid), dim3(TC_THREADS), pl.smem, s,
                                pdl_enabled(), args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "tensor-core kernel launch");
  }
  if (stages_used) *stages_used = p.stages;
  return DFK_OK;
}

static int check_gemv(const void *x, const void *w, const void *out, int B, int K, int N,
                      int variant);

// The split-K tensor-core down projection on caller-provided scratch: a
// fixed configuration (no timing), no workspace of its own.  Used by the
// entry point for callers that cannot allocate (noalloc.cu).  With
// clear_counters the row-block counters are zeroed on the stream right
// before the launch, after every argument has been checked (an invalid call
// enqueues nothing).
int down_proj_with_scratch(const void *h, const void *w_down, void *y, int B, int d_model,
                           int d_ff, float *part, size_t part_capacity, unsigned *counters,
                           size_t counter_capacity, bool clear_counters, cudaStream_t s) {
  int rc = check_gemv(h, w_down, y, B, d_ff, d_model, 0);
  if (rc || B == 0) return rc;
  DeviceState *ds;
  int dev;
  if ((rc = current_device(&ds, &dev))) return rc;
  const CcCall c{LAYOUT_ROW, 1, false, h, nullptr, 0.f, w_down, nullptr, y, B, d_ff, d_model};
  // preferred split configurations, most parallel first
  static const int kPrefs[][2] = {{4, 2}, {4, 1}, {2, 2}, {2, 1}};
  TcPlan pl;
  bool found = false;
  for (const auto &pref : kPrefs) {
    for (const VDef &d : variants()) {
      if (d.cls != CLS_GEMV || d.family != DFK_FAMILY_TENSOR_CORE || d.ksplit != pref[0] ||
          d.nt != pref[1])
        continue;
      if (plan_tc(c.layout, 1, false, d, B, c.K, c.N, *ds, &pl, nullptr) && pl.p.kslices > 1) {
        found = true;
        break;
      }
    }
    if (found) break;
  }
  if (!found)
    return fail(DFK_ERR_NO_VARIANT, "no split-K configuration fits B=%d d_model=%d d_ff=%d", B,
                d_model, d_ff);
  const size_t part_bytes =
      static_cast<size_t>(pl.p.kslices) * pl.p.nblocks * pl.p.bn * 128 * sizeof(float);
  const size_t counter_bytes = static_cast<size_t>(pl.p.nblocks) * sizeof(unsigned);
  if (part_bytes > part_capacity || counter_bytes > counter_capacity)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE,
                "B=%d d_model=%d needs %zu bytes of partial sums and %zu of counters; the "
                "static scratch holds %zu and %zu",
                B, d_model, part_bytes, counter_bytes, part_capacity, counter_capacity);
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  TcMaps maps;
  memset(&maps, 0, sizeof maps);
  for (int lo = 0; lo < 2; ++lo) {
    const uint32_t hgt = static_cast<uint32_t>(std::max(1, pl.p.hmax - lo));
    if ((rc = tensor_map_2d(w_down, c.K, c.N, static_cast<uint64_t>(c.K) * 2, TC_TILE_K, hgt,
                            &maps.wg[lo], true)))
      return rc;
  }
  if ((rc = tensor_map_2d(h, c.K, c.B, static_cast<uint64_t>(c.K) * 2, TC_TILE_K, pl.p.bn,
                          &maps.x, true)))
    return rc;
  TcParams p = pl.p;
  p.out = static_cast<uint16_t *>(y);
  p.gamma = nullptr;
  p.err = ds->err;
  p.eps = 0.f;
  p.part = part;
  p.counters = counters;
  if (clear_counters) {
    cudaError_t e = cudaMemsetAsync(counters, 0, counter_bytes, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "zeroing the split-K counters");
    }
  }
  void *args[] = {&maps, &p};
  cudaError_t e = launch_kernel(pl.fn, dim3(pl.grid), dim3(TC_THREADS), pl.smem, s,
                                pdl_enabled(), args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "tensor-core kernel launch");
  }
  return DFK_OK;
}

static bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// ---------------------------------------------------------------- tensor parallel

int report_error(int status, const char *msg) { return fail(status, "%s", msg); }

TpLayout tp_layout(int world, int bmax, int d_model) {
  TpLayout l;
  l.recv_bytes = static_cast<size_t>(2) * world * bmax * d_model * sizeof(float);
  l.flags_off = (l.recv_bytes + 255) & ~static_cast<size_t>(255);
  l.seq_off = l.flags_off + static_cast<size_t>(TP_MAX_BLOCKS) * world * 8;
  l.exit_off = l.seq_off + 8;
  l.total = (l.exit_off + 8 + 255) & ~static_cast<size_t>(255);
  return l;
}

// The tensor-parallel down projection with the all-reduce fused in: the
// tensor-core GEMV (no split-K, one CTA per SM over this rank's rows) whose
// epilogue exchanges the fp32 partial sums (tc_engine.cuh, tp_* fields).
int launch_tp_down(const TpLaunch &a, cudaStream_t s) {
  if (a.world < 1 || a.world > TP_MAX_RANKS || a.ranks_here < 1 || a.rank0 < 0 ||
      a.rank0 + a.ranks_here > a.world)
    return fail(DFK_ERR_INVALID_ARG, "bad tensor-parallel group (world %d)", a.world);
  int rc = check_gemv(a.h, a.w, a.y, a.B, a.d_ff_shard, a.d_model, 0);
  if (rc || a.B == 0) return rc;
  if (a.B > a.bmax)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "B=%d exceeds the group's capacity %d", a.B, a.bmax);
  DeviceState *ds;
  int dev;
  if ((rc = current_device(&ds, &dev))) return rc;
  DeviceState sub = *ds;
  sub.sms = ds->sms / a.ranks_here;
  const VDef *v = nullptr;
  for (const VDef &d : variants())
    if (d.cls == CLS_GEMV && d.family == DFK_FAMILY_TENSOR_CORE && bf16_capable(d) &&
        d.ksplit == 1 && d.nt == 2 && d.full == 0)
      v = &d;
  TcPlan pl;
  std::string why;
  if (!v || !plan_tc(LAYOUT_ROW, 1, false, *v, a.B, a.d_ff_shard, a.d_model, sub, &pl, &why))
    return fail(DFK_ERR_NO_VARIANT, "no tensor-parallel plan for B=%d d_model=%d shard=%d: %s",
                a.B, a.d_model, a.d_ff_shard, why.c_str());
  if (pl.grid > sub.sms || pl.grid > TP_MAX_BLOCKS || pl.p.kslices != 1)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "d_model=%d needs %d row blocks per rank; at most %d "
                "fit (one co-resident CTA per block)", a.d_model, pl.grid,
                std::min(sub.sms, TP_MAX_BLOCKS));
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  TcMaps maps;
  memset(&maps, 0, sizeof maps);
  const uint64_t rows = static_cast<uint64_t>(a.ranks_here) * a.d_model;
  for (int lo = 0; lo < 2; ++lo) {
    const uint32_t hgt = static_cast<uint32_t>(std::max(1, pl.p.hmax - lo));
    if ((rc = tensor_map_2d(a.w, a.d_ff_shard, rows, static_cast<uint64_t>(a.d_ff_shard) * 2,
                            TC_TILE_K, hgt, &maps.wg[lo], true)))
      return rc;
  }
  if ((rc = tensor_map_2d(a.h, a.d_ff_shard, static_cast<uint64_t>(a.ranks_here) * a.B,
                          static_cast<uint64_t>(a.d_ff_shard) * 2, TC_TILE_K, pl.p.bn, &maps.x,
                          true)))
    return rc;
  TcParams p = pl.p;
  p.out = static_cast<uint16_t *>(a.y);
  p.err = ds->err;
  p.tp_world = a.world;
  p.tp_rank0 = a.rank0;
  p.tp_blocks = pl.grid;
  p.tp_bmax = a.bmax;
  const TpLayout L = tp_layout(a.world, a.bmax, a.d_model);
  for (int r = 0; r < a.world; ++r) {
    char *b = static_cast<char *>(a.buf[r]);
    if (!b) return fail(DFK_ERR_INVALID_ARG, "rank %d's buffer is not connected", r);
    p.tp_recv[r] = reinterpret_cast<float *>(b);
    p.tp_flags[r] = reinterpret_cast<unsigned long long *>(b + L.flags_off);
  }
  p.tp_seq = reinterpret_cast<unsigned long long *>(static_cast<char *>(a.ctl) + L.seq_off);
  p.tp_exit = reinterpret_cast<unsigned *>(static_cast<char *>(a.ctl) + L.exit_off);
  void *args[] = {&maps, &p};
  cudaError_t e = launch_kernel(pl.fn, dim3(pl.grid * a.ranks_here), dim3(TC_THREADS), pl.smem,
                                s, pdl_enabled() && !a.cooperative, args, 1, a.cooperative);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "tensor-parallel down projection launch");
  }
  return DFK_OK;
}

// ---------------------------------------------------------------- persistent decode step

const void *pstack_fn();

struct PsPlan {
  PsParams p{};
  size_t smem = 0;
  size_t ws_ctl = 0, ws_part = 0;  // workspace: control words, then partial sums
};

// Partition and shared-memory plan of the persistent decode step
// (pstack_engine.cuh) for an L-layer stack on a device with `sms` SMs.
static bool plan_pstack(int L, int B, int D, int F, int sms, int smem_cap, PsPlan *pl,
                        std::string *why, bool col = false) {
  auto no = [&](const char *m) {
    if (why) *why = m;
    return false;
  };
  if (L < 1 || B < 1 || B > PS_BN) return no("need L >= 1 and 1 <= B <= 16");
  if (D % 8 || F % 8) return no("d_model and d_ff must be multiples of 8");
  const int G = sms - sms % PS_KSPLIT;
  if (G < PS_KSPLIT) return no("too few SMs");
  PsParams &p = pl->p;
  p = PsParams{};
  p.L = L;
  p.B = B;
  p.D = D;
  p.F = F;
  p.gu_col = col ? 1 : 0;
  p.gu_rbase = F / G;
  p.gu_rextra = F % G;
  p.gu_hmax = p.gu_rbase + (p.gu_rextra ? 1 : 0);
  if (col) {
    if (ceil_div(F, 128) > G) return no("column-major d_ff needs at most 128 columns per SM");
    p.gu_rc = 128;  // two 64-column boxes per matrix and k tile
  } else {
    if (p.gu_rbase < 1 || p.gu_hmax > 128) return no("d_ff needs 1 .. 128 rows per SM");
    p.gu_rc = round_up(p.gu_hmax, 8);
  }
  p.gu_tiles = ceil_div(D, PS_TILE_K);
  p.dn_nblk = G / PS_KSPLIT;
  p.dn_rbase = D / p.dn_nblk;
  p.dn_rextra = D % p.dn_nblk;
  p.dn_hmax = p.dn_rbase + (p.dn_rextra ? 1 : 0);
  if (p.dn_rbase < 1 || p.dn_hmax > 128) return no("d_model needs 1 .. 128 rows per row block");
  p.dn_rc = round_up(p.dn_hmax, 8);
  p.dn_tiles = ceil_div(F, PS_TILE_K);
  if (p.dn_tiles < PS_KSPLIT) return no("d_ff too short for four reduction slices");
  // k tiles per ring step: 256 / 512 contiguous bytes of each weight row per
  // step (the tensor-core kernels' tuned stage sizes for these phases)
  // (measured: 1 / 2 / 3 gate/up tiles and 1 - 6 down tiles per step, with
  // the ring depth that fits; two and four are the fastest mix)
  p.gu_nt = 2;
  p.dn_nt = 4;
  // a slot: the step's weight tiles, then its activation tiles (gate/up: hi
  // + lo rows each; down: h rows), then the gamma slices of a gate/up step.
  // An MMA reads 128 rows from each weight tile start; the over-read past
  // the weights stays inside the slot.
  const int w_bytes = std::max(p.gu_nt * 2 * p.gu_rc * 128, p.dn_nt * p.dn_rc * 128);
  p.x_off = round_up(w_bytes, 1024);
  p.g_off = p.x_off + std::max(p.gu_nt * PS_ATILE, p.dn_nt * PS_DTILE);
  p.slot_bytes = round_up(p.g_off + p.gu_nt * 128, 1024);
  if (p.slot_bytes < std::max((2 * p.gu_nt - 1) * p.gu_rc * 128, (p.dn_nt - 1) * p.dn_rc * 128) +
                         16384)
    p.slot_bytes = round_up(std::max((2 * p.gu_nt - 1) * p.gu_rc * 128,
                                     (p.dn_nt - 1) * p.dn_rc * 128) + 16384, 1024);
  const int bar_bytes = (4 * 8 + 5) * 8 + 32 + PS_BN * 4;
  const int fixed = 1024 /* alignment */ + round_up(bar_bytes, 128);
  p.S = std::min(8, (smem_cap - fixed) / p.slot_bytes);
  if (p.S < 2) return no("the ring does not fit shared memory");
  p.bar_off = p.S * p.slot_bytes;
  pl->smem = 1024 + static_cast<size_t>(p.bar_off) + round_up(bar_bytes, 128);
  pl->ws_ctl = round_up((2 + 2 * L + p.dn_nblk) * 4, 256);
  pl->ws_part = static_cast<size_t>(PS_KSPLIT) * p.dn_nblk * PS_BN * 128 * sizeof(float);
  return true;
}

static int pstack_step(const void *gamma, float eps, const void *wg, const void *wu, int layout,
                       const void *wd, void *x, void *h_all, void *y_all, void *ws,
                       size_t ws_bytes, int L, int B, int D, int F, cudaStream_t s) {
  if (L < 1 || B < 0 || D <= 0 || F <= 0) return fail(DFK_ERR_INVALID_ARG, "bad sizes");
  if (layout != DFK_W_ROW_MAJOR && layout != DFK_W_COL_MAJOR)
    return fail(DFK_ERR_UNSUPPORTED_LAYOUT, "the decode step takes row- or column-major "
                "gate/up weights");
  const bool col = layout == DFK_W_COL_MAJOR;
  if (!(eps >= 0.f && std::isfinite(eps))) return fail(DFK_ERR_INVALID_ARG, "bad eps");
  if (B == 0) return DFK_OK;
  if (!gamma || !wg || !wu || !wd || !x || !h_all || !y_all || !ws)
    return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if (misaligned(gamma) || misaligned(wg) || misaligned(wu) || misaligned(wd) ||
      misaligned(x) || misaligned(h_all) || misaligned(y_all) || misaligned(ws))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  PsPlan pl;
  std::string why;
  if (!plan_pstack(L, B, D, F, ds->sms, std::min(ds->smem_optin, 232448), &pl, &why, col))
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "persistent decode step: %s", why.c_str());
  if (ws_bytes < pl.ws_ctl + pl.ws_part)
    return fail(DFK_ERR_INVALID_ARG, "workspace of %zu bytes; %zu needed", ws_bytes,
                pl.ws_ctl + pl.ws_part);
  const void *fn = pstack_fn();
  if ((rc = ensure_smem_attr(dev, fn))) return rc;
  PsMaps maps;
  memset(&maps, 0, sizeof maps);
  PsParams &p = pl.p;
  for (int lo = 0; lo < 2; ++lo) {
    const uint32_t gh = static_cast<uint32_t>(std::max(1, p.gu_hmax - lo));
    const uint32_t dh = static_cast<uint32_t>(std::max(1, p.dn_hmax - lo));
    if (col) {
      // [L * D][F]: boxes of 64 columns x 64 k rows
      if ((rc = tensor_map_2d(wg, F, static_cast<uint64_t>(L) * D, static_cast<uint64_t>(F) * 2,
                              64, PS_TILE_K, &maps.wg[lo], true)) ||
          (rc = tensor_map_2d(wu, F, static_cast<uint64_t>(L) * D, static_cast<uint64_t>(F) * 2,
                              64, PS_TILE_K, &maps.wu[lo], true)))
        return rc;
    } else if ((rc = tensor_map_2d(wg, D, static_cast<uint64_t>(L) * F,
                                   static_cast<uint64_t>(D) * 2, PS_TILE_K, gh, &maps.wg[lo],
                                   true)) ||
               (rc = tensor_map_2d(wu, D, static_cast<uint64_t>(L) * F,
                                   static_cast<uint64_t>(D) * 2, PS_TILE_K, gh, &maps.wu[lo],
                                   true))) {
      return rc;
    }
    if ((rc = tensor_map_2d(wd, F, static_cast<uint64_t>(L) * D, static_cast<uint64_t>(F) * 2,
                            PS_TILE_K, dh, &maps.wd[lo], true)))
      return rc;
  }
  // activations (16-row boxes: rows past a layer's B tokens feed ignored MMA
  // columns) and the gammas
  if ((rc = tensor_map_2d(x, D, B, static_cast<uint64_t>(D) * 2, PS_TILE_K, PS_BN, &maps.x,
                          true)) ||
      (rc = tensor_map_2d(y_all, D, static_cast<uint64_t>(L) * B, static_cast<uint64_t>(D) * 2,
                          PS_TILE_K, PS_BN, &maps.y, true)) ||
      (rc = tensor_map_2d(h_all, F, static_cast<uint64_t>(L) * B, static_cast<uint64_t>(F) * 2,
                          PS_TILE_K, PS_BN, &maps.h, true)) ||
      (rc = tensor_map_2d(gamma, D, L, static_cast<uint64_t>(D) * 2, PS_TILE_K, 1, &maps.gam,
                          false)))
    return rc;
  p.gamma = static_cast<const uint16_t *>(gamma);
  p.x = static_cast<uint16_t *>(x);
  p.h = static_cast<uint16_t *>(h_all);
  p.y = static_cast<uint16_t *>(y_all);
  p.ctl = static_cast<unsigned *>(ws);
  p.part = reinterpret_cast<float *>(static_cast<char *>(ws) + pl.ws_ctl);
  p.err = ds->err;
  p.eps = eps;
  void *args[] = {&maps, &p};
  const int G = ds->sms - ds->sms % PS_KSPLIT;
  cudaError_t e = launch_kernel(fn, dim3(G), dim3(PS_THREADS), pl.smem, s, false, args, 1,
                                /*cooperative=*/true);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "persistent decode-step launch");
  }
  return DFK_OK;
}

// ---------------------------------------------------------------- FP8 tensor-core plan

struct Tf8Plan {
  const void *fn = nullptr;
  int grid = 0;
  size_t smem = 0;
  Tf8Params p{};
};

// Row blocks of at most 128 rows (one per SM, or per SM / kslices for the
// split-K GEMV), one 128-wide k tile per ring stage.  FP8 weights use the
// tensor-core variants with one k tile per stage that own no full M tiles.
static bool plan_tf8(int nmat, bool norm, const VDef &v, int B, int K, int N,
                     const DeviceState &ds, Tf8Plan *pl, std::string *why) {
  if (v.nt != 1 || v.full != 0 || v.e4m3mma) {
    if (why) *why = "FP8 tensor-core kernel: one k tile per stage, rows spread over the SMs";
    return false;
  }
  if (B < 1 || B > 64) {
    if (why) *why = "batch outside 1..64";
    return false;
  }
  const int bn = B <= 16 ? 16 : (B <= 32 ? 32 : 64);
  const int ks = nmat == 1 ? v.ksplit : 1;
  const int ntiles = ceil_div(K, TF8_TILE_K);
  if (ks > ntiles) {
    if (why) *why = "more k slices than k tiles";
    return false;
  }
  const int nblocks = std::max(1, std::min(N, ds.sms / ks));
  const int rbase = N / nblocks, rextra = N % nblocks;
  const int hmax = rbase + (rextra ? 1 : 0);
  if (hmax > 128) {
    if (why) *why = "more than 128 output rows per CTA";
    return false;
  }
  const int r8 = round_up(hmax, 8);
  const int a8 = nmat * r8 * 128;
  const int xt = bn * 128 * (norm ? 2 : 1);
  const int stage = a8 + 2 * xt;  // both multiples of 1024
  const int g_bytes = norm ? round_up(ntiles * TF8_TILE_K * 2, 1024) : 0;
  const int bar_bytes = 512;      // 2 S + 5 barriers, flags, r_b of 64 tokens
  const int smem_cap = std::min(ds.smem_optin, 232448);
  const int avail = smem_cap - 1024 - g_bytes - bar_bytes;
  const int S = std::min(8, avail / stage);
  if (S < 2) {
    if (why) *why = "shared memory too small for two ring stages";
    return false;
  }
  const int wn = norm ? 2 * bn : bn;
  const int acol = round_up(nmat * wn, 64);
  const int cols = acol + 2 * nmat * 64;
  const int tmem_cols = std::max(32, pow2_ceil(cols));
  if (tmem_cols > 512) {
    if (why) *why = "accumulators and A buffers exceed TMEM";
    return false;
  }
  const void *fn = tf8_find_kernel(nmat, norm);
  if (!fn) {
    if (why) *why = "FP8 tensor-core kernel not compiled for this op";
    return false;
  }
  Tf8Params &p = pl->p;
  p = Tf8Params{};
  p.B = B;
  p.K = K;
  p.N = N;
  p.rbase = rbase;
  p.rextra = rextra;
  p.hmax = hmax;
  p.r8 = r8;
  p.bn = bn;
  p.stages = S;
  p.stage_bytes = stage;
  p.a8_bytes = a8;
  p.xt_bytes = xt;
  p.tmem_cols = tmem_cols;
  p.acol = acol;
  p.g_off = S * stage;
  p.bar_off = p.g_off + g_bytes;
  p.ntiles = ntiles;
  p.kslices = ks;
  p.nblocks = nblocks;
  pl->fn = fn;
  pl->grid = nblocks * ks;
  pl->smem = 1024 + static_cast<size_t>(p.bar_off) + bar_bytes;
  return true;
}

static int launch_tf8(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used) {
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  Tf8Plan pl;
  std::string why;
  if (!plan_tf8(c.nmat, c.norm, v, c.B, c.K, c.N, *ds, &pl, &why))
    return fail(DFK_ERR_NO_VARIANT, "variant %d does not fit FP8 B=%d K=%d N=%d: %s", v.id, c.B,
                c.K, c.N, why.c_str());
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  Tf8Maps maps;
  memset(&maps, 0, sizeof maps);
  const void *w[2] = {c.w0, c.w1};
  for (int m = 0; m < c.nmat; ++m)
    for (int lo = 0; lo < 2; ++lo) {
      const uint32_t hgt = static_cast<uint32_t>(std::max(1, pl.p.hmax - lo));
      if ((rc = tensor_map_2d(w[m], c.K, c.N, static_cast<uint64_t>(c.K), TF8_TILE_K, hgt,
                              &maps.w[m][lo], true, CU_TENSOR_MAP_DATA_TYPE_UINT8)))
        return rc;
    }
  if ((rc = tensor_map_2d(c.x, c.K, c.B, static_cast<uint64_t>(c.K) * 2, 64, pl.p.bn, &maps.x,
                          true)))
    return rc;
  Tf8Params p = pl.p;
  p.out = static_cast<uint16_t *>(c.out);
  p.gamma = static_cast<const uint16_t *>(c.gamma);
  p.scale[0] = c.s0;
  p.scale[1] = c.s1;
  p.err = ds->err;
  p.eps = c.eps;
  if (p.kslices > 1) {
    const size_t part_bytes =
        static_cast<size_t>(p.kslices) * p.nblocks * p.bn * 128 * sizeof(float);
    const size_t counter_bytes = static_cast<size_t>(ds->sms) * 8 * sizeof(unsigned);
    if ((rc = get_workspace(dev, s, part_bytes, counter_bytes, &p.part, &p.counters))) {
      if (rc != DFK_ERR_NO_VARIANT || !stream_capturing(s)) return rc;
      VDef whole = v;
      whole.ksplit = 1;
      log_msg("split-K workspace missing during capture: launching without the split");
      return launch_tf8(c, whole, s, stages_used);
    }
  }
  void *args[] = {&maps, &p};
  cudaError_t e = launch_kernel(pl.fn, dim3(pl.grid), dim3(TF8_THREADS), pl.smem, s,
                                pdl_enabled(), args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "FP8 tensor-core kernel launch");
  }
  if (stages_used) *stages_used = p.stages;
  return DFK_OK;
}

// ---------------------------------------------------------------- FP8 E4M3-MMA plan

struct Tm8Plan {
  const void *fn = nullptr;
  int grid = 0, threads = TM8_THREADS;
  size_t smem = 0;
  Tm8Params p{};
  size_t term_bytes = 0;  // activation-term buffer: codes + per-token factors
};

// Terms per token: 2 carry a bf16 activation exactly, 4 the 16-bit x * gamma
// products of the RMSNorm path.  Rows of <= 128 per CTA as for the other
// tensor-core kernels; one 128-wide k tile per stage.
static bool plan_tm8(int nmat, bool norm, const VDef &v, int B, int K, int N,
                     const DeviceState &ds, Tm8Plan *pl, std::string *why) {
  if (!v.e4m3mma) {
    if (why) *why = "not an E4M3-MMA variant";
    return false;
  }
  if (B < 1 || B > 64) {
    if (why) *why = "batch outside 1..64";
    return false;
  }
  const bool ink = v.e4m3mma == 2;  // activation terms derived in the kernel
  const int T = norm ? 4 : 2;
  // in-kernel terms: the fewest token slots holding B with 16 or 32 MMA columns
  const int ibp = !ink ? 0 : (T == 4 ? (B <= 4 ? 4 : (B <= 8 ? 8 : 0))
                                     : (B <= 8 ? 8 : (B <= 16 ? 16 : 0)));
  if (ink && !ibp) {
    if (why) *why = "in-kernel activation terms: up to 8 tokens with RMSNorm, 16 without";
    return false;
  }
  const int bnp = ink ? ibp : (B <= 16 ? 16 : (B <= 32 ? 32 : 64));
  const int np = T * bnp;
  if (np > 256 || nmat * np > 512) {
    if (why) *why = "activation terms exceed N = 256";
    return false;
  }
  const int ks = nmat == 1 ? v.ksplit : 1;
  const int ntiles = ceil_div(K, TM8_TILE_K);
  if (norm && ks > 1) {  // r_b needs all of K in one prep CTA per token
    if (why) *why = "RMSNorm with a k split";
    return false;
  }
  if (ks > ntiles) {
    if (why) *why = "more k slices than k tiles";
    return false;
  }
  const int nblocks = std::max(1, std::min(N, ds.sms / ks));
  const int rbase = N / nblocks, rextra = N % nblocks;
  const int hmax = rbase + (rextra ? 1 : 0);
  if (hmax > 128) {
    if (why) *why = "more than 128 output rows per CTA";
    return false;
  }
  if (v.nt < 1 || v.nt > 2) {
    if (why) *why = "one or two k tiles per stage";
    return false;
  }
  const int r8 = round_up(hmax, 8);
  const int a8 = nmat * r8 * 128;
  // stage: code tiles (+ the term tiles with prep terms); in-kernel terms
  // keep the whole k range's terms resident after the ring
  const int stage = v.nt * (a8 + (ink ? 0 : np * 128));  // multiples of 1024
  const int tarea = ink ? ceil_div(ntiles, ks) * np * 128 : 0;
  // the last code tile's 128-row MMA read may run past the last stage
  const int over = (v.nt * nmat - 1) * r8 * 128 + 128 * 128;
  const int slack = std::max(0, over - stage - tarea);
  const int bar_bytes = 512;  // 2 S + 2 barriers, flags, per-token factors and scales
  const int smem_cap = std::min(ds.smem_optin, ink ? 232448 : SMEM_BESIDE_PREP);
  const int S = std::min(8, (smem_cap - 1024 - bar_bytes - slack - tarea) / stage);
  if (S < 2) {
    if (why) *why = "shared memory too small for two ring stages";
    return false;
  }
  const void *fn = tf8mma_find_kernel(nmat, ibp, ink ? T : 0);
  if (!fn) {
    if (why) *why = "E4M3-MMA kernel not compiled for this op";
    return false;
  }
  Tm8Params &p = pl->p;
  p = Tm8Params{};
  p.B = B;
  p.K = K;
  p.N = N;
  p.rbase = rbase;
  p.rextra = rextra;
  p.hmax = hmax;
  p.r8 = r8;
  p.bnp = bnp;
  p.T = T;
  p.np = np;
  p.nt = v.nt;
  p.stages = S;
  p.stage_bytes = stage;
  p.a8_bytes = a8;
  p.tmem_cols = std::max(32, pow2_ceil(nmat * np));
  p.bar_off = S * stage + tarea + slack;
  p.ntiles = ntiles;
  p.kslices = ks;
  p.nblocks = nblocks;
  p.term_off = ink ? S * stage : v.nt * a8;
  pl->fn = fn;
  pl->grid = nblocks * ks;
  pl->threads = ink ? TM8_INK_THREADS : TM8_THREADS;
  pl->smem = 1024 + static_cast<size_t>(p.bar_off) + bar_bytes;
  // codes, then the factors [kslices][bnp] (at most 8 x 64)
  pl->term_bytes = ink ? 0 : static_cast<size_t>(ntiles) * np * 128 + 8 * 64 * sizeof(float);
  return true;
}

// Activation-term buffer: one per (device, stream), grown on demand outside
// stream capture.
static std::map<std::pair<int, cudaStream_t>, Workspace> g_terms;

static int get_term_buffer(int dev, cudaStream_t s, size_t bytes, void **out) {
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace &w = g_terms[std::make_pair(dev, s)];
  if (w.bytes < bytes) {
    if (stream_capturing(s))
      return fail(DFK_ERR_NO_VARIANT, "FP8 activation-term buffer must be allocated before "
                  "capture (make one call of this shape on the stream first)");
    if (w.base) {
      cudaStreamSynchronize(s);
      cudaFree(w.base);
      w.base = nullptr;
      w.bytes = 0;
    }
    const size_t grow = std::max(bytes, static_cast<size_t>(4) << 20);
    cudaError_t e = cudaMalloc(&w.base, grow);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "cudaMalloc (FP8 activation-term buffer)");
    }
    w.bytes = grow;
  }
  *out = w.base;
  return DFK_OK;
}

static int launch_tf8(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used);

static int launch_tm8(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used) {
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  Tm8Plan pl;
  std::string why;
  if (!plan_tm8(c.nmat, c.norm, v, c.B, c.K, c.N, *ds, &pl, &why))
    return fail(DFK_ERR_NO_VARIANT, "variant %d does not fit FP8 B=%d K=%d N=%d: %s", v.id, c.B,
                c.K, c.N, why.c_str());
  const bool ink = v.e4m3mma == 2;  // no prep kernel, no term buffer
  void *terms = nullptr;
  if (!ink && (rc = get_term_buffer(dev, s, pl.term_bytes, &terms))) {
    if (rc != DFK_ERR_NO_VARIANT || !stream_capturing(s)) return rc;
    // captured on a stream without the buffer: the widening tensor-core kernel
    VDef alt = v;
    alt.e4m3mma = 0;
    log_msg("FP8 term buffer missing during capture: launching the widening kernel");
    return launch_tf8(c, alt, s, stages_used);
  }
  if ((rc = ensure_smem_attr(dev, pl.fn))) return rc;
  Tm8Params p = pl.p;
  const size_t code_bytes = static_cast<size_t>(p.ntiles) * p.np * 128;
  float *fac = ink ? nullptr : reinterpret_cast<float *>(static_cast<char *>(terms) + code_bytes);
  Tm8Maps maps;
  memset(&maps, 0, sizeof maps);
  const void *w[2] = {c.w0, c.w1};
  for (int m = 0; m < c.nmat; ++m)
    for (int lo = 0; lo < 2; ++lo) {
      const uint32_t hgt = static_cast<uint32_t>(std::max(1, p.hmax - lo));
      if ((rc = tensor_map_2d(w[m], c.K, c.N, static_cast<uint64_t>(c.K), TM8_TILE_K, hgt,
                              &maps.w[m][lo], true, CU_TENSOR_MAP_DATA_TYPE_UINT8)))
        return rc;
    }
  if (!ink && (rc = tensor_map_2d(terms, TM8_TILE_K, static_cast<uint64_t>(p.ntiles) * p.np,
                                  TM8_TILE_K, TM8_TILE_K, static_cast<uint32_t>(p.np), &maps.x,
                                  true, CU_TENSOR_MAP_DATA_TYPE_UINT8)))
    return rc;
  p.x = static_cast<const uint16_t *>(c.x);
  p.gamma = c.norm ? static_cast<const uint16_t *>(c.gamma) : nullptr;
  p.eps = c.eps;
  p.out = static_cast<uint16_t *>(c.out);
  p.scale[0] = c.s0;
  p.scale[1] = c.s1;
  p.fac = fac;
  p.err = ds->err;
  if (p.kslices > 1) {
    const size_t part_bytes =
        static_cast<size_t>(p.kslices) * p.nblocks * p.bnp * 128 * sizeof(float);
    const size_t counter_bytes = static_cast<size_t>(ds->sms) * 8 * sizeof(unsigned);
    if ((rc = get_workspace(dev, s, part_bytes, counter_bytes, &p.part, &p.counters))) {
      if (rc != DFK_ERR_NO_VARIANT || !stream_capturing(s)) return rc;
      VDef whole = v;
      whole.ksplit = 1;
      log_msg("split-K workspace missing during capture: launching without the split");
      return launch_tm8(c, whole, s, stages_used);
    }
  }
  cudaError_t e = cudaSuccess;
  if (!ink) {
    // prep: scales, r_b and the E4M3 terms of the activations
    Tm8PrepParams pp{};
    pp.x = static_cast<const uint16_t *>(c.x);
    pp.gamma = c.norm ? static_cast<const uint16_t *>(c.gamma) : nullptr;
    pp.terms = static_cast<uint8_t *>(terms);
    pp.fac = fac;
    pp.B = c.B;
    pp.K = c.K;
    pp.bnp = p.bnp;
    pp.T = p.T;
    pp.ntiles = p.ntiles;
    pp.kslices = p.kslices;
    pp.eps = c.eps;
    pp.err = ds->err;
    void *pargs[] = {&pp};
    // one CTA per token slot and reduction slice
    e = launch_kernel(tf8mma_prep_fn(), dim3(p.bnp, p.kslices), dim3(TM8_PREP_THREADS), 0, s,
                      pdl_enabled(), pargs);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "FP8 activation-term kernel launch");
    }
  }
  void *args[] = {&maps, &p};
  e = launch_kernel(pl.fn, dim3(pl.grid), dim3(pl.threads), pl.smem, s, pdl_enabled(), args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "FP8 E4M3-MMA kernel launch");
  }
  if (stages_used) *stages_used = p.stages;
  return DFK_OK;
}

static int launch_variant(const CcCall &c, const VDef &v, cudaStream_t s, int *stages_used) {
  if (v.family == DFK_FAMILY_TENSOR_CORE) {
    if (!c.w8) return launch_tc(c, v, s, stages_used);
    return v.e4m3mma ? launch_tm8(c, v, s, stages_used) : launch_tf8(c, v, s, stages_used);
  }
  return launch_cc(c, v, s, stages_used);
}

// ---------------------------------------------------------------- scheduler

struct TuneKey {
  int dev, op, B, D, F, layout;
  bool operator<(const TuneKey &o) const {
    return std::tie(dev, op, B, D, F, layout) < std::tie(o.dev, o.op, o.B, o.D, o.F, o.layout);
  }
};

static std::mutex g_tune_mu;
static std::map<TuneKey, dfk_variant> g_tuned;

static bool op_is_down(int op) { return op == DFK_OP_DOWN || op == DFK_OP_DOWN_FP8; }
static bool op_is_qkv(int op) { return op == DFK_OP_QKV || op == DFK_OP_RMSNORM_QKV; }
static bool op_is_fp8(int op) {
  return op == DFK_OP_GATE_UP_FP8 || op == DFK_OP_RMSNORM_GATE_UP_FP8 || op == DFK_OP_DOWN_FP8;
}
static bool op_is_norm(int op) {
  return op == DFK_OP_RMSNORM_GATE_UP || op == DFK_OP_RMSNORM_GATE_UP_FP8 ||
         op == DFK_OP_RMSNORM_QKV;
}
static int op_class(int op) { return (op_is_down(op) || op_is_qkv(op)) ? CLS_GEMV : CLS_GATE_UP; }

static void fill_variant(const VDef &d, int op, int layout, int stages, float us,
                         dfk_variant *out) {
  out->variant_id = d.id;
  out->op = op;
  out->layout = layout;
  out->family = d.family;
  out->j_per_thread = d.jpt;
  out->token_tile = d.bt;
  out->k_split = d.ksplit;
  out->k_tiles_per_stage = d.nt;
  out->acc_banks = d.nbank;
  out->paired_fma = d.pair;
  out->full_m_tiles = d.full;
  out->e4m3_mma = d.e4m3mma;
  out->stages = stages;
  out->measured_us = us;
}

// ---- persistent decisions: $DFK_TUNE_CACHE, one text line per decision
//   dfk-tune 1 <device name> <SMs> <driver> <op> <B> <d_model> <d_ff> <layout> <variant> <us>
// (spaces in the device name replaced by '_').  Lines for another device or
// driver, malformed lines and unknown variant ids are skipped with a warning.

static std::map<int, bool> g_cache_loaded;  // per device

static std::string device_tag(int dev, int sms) {
  cudaDeviceProp prop;
  std::string name = "unknown";
  if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) name = prop.name;
  else cudaGetLastError();
  for (char &ch : name)
    if (ch == ' ') ch = '_';
  int drv = 0;
  cudaDriverGetVersion(&drv);
  return name + " " + std::to_string(sms) + " " + std::to_string(drv);
}

static void tune_cache_load(int dev, int sms) {  // caller holds g_tune_mu
  if (g_cache_loaded[dev]) return;
  g_cache_loaded[dev] = true;
  const char *path = getenv("DFK_TUNE_CACHE");
  if (!path || !*path) return;
  FILE *f = fopen(path, "r");
  if (!f) return;
  const std::string tag = device_tag(dev, sms);
  char line[512];
  int lineno = 0, bad = 0, used = 0;
  while (fgets(line, sizeof line, f)) {
    ++lineno;
    char magic[16], name[256];
    int ver, n_sms, drv, op, B, D, F, layout, vid;
    float us;
    if (sscanf(line, "%15s %d %255s %d %d %d %d %d %d %d %d %f", magic, &ver, name, &n_sms, &drv,
               &op, &B, &D, &F, &layout, &vid, &us) != 12 ||
        strcmp(magic, "dfk-tune") != 0 || ver != 1) {
      ++bad;
      continue;
    }
    if (std::string(name) + " " + std::to_string(n_sms) + " " + std::to_string(drv) != tag)
      continue;
    const VDef *d = find_variant(vid);
    if (!d || d->cls != op_class(op) || B < 1 || B > 64 ||
        (op_is_fp8(op) && !fp8_capable(*d)) || (!op_is_fp8(op) && !bf16_capable(*d))) {
      ++bad;
      continue;
    }
    dfk_variant rec;
    fill_variant(*d, op, layout, 0, us, &rec);
    g_tuned[TuneKey{dev, op, B, D, F, layout}] = rec;
    ++used;
  }
  fclose(f);
  if (bad)
    fprintf(stderr, "[dfk] warning: %s: skipped %d malformed line(s) of %d\n", path, bad,
            lineno);
  log_msg("tune cache %s: %d decision(s) loaded", path, used);
}

static void tune_cache_append(int dev, int sms, const TuneKey &k, const dfk_variant &v) {
  const char *path = getenv("DFK_TUNE_CACHE");
  if (!path || !*path) return;
  FILE *f = fopen(path, "a");
  if (!f) {
    log_msg("cannot append to tune cache %s", path);
    return;
  }
  fprintf(f, "dfk-tune 1 %s %d %d %d %d %d %d %.3f\n", device_tag(dev, sms).c_str(), k.op, k.B,
          k.D, k.F, k.layout, v.variant_id, v.measured_us);
  fclose(f);
}


// Candidates worth timing for (op, B): every CUDA-core j-per-thread / k-split
// / tiles-per-stage / pairing choice at its largest useful token tile, plus the
// tensor-core variants from B = 4 (gate/up) or B = 2 (GEMV); at B = 1 fp32
// FMA on CUDA cores keeps up with HBM.  FP8 weights: CUDA-core variants with
// one or two tiles per stage only.
static std::vector<const VDef *> candidates(int op, int B, const CcCall &c) {
  std::vector<const VDef *> out;
  for (const VDef &d : variants()) {
    if (d.cls != op_class(op)) continue;
    if (c.w8 && d.family == DFK_FAMILY_TENSOR_CORE) {
      // FP8: the tensor-core kernels (widening, E4M3 MMA) at every batch
      if (fp8_capable(d)) out.push_back(&d);
      continue;
    }
    if (!c.w8 && !bf16_capable(d)) continue;
    if (c.w8 && d.nt > 2) continue;
    if (d.family == DFK_FAMILY_TENSOR_CORE) {
      // gate/up from B = 4 (where CUDA cores fall below HBM speed), the GEMV
      // (split-K) from B = 2
      if (B >= (d.cls == CLS_GEMV ? 2 : 4)) out.push_back(&d);
      continue;
    }
    if (d.bt != bt_for(B, d.jpt)) continue;
    out.push_back(&d);
  }
  return out;
}

static bool feasible(const VDef &d, const CcCall &c, const DeviceState &ds) {
  if (d.family == DFK_FAMILY_TENSOR_CORE) {
    if (c.w8 && d.e4m3mma) {
      Tm8Plan pl;
      return plan_tm8(c.nmat, c.norm, d, c.B, c.K, c.N, ds, &pl, nullptr);
    }
    if (c.w8) {
      Tf8Plan pl;
      return plan_tf8(c.nmat, c.norm, d, c.B, c.K, c.N, ds, &pl, nullptr);
    }
    TcPlan pl;
    return plan_tc(c.layout, c.nmat, c.norm, d, c.B, c.K, c.N, ds, &pl, nullptr,
                   tc_prepared(c));
  }
  CcPlan pl;
  return plan_cc(c.layout, c.nmat, c.norm, c.w8, d, c.B, c.K, c.N, ds, &pl, nullptr);
}

// Heuristic default (no timing): the tensor-core family from B = 8 up (one
// k-tile per stage for gate/up, four for the GEMV); below that CUDA cores
// with 4 rows per thread (2 rows from B = 5), two k-tiles per stage, and for
// the GEMV the largest k split whose CTA fits.  If nothing of that shape
// fits, the feasible CUDA-core variant with the fewest passes wins.
static const VDef *heuristic(int op, int B, const CcCall &c, const DeviceState &ds) {
  if (c.w8 && B >= 2) {
    // FP8 weights: the E4M3-MMA kernel (with in-kernel activation terms up
    // to 16 tokens), else the widening one (split-K 4 for the GEMV)
    const int want_ks = op_class(op) == CLS_GEMV ? 4 : 1;
    for (int mma : {2, 1, 0})
      for (const VDef &d : variants())
        if (d.cls == op_class(op) && d.family == DFK_FAMILY_TENSOR_CORE && d.nt == 1 &&
            d.full == 0 && d.e4m3mma == mma && d.ksplit == want_ks && feasible(d, c, ds))
          return &d;
  }
  if (B >= 8 && !c.w8) {
    const bool gemv = op_class(op) == CLS_GEMV;
    const int want_nt = gemv ? 2 : 1, want_ks = gemv ? 4 : 1;
    for (const VDef &d : variants())
      if (d.cls == op_class(op) && d.family == DFK_FAMILY_TENSOR_CORE && bf16_capable(d) &&
          d.nt == want_nt &&
          d.ksplit == want_ks && d.nbank == 1 && feasible(d, c, ds))
        return &d;
  }
  const int jpt = B <= 4 ? 4 : 2;
  const VDef *best = nullptr;
  for (const VDef &d : variants()) {
    if (d.cls != op_class(op) || d.family != DFK_FAMILY_CUDA_CORE) continue;
    if (d.jpt != jpt || d.bt != bt_for(B, jpt) || d.nt != 2) continue;
    if (!feasible(d, c, ds)) continue;
    if (!best || d.ksplit > best->ksplit) best = &d;
  }
  if (best) return best;
  int best_pass = 1 << 30;
  for (const VDef &d : variants()) {
    if (d.cls != op_class(op) || d.family != DFK_FAMILY_CUDA_CORE) continue;
    if (!feasible(d, c, ds)) continue;
    const int passes = ceil_div(B, d.bt);
    if (passes < best_pass || (passes == best_pass && d.ksplit > best->ksplit)) {
      best = &d;
      best_pass = passes;
    }
  }
  return best;
}

static bool stream_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return true;  // be conservative: do not time
  }
  return cs != cudaStreamCaptureStatusNone;
}

// Time `cands` for call `c` on stream s; returns the winner (or nullptr).
static const VDef *time_candidates(int op, const CcCall &c, const std::vector<const VDef *> &cands,
                                   cudaStream_t s, const DeviceState &ds, float *best_us,
                                   int *best_stages) {
  const char *fault = getenv("DFK_FAULT");
  if (fault && strcmp(fault, "tune") == 0) {
    log_msg("tuning disabled by DFK_FAULT=tune; using the heuristic");
    return nullptr;
  }
  const int reps = std::max(1, env_int("DFK_TUNE_REPS", 7));
  size_t flush_bytes = static_cast<size_t>(std::max(ds.l2_bytes, 1 << 20)) * 2;
  void *flush = nullptr;
  cudaError_t e = cudaMallocAsync(&flush, flush_bytes, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    flush = nullptr;
  }
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  // When one call's weights fit in L2, a burst's later launches would read
  // them from L2: the burst then rotates over copies of the weights that
  // together exceed L2 (made here, freed below); without memory for them
  // each sample is one launch after its own flush.
  const size_t wbytes = static_cast<size_t>(c.K) * c.N * c.nmat * (c.w8 ? 1 : 2);
  const size_t l2 = static_cast<size_t>(std::max(ds.l2_bytes, 1 << 20));
  std::vector<CcCall> rot;
  void *wcopies = nullptr;
  if (flush && wbytes < l2) {
    const int ncopy = static_cast<int>(std::min<size_t>(8, l2 / wbytes + 2));
    const size_t b0 = c.w1 ? wbytes / c.nmat : wbytes;  // bytes at w0 (w1 holds the rest)
    const size_t stride = (wbytes + 1023) & ~static_cast<size_t>(1023);
    if (cudaMallocAsync(&wcopies, stride * ncopy, s) == cudaSuccess) {
      for (int i = 0; i < ncopy; ++i) {
        char *base = static_cast<char *>(wcopies) + stride * i;
        CcCall ci = c;
        cudaMemcpyAsync(base, c.w0, b0, cudaMemcpyDeviceToDevice, s);
        ci.w0 = base;
        if (c.w1) {
          cudaMemcpyAsync(base + b0, c.w1, wbytes - b0, cudaMemcpyDeviceToDevice, s);
          ci.w1 = base + b0;
        }
        rot.push_back(ci);
      }
    } else {
      cudaGetLastError();
      wcopies = nullptr;
    }
  }
  const VDef *best = nullptr;
  float best_t = 1e30f;
  for (const VDef *d : cands) {
    int st = 0;
    if (launch_variant(c, *d, s, &st) != DFK_OK) continue;  // warm-up; skips infeasible ones
    // Each repetition: flush L2, then a burst of back-to-back launches (the
    // way a decode loop issues them, neighbours overlapping through
    // programmatic dependent launch); the sample is the burst's mean.
    const int burst = (flush && wbytes < l2 && rot.empty()) ? 1 : 4;
    std::vector<float> ts;
    bool ok = true;
    for (int r = 0; r < reps && ok; ++r) {
      if (flush) cudaMemsetAsync(flush, r & 0xff, flush_bytes, s);
      cudaEventRecord(e0, s);
      for (int b = 0; b < burst && ok; ++b)
        ok = launch_variant(rot.empty() ? c : rot[b % rot.size()], *d, s, nullptr) == DFK_OK;
      cudaEventRecord(e1, s);
      if (cudaEventSynchronize(e1) != cudaSuccess) ok = false;
      float ms = 0.f;
      cudaEventElapsedTime(&ms, e0, e1);
      ts.push_back(ms * 1000.f / burst);
    }
    if (!ok || ts.empty()) continue;
    std::sort(ts.begin(), ts.end());
    const float med = ts[ts.size() / 2];
    log_msg("op %d B=%d K=%d N=%d layout %d: variant %d (jpt %d bt %d ks %d nt %d, %d stages) "
            "%.2f us", op, c.B, c.K, c.N, c.layout, d->id, d->jpt, d->bt, d->ksplit, d->nt, st,
            med);
    if (med < best_t) {
      best_t = med;
      best = d;
      *best_stages = st;
    }
  }
  if (flush) cudaFreeAsync(flush, s);
  if (wcopies) cudaFreeAsync(wcopies, s);
  cudaStreamSynchronize(s);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaGetLastError();
  *best_us = best_t;
  return best;
}

// Pick the variant for call `c` (variant 0 = scheduler's choice).
static int resolve(int op, int variant, const CcCall &c, cudaStream_t s, const VDef **out) {
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  if (variant > 0) {
    const VDef *d = find_variant(variant);
    if (!d || d->cls != op_class(op))
      return fail(DFK_ERR_INVALID_ARG, "variant %d is not a variant of op %d", variant, op);
    if (c.w8 && !fp8_capable(*d))
      return fail(DFK_ERR_INVALID_ARG, "variant %d cannot run FP8 weights", variant);
    if (!c.w8 && !bf16_capable(*d))
      return fail(DFK_ERR_INVALID_ARG, "variant %d runs FP8 weights only", variant);
    *out = d;
    return DFK_OK;
  }
  TuneKey key{dev, op, c.B, op_is_down(op) ? c.N : c.K, op_is_down(op) ? c.K : c.N, c.layout};
  {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    tune_cache_load(dev, ds->sms);
    auto it = g_tuned.find(key);
    if (it != g_tuned.end()) {
      *out = find_variant(it->second.variant_id);
      return DFK_OK;
    }
  }
  // Layouts of one gate/up shape agree bit for bit within a variant family
  // (the same k order reaches the same accumulators), not across families.
  // Once one layout of this shape has a decision, the other layouts are
  // chosen within its family, so the row- and column-major results a caller
  // gets from the scheduler are identical.
  int lock_family = -1;
  if (op_class(op) == CLS_GATE_UP) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    for (int l : {LAYOUT_ROW, LAYOUT_COL, LAYOUT_IL}) {
      TuneKey k2 = key;
      k2.layout = l;
      auto it = g_tuned.find(k2);
      if (l != c.layout && it != g_tuned.end()) {
        lock_family = it->second.family;
        break;
      }
    }
  }
  std::vector<const VDef *> cands = candidates(op, c.B, c);
  const VDef *h = heuristic(op, c.B, c, *ds);
  if (lock_family >= 0) {
    cands.erase(std::remove_if(cands.begin(), cands.end(),
                               [&](const VDef *d) { return d->family != lock_family; }),
                cands.end());
    if (h && h->family != lock_family) {
      h = nullptr;
      for (const VDef *d : cands)
        if (feasible(*d, c, *ds)) {
          h = d;
          break;
        }
    }
  }
  if (!h) return fail(DFK_ERR_NO_VARIANT, "no variant fits B=%d K=%d N=%d", c.B, c.K, c.N);
  const bool tune = env_flag("DFK_TUNE", true) && !stream_capturing(s);
  const VDef *win = h;
  float us = -1.f;
  int stages = 0;
  if (tune) {
    const VDef *t = time_candidates(op, c, cands, s, *ds, &us, &stages);
    if (t) win = t;
    else us = -1.f;
  }
  if (tune || !env_flag("DFK_TUNE", true)) {
    dfk_variant rec;
    fill_variant(*win, op, c.layout, stages, us, &rec);
    std::lock_guard<std::mutex> lk(g_tune_mu);
    g_tuned[key] = rec;
    if (us >= 0) tune_cache_append(dev, ds->sms, key, rec);
  }
  log_msg("op %d B=%d D=%d F=%d layout %d -> variant %d (%s)", op, c.B, key.D, key.F, c.layout,
          win->id, us >= 0 ? "timed" : "heuristic");
  *out = win;
  return DFK_OK;
}

// ---------------------------------------------------------------- validation


static int check_gate_up(const void *x, const void *gamma, bool norm, float eps, const void *wg,
                         const void *wu, int layout, const void *h, int B, int D, int F,
                         int variant) {
  if (layout != DFK_W_ROW_MAJOR && layout != DFK_W_COL_MAJOR && layout != DFK_W_GU_INTERLEAVED)
    return fail(DFK_ERR_UNSUPPORTED_LAYOUT, "layout %d is not a weight layout", layout);
  if (B < 0 || D <= 0 || F <= 0) return fail(DFK_ERR_INVALID_ARG, "negative or zero size");
  if (variant < 0) return fail(DFK_ERR_INVALID_ARG, "variant id %d < 0", variant);
  if (variant > 0) {
    const VDef *d = find_variant(variant);
    if (!d || d->cls != CLS_GATE_UP || !bf16_capable(*d))
      return fail(DFK_ERR_INVALID_ARG, "variant %d is not a bf16 gate/up variant", variant);
  }
  if (norm && !(eps >= 0.f && std::isfinite(eps)))
    return fail(DFK_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (B > 64) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "B=%d > 64 (decode batches only)", B);
  if (D % 8) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "d_model %% 8 != 0 (d_model=%d)", D);
  if (layout == DFK_W_COL_MAJOR && F % 8)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "column-major needs d_ff %% 8 == 0 (d_ff=%d)", F);
  if (static_cast<long long>(F) * 2 > (1ll << 31))
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "d_ff too large");
  if (layout == DFK_W_GU_INTERLEAVED && wu)
    return fail(DFK_ERR_INVALID_ARG, "interleaved layout: w_up must be NULL");
  if (B == 0) return DFK_OK;
  if (!x || !wg || !h || (norm && !gamma) || (layout != DFK_W_GU_INTERLEAVED && !wu))
    return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if (misaligned(x) || misaligned(wg) || misaligned(h) || (wu && misaligned(wu)) ||
      (norm && misaligned(gamma)))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  return DFK_OK;
}

static int check_gemv(const void *x, const void *w, const void *out, int B, int K, int N,
                      int variant) {
  if (B < 0 || K <= 0 || N <= 0) return fail(DFK_ERR_INVALID_ARG, "negative or zero size");
  if (variant < 0) return fail(DFK_ERR_INVALID_ARG, "variant id %d < 0", variant);
  if (variant > 0) {
    const VDef *d = find_variant(variant);
    if (!d || d->cls != CLS_GEMV || !bf16_capable(*d))
      return fail(DFK_ERR_INVALID_ARG, "variant %d is not a bf16 GEMV variant", variant);
  }
  if (B > 64) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "B=%d > 64 (decode batches only)", B);
  if (K % 8) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "reduction length %% 8 != 0 (K=%d)", K);
  if (B == 0) return DFK_OK;
  if (!x || !w || !out) return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if (misaligned(x) || misaligned(w) || misaligned(out))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  return DFK_OK;
}

static int to_engine_layout(int layout) {
  return layout == DFK_W_COL_MAJOR ? LAYOUT_COL
                                   : (layout == DFK_W_GU_INTERLEAVED ? LAYOUT_IL : LAYOUT_ROW);
}

static int gate_up_impl(int op, const void *x, const void *gamma, float eps, const void *wg,
                        const void *wu, int layout, void *h, int B, int D, int F, int variant,
                        cudaStream_t s) {
  const bool norm = op == DFK_OP_RMSNORM_GATE_UP;
  int rc = check_gate_up(x, gamma, norm, eps, wg, wu, layout, h, B, D, F, variant);
  if (rc || B == 0) return rc;
  CcCall c{to_engine_layout(layout), 2, norm, x, gamma, eps, wg, wu, h, B, D, F};
  const VDef *v = nullptr;
  if ((rc = resolve(op, variant, c, s, &v))) return rc;
  return launch_variant(c, *v, s, nullptr);
}

static int gemv_impl(int op, const void *x, const void *w, void *out, int B, int K, int N,
                     int variant, cudaStream_t s) {
  int rc = check_gemv(x, w, out, B, K, N, variant);
  if (rc || B == 0) return rc;
  CcCall c{LAYOUT_ROW, 1, false, x, nullptr, 0.f, w, nullptr, out, B, K, N};
  const VDef *v = nullptr;
  if ((rc = resolve(op, variant, c, s, &v))) return rc;
  return launch_variant(c, *v, s, nullptr);
}

// FP8 weights: row-major E4M3 codes (1 byte each) and fp32 row scales.
static int check_fp8(const void *x, const void *gamma, bool norm, float eps, const void *q0,
                     const float *s0, const void *q1, const float *s1, const void *out, int B,
                     int K, int N, int variant, int cls) {
  if (B < 0 || K <= 0 || N <= 0) return fail(DFK_ERR_INVALID_ARG, "negative or zero size");
  if (variant < 0) return fail(DFK_ERR_INVALID_ARG, "variant id %d < 0", variant);
  if (variant > 0) {
    const VDef *d = find_variant(variant);
    if (!d || d->cls != cls || !fp8_capable(*d))
      return fail(DFK_ERR_INVALID_ARG, "variant %d cannot run this FP8 op", variant);
  }
  if (norm && !(eps >= 0.f && std::isfinite(eps)))
    return fail(DFK_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (B > 64) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "B=%d > 64 (decode batches only)", B);
  if (K % 16)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "FP8 weights: reduction length %% 16 != 0 (%d)", K);
  if (B == 0) return DFK_OK;
  const bool two = cls == CLS_GATE_UP;
  if (!x || !q0 || !s0 || !out || (norm && !gamma) || (two && (!q1 || !s1)))
    return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if (misaligned(x) || misaligned(q0) || misaligned(out) || (two && misaligned(q1)) ||
      (norm && misaligned(gamma)))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(s0) | reinterpret_cast<uintptr_t>(s1)) & 3u)
    return fail(DFK_ERR_MISALIGNED, "scale pointers must be 4-byte aligned");
  return DFK_OK;
}

static int fp8_impl(int op, const void *x, const void *gamma, float eps, const void *q0,
                    const float *s0, const void *q1, const float *s1, void *out, int B, int K,
                    int N, int variant, cudaStream_t s) {
  const bool down = op_is_down(op), norm = op_is_norm(op);
  int rc = check_fp8(x, gamma, norm, eps, q0, s0, q1, s1, out, B, K, N, variant,
                     down ? CLS_GEMV : CLS_GATE_UP);
  if (rc || B == 0) return rc;
  CcCall c{LAYOUT_ROW, down ? 1 : 2, norm, x, gamma, eps, q0, down ? nullptr : q1, out, B, K, N};
  c.w8 = true;
  c.s0 = s0;
  c.s1 = down ? nullptr : s1;
  const VDef *v = nullptr;
  if ((rc = resolve(op, variant, c, s, &v))) return rc;
  return launch_variant(c, *v, s, nullptr);
}

// RMSNorm (optional) + packed QKV projection: one GEMV over W_qkv
// [n_q + n_k + n_v][d_model], the output rows routed to q, k and v.
static int qkv_impl(const void *x, const void *gamma, float eps, const void *w, void *q, void *k,
                    void *v, int B, int D, int nq, int nk, int nv, int variant,
                    cudaStream_t s) {
  const bool norm = gamma != nullptr;
  if (nq < 0 || nk < 0 || nv < 0 || static_cast<long long>(nq) + nk + nv <= 0 ||
      static_cast<long long>(nq) + nk + nv > (1 << 30))
    return fail(DFK_ERR_INVALID_ARG, "bad part sizes n_q=%d n_k=%d n_v=%d", nq, nk, nv);
  if (norm && !(eps >= 0.f && std::isfinite(eps)))
    return fail(DFK_ERR_INVALID_ARG, "eps must be finite and >= 0");
  const int N = nq + nk + nv;
  int rc = check_gemv(x, w, B > 0 ? (q ? q : (k ? k : v)) : nullptr, B, D, N, variant);
  if (rc || B == 0) return rc;
  if ((nq && !q) || (nk && !k) || (nv && !v))
    return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if ((q && misaligned(q)) || (k && misaligned(k)) || (v && misaligned(v)) ||
      (norm && misaligned(gamma)))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  CcCall c{LAYOUT_ROW, 1, norm, x, gamma, eps, w, nullptr, q, B, D, N};
  c.outs[0] = q;
  c.outs[1] = k;
  c.outs[2] = v;
  c.split[0] = nq;
  c.split[1] = nq + nk;
  const VDef *vd = nullptr;
  const int op = norm ? DFK_OP_RMSNORM_QKV : DFK_OP_QKV;
  if ((rc = resolve(op, variant, c, s, &vd))) return rc;
  return launch_variant(c, *vd, s, nullptr);
}

}  // namespace dfk

using namespace dfk;

// ================================================================ C ABI

extern "C" {

int dfk_swiglu_gate_up(const void *x, const void *w_gate, const void *w_up, int layout, void *h,
                       int B, int d_model, int d_ff, int variant, void *stream) {
  return gate_up_impl(DFK_OP_GATE_UP, x, nullptr, 0.f, w_gate, w_up, layout, h, B, d_model,
                      d_ff, variant, static_cast<cudaStream_t>(stream));
}

int dfk_rmsnorm_swiglu_gate_up(const void *x, const void *gamma, float eps, const void *w_gate,
                               const void *w_up, int layout, void *h, int B, int d_model,
                               int d_ff, int variant, void *stream) {
  return gate_up_impl(DFK_OP_RMSNORM_GATE_UP, x, gamma, eps, w_gate, w_up, layout, h, B,
                      d_model, d_ff, variant, static_cast<cudaStream_t>(stream));
}

int dfk_down_proj(const void *h, const void *w_down, void *y, int B, int d_model, int d_ff,
                  int variant, void *stream) {
  return gemv_impl(DFK_OP_DOWN, h, w_down, y, B, d_ff, d_model, variant,
                   static_cast<cudaStream_t>(stream));
}

int dfk_swiglu_gate_up_fp8(const void *x, const void *q_gate, const float *s_gate,
                           const void *q_up, const float *s_up, void *h, int B, int d_model,
                           int d_ff, int variant, void *stream) {
  return fp8_impl(DFK_OP_GATE_UP_FP8, x, nullptr, 0.f, q_gate, s_gate, q_up, s_up, h, B,
                  d_model, d_ff, variant, static_cast<cudaStream_t>(stream));
}

int dfk_rmsnorm_swiglu_gate_up_fp8(const void *x, const void *gamma, float eps,
                                   const void *q_gate, const float *s_gate, const void *q_up,
                                   const float *s_up, void *h, int B, int d_model, int d_ff,
                                   int variant, void *stream) {
  return fp8_impl(DFK_OP_RMSNORM_GATE_UP_FP8, x, gamma, eps, q_gate, s_gate, q_up, s_up, h, B,
                  d_model, d_ff, variant, static_cast<cudaStream_t>(stream));
}

int dfk_down_proj_fp8(const void *h, const void *q_down, const float *s_down, void *y, int B,
                      int d_model, int d_ff, int variant, void *stream) {
  return fp8_impl(DFK_OP_DOWN_FP8, h, nullptr, 0.f, q_down, s_down, nullptr, nullptr, y, B,
                  d_ff, d_model, variant, static_cast<cudaStream_t>(stream));
}

int dfk_rmsnorm_qkv_proj(const void *x, const void *gamma, float eps, const void *w_qkv,
                         void *q, void *k, void *v, int B, int d_model, int n_q, int n_k,
                         int n_v, int variant, void *stream) {
  return qkv_impl(x, gamma, eps, w_qkv, q, k, v, B, d_model, n_q, n_k, n_v, variant,
                  static_cast<cudaStream_t>(stream));
}

int dfk_gemv(const void *x, const void *w, void *out, int B, int K, int N, int variant,
             void *stream) {
  return gemv_impl(DFK_OP_DOWN, x, w, out, B, K, N, variant, static_cast<cudaStream_t>(stream));
}

int dfk_select_variant(int op, int B, int d_model, int d_ff, int layout,
                       const void *const *sample_ptrs, void *stream, dfk_variant *out) {
  if (!out) return fail(DFK_ERR_INVALID_ARG, "out is NULL");
  if (op < DFK_OP_GATE_UP || op > DFK_OP_RMSNORM_QKV)
    return fail(DFK_ERR_INVALID_ARG, "unknown op %d", op);
  const bool down = op_is_down(op), w8 = op_is_fp8(op), norm = op_is_norm(op);
  const bool qkv = op_is_qkv(op);  // d_ff = n_q + n_k + n_v; one packed output
  if (B <= 0 || B > 64 || d_model <= 0 || d_ff <= 0)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "bad shape B=%d d_model=%d d_ff=%d", B, d_model, d_ff);
  if ((down || w8 || qkv) && layout != DFK_W_ROW_MAJOR && layout != DFK_W_ANY)
    return fail(DFK_ERR_UNSUPPORTED_LAYOUT, "op %d reads row-major weights only", op);
  if (layout != DFK_W_ANY && layout != DFK_W_ROW_MAJOR && layout != DFK_W_COL_MAJOR &&
      layout != DFK_W_GU_INTERLEAVED)
    return fail(DFK_ERR_UNSUPPORTED_LAYOUT, "layout %d", layout);
  if (d_model % 8 || (down && d_ff % 8))
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "sizes must be multiples of 8");
  if (w8 && (down ? d_ff : d_model) % 16)
    return fail(DFK_ERR_UNSUPPORTED_SHAPE, "FP8 weights: reduction length %% 16 != 0");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  if (stream_capturing(s))
    return fail(DFK_ERR_INVALID_ARG, "dfk_select_variant cannot time inside stream capture");

  std::vector<int> layouts;
  if (down || w8 || qkv) layouts = {DFK_W_ROW_MAJOR};
  else if (layout == DFK_W_ANY) layouts = {DFK_W_ROW_MAJOR, DFK_W_COL_MAJOR, DFK_W_GU_INTERLEAVED};
  else layouts = {layout};

  const int K = down ? d_ff : d_model, N = down ? d_model : d_ff, nmat = (down || qkv) ? 1 : 2;
  const size_t xb = static_cast<size_t>(B) * K * 2;
  const size_t wb = static_cast<size_t>(d_model) * d_ff * (w8 ? 1 : 2);
  const size_t ob = static_cast<size_t>(B) * N * 2;
  const size_t sb = w8 ? static_cast<size_t>(N) * sizeof(float) : 0;
  bool best_set = false;
  dfk_variant best{};
  for (int L : layouts) {
    if (L == DFK_W_COL_MAJOR && d_ff % 8) continue;
    const bool own = !sample_ptrs || layout == DFK_W_ANY;
    void *bx = nullptr, *bg = nullptr, *bw = nullptr, *bo = nullptr, *bs = nullptr;
    const void *px = nullptr, *pg = nullptr, *pw0 = nullptr, *pw1 = nullptr;
    const float *ps0 = nullptr, *ps1 = nullptr;
    void *po = nullptr;
    if (own) {
      cudaError_t e = cudaMallocAsync(&bx, xb, s);
      if (!e) e = cudaMallocAsync(&bo, ob, s);
      if (!e && norm) e = cudaMallocAsync(&bg, d_model * 2, s);
      if (!e) e = cudaMallocAsync(&bw, nmat * wb, s);
      if (!e && w8) e = cudaMallocAsync(&bs, nmat * sb, s);
      if (e) {
        cudaGetLastError();
        for (void *q : {bx, bo, bg, bw, bs})
          if (q) cudaFreeAsync(q, s);
        return cuda_fail(e, "cudaMallocAsync (tuning buffers)");
      }
      cudaMemsetAsync(bx, 0, xb, s);
      if (bg) cudaMemsetAsync(bg, 0, d_model * 2, s);
      cudaMemsetAsync(bw, 0, nmat * wb, s);
      if (bs) cudaMemsetAsync(bs, 0, nmat * sb, s);
      px = bx; pg = bg; po = bo; pw0 = bw;
      pw1 = (nmat == 1 || L == DFK_W_GU_INTERLEAVED) ? nullptr : static_cast<char *>(bw) + wb;
      ps0 = static_cast<const float *>(bs);
      ps1 = (bs && nmat == 2) ? static_cast<const float *>(bs) + N : nullptr;
    } else {
      // argument order of the op's entry point
      int i = 0;
      px = sample_ptrs[i++];
      if (norm) pg = sample_ptrs[i++];
      pw0 = sample_ptrs[i++];
      if (w8) ps0 = static_cast<const float *>(sample_ptrs[i++]);
      if (!down && !qkv) {
        pw1 = sample_ptrs[i++];
        if (w8) ps1 = static_cast<const float *>(sample_ptrs[i++]);
      }
      po = const_cast<void *>(sample_ptrs[i++]);
    }
    CcCall c;
    if (down || qkv) c = CcCall{LAYOUT_ROW, 1, norm, px, pg, 1e-5f, pw0, nullptr, po, B, K, N};
    else c = CcCall{to_engine_layout(L), 2, norm, px, pg, 1e-5f, pw0,
                    L == DFK_W_GU_INTERLEAVED ? nullptr : pw1, po, B, K, N};
    c.w8 = w8;
    c.s0 = ps0;
    c.s1 = ps1;
    float us = -1.f;
    int stages = 0;
    const VDef *win = time_candidates(op, c, candidates(op, B, c), s, *ds, &us, &stages);
    if (!win) {
      win = heuristic(op, B, c, *ds);
      us = -1.f;
    }
    if (own) {
      for (void *q : {bx, bo, bg, bw, bs})
        if (q) cudaFreeAsync(q, s);
      cudaStreamSynchronize(s);
    }
    if (!win) continue;
    dfk_variant rec;
    fill_variant(*win, op, L, stages, us, &rec);
    {
      TuneKey key{dev, op, B, d_model, d_ff, L};
      std::lock_guard<std::mutex> lk(g_tune_mu);
      tune_cache_load(dev, ds->sms);
      g_tuned[key] = rec;
      if (us >= 0) tune_cache_append(dev, ds->sms, key, rec);
    }
    if (!best_set || (us >= 0 && (best.measured_us < 0 || us < best.measured_us))) {
      best = rec;
      best_set = true;
    }
  }
  if (!best_set) return fail(DFK_ERR_NO_VARIANT, "no variant fits this shape");
  *out = best;
  return DFK_OK;
}

int dfk_cached_variant(int op, int B, int d_model, int d_ff, int layout, dfk_variant *out) {
  if (!out) return fail(DFK_ERR_INVALID_ARG, "out is NULL");
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  TuneKey key{dev, op, B, d_model, d_ff, layout};
  std::lock_guard<std::mutex> lk(g_tune_mu);
  tune_cache_load(dev, ds->sms);
  auto it = g_tuned.find(key);
  if (it == g_tuned.end()) return fail(DFK_ERR_NO_VARIANT, "no cached decision for this shape");
  *out = it->second;
  return DFK_OK;
}

long long dfk_mlp_stack_workspace_bytes(int layers, int B, int d_model, int d_ff) {
  DeviceState *ds;
  if (dfk::current_device(&ds)) return -1;
  dfk::PsPlan pl;
  std::string why;
  if (!dfk::plan_pstack(layers, B, d_model, d_ff, ds->sms, std::min(ds->smem_optin, 232448),
                        &pl, &why)) {
    dfk::fail(DFK_ERR_UNSUPPORTED_SHAPE, "persistent decode step: %s", why.c_str());
    return -1;
  }
  return static_cast<long long>(pl.ws_ctl + pl.ws_part);
}

int dfk_mlp_stack_step(const void *gammas, float eps, const void *w_gate, const void *w_up,
                       int layout, const void *w_down, void *x, void *h_all, void *y_all,
                       void *workspace, long long workspace_bytes, int layers, int B,
                       int d_model, int d_ff, void *stream) {
  if (workspace_bytes < 0) return dfk::fail(DFK_ERR_INVALID_ARG, "negative workspace size");
  return dfk::pstack_step(gammas, eps, w_gate, w_up, layout, w_down, x, h_all, y_all, workspace,
                          static_cast<size_t>(workspace_bytes), layers, B, d_model, d_ff,
                          static_cast<cudaStream_t>(stream));
}

int dfk_variant_count(void) { return static_cast<int>(variants().size()); }

int dfk_variant_info(int variant_id, dfk_variant *out) {
  if (!out) return fail(DFK_ERR_INVALID_ARG, "out is NULL");
  const VDef *d = find_variant(variant_id);
  if (!d) return fail(DFK_ERR_INVALID_ARG, "no variant %d", variant_id);
  const int op = d->e4m3mma ? (d->cls == CLS_GEMV ? DFK_OP_DOWN_FP8 : DFK_OP_GATE_UP_FP8)
                            : (d->cls == CLS_GEMV ? DFK_OP_DOWN : DFK_OP_GATE_UP);
  fill_variant(*d, op, -1, 0, -1.f, out);
  return DFK_OK;
}

void dfk_clear_variant_cache(void) {
  std::lock_guard<std::mutex> lk(g_tune_mu);
  g_tuned.clear();
}

int dfk_rmsnorm(const void *x, const void *gamma, float eps, void *xn, int B, int d,
                void *stream) {
  if (B < 0 || d <= 0) return fail(DFK_ERR_INVALID_ARG, "negative or zero size");
  if (!(eps >= 0.f && std::isfinite(eps))) return fail(DFK_ERR_INVALID_ARG, "bad eps");
  if (d % 8) return fail(DFK_ERR_UNSUPPORTED_SHAPE, "d %% 8 != 0");
  if (B == 0) return DFK_OK;
  if (!x || !xn) return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if (misaligned(x) || misaligned(xn) || (gamma && misaligned(gamma)))
    return fail(DFK_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
  DeviceState *ds;
  int rc = current_device(&ds);
  if (rc) return rc;
  cudaError_t e = launch_rmsnorm_rows(x, gamma, eps, xn, B, d, static_cast<cudaStream_t>(stream),
                                      pdl_enabled());
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "rmsnorm launch");
  }
  return DFK_OK;
}

int dfk_rms_rescale(const void *y, float eps, void *x_next, int B, int d, void *stream) {
  return dfk_rmsnorm(y, nullptr, eps, x_next, B, d, stream);
}

static int ew_check(const void *a, const void *b, const void *out, long long n, bool two) {
  if (n < 0) return fail(DFK_ERR_INVALID_ARG, "negative size");
  if (n == 0) return DFK_OK;
  if (!a || !out || (two && !b)) return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(out) |
       reinterpret_cast<uintptr_t>(b)) & 1u)
    return fail(DFK_ERR_MISALIGNED, "bf16 pointers must be 2-byte aligned");
  return DFK_OK;
}

int dfk_silu(const void *a, void *out, long long n, void *stream) {
  int rc = ew_check(a, nullptr, out, n, false);
  if (rc || n == 0) return rc;
  DeviceState *ds;
  if ((rc = current_device(&ds))) return rc;
  cudaError_t e = launch_silu(a, out, n, static_cast<cudaStream_t>(stream), pdl_enabled());
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "silu launch");
  }
  return DFK_OK;
}

int dfk_mul(const void *a, const void *b, void *out, long long n, void *stream) {
  int rc = ew_check(a, b, out, n, true);
  if (rc || n == 0) return rc;
  DeviceState *ds;
  if ((rc = current_device(&ds))) return rc;
  cudaError_t e = launch_mul(a, b, out, n, static_cast<cudaStream_t>(stream), pdl_enabled());
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "mul launch");
  }
  return DFK_OK;
}

}  // extern "C"

namespace dfk {

// ---- dfk_mlp_forward_host: one layer from host memory.  With pinned host
// buffers the whole step (copy in, fused gate/up, down projection, copy out)
// is replayed as one CUDA graph per distinct argument set; the graph is
// captured on an internal stream after one eager run there (which settles
// the scheduler's decisions and the split-K workspace of that stream).

struct HostCall {
  const void *x_host, *gamma;
  float eps;
  const void *w_gate, *w_up;
  int layout;
  const void *w_down;
  void *y_host, *x_dev, *h_dev, *y_dev;
  int B, d_model, d_ff;
};

using HostKey = std::tuple<int, uintptr_t, uintptr_t, uintptr_t, uintptr_t, uintptr_t,
                           uintptr_t, uintptr_t, uintptr_t, uintptr_t, uintptr_t, int, int,
                           int, int, uint32_t>;
static std::mutex g_host_mu;
static std::map<HostKey, cudaGraphExec_t> g_host_graphs;  // nullptr: capture failed, run eager
static std::map<int, cudaStream_t> g_capture_streams;

// Device address of a pinned host buffer (unified addressing), or nullptr.
static void *mapped_host_ptr(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

static int forward_host_enqueue(const HostCall &a, cudaStream_t s) {
  const size_t xb = static_cast<size_t>(a.B) * a.d_model * 2;
  // pinned, device-addressable host buffers: copy kernels (which overlap the
  // neighbouring kernels through programmatic dependent launch); otherwise
  // copy-engine transfers
  void *xh = mapped_host_ptr(a.x_host), *yh = mapped_host_ptr(a.y_host);
  const bool kern = xh && yh && xb % 16 == 0 &&
                    ((reinterpret_cast<uintptr_t>(xh) | reinterpret_cast<uintptr_t>(yh)) & 15u) == 0;
  cudaError_t e = kern ? launch_copy16(xh, a.x_dev, xb, false, s, pdl_enabled())
                       : cudaMemcpyAsync(a.x_dev, a.x_host, xb, cudaMemcpyHostToDevice, s);
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "copy x to device");
  }
  int rc = a.gamma ? dfk_rmsnorm_swiglu_gate_up(a.x_dev, a.gamma, a.eps, a.w_gate, a.w_up,
                                                a.layout, a.h_dev, a.B, a.d_model, a.d_ff, 0, s)
                   : dfk_swiglu_gate_up(a.x_dev, a.w_gate, a.w_up, a.layout, a.h_dev, a.B,
                                        a.d_model, a.d_ff, 0, s);
  if (rc) return rc;
  if ((rc = dfk_down_proj(a.h_dev, a.w_down, a.y_dev, a.B, a.d_model, a.d_ff, 0, s))) return rc;
  e = kern ? launch_copy16(a.y_dev, yh, xb, true, s, pdl_enabled())
           : cudaMemcpyAsync(a.y_host, a.y_dev, xb, cudaMemcpyDeviceToHost, s);
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "copy y to host");
  }
  return DFK_OK;
}

static bool pinned_host(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

static int forward_host_graph(const HostCall &a, int dev, cudaStream_t s, bool *done) {
  *done = false;
  uint32_t eps_bits;
  memcpy(&eps_bits, &a.eps, sizeof eps_bits);
  const HostKey key{dev, reinterpret_cast<uintptr_t>(s), reinterpret_cast<uintptr_t>(a.x_host),
                    reinterpret_cast<uintptr_t>(a.gamma), reinterpret_cast<uintptr_t>(a.w_gate),
                    reinterpret_cast<uintptr_t>(a.w_up), reinterpret_cast<uintptr_t>(a.w_down),
                    reinterpret_cast<uintptr_t>(a.y_host), reinterpret_cast<uintptr_t>(a.x_dev),
                    reinterpret_cast<uintptr_t>(a.h_dev), reinterpret_cast<uintptr_t>(a.y_dev),
                    a.layout, a.B, a.d_model, a.d_ff, eps_bits};
  std::lock_guard<std::mutex> lk(g_host_mu);
  auto it = g_host_graphs.find(key);
  if (it != g_host_graphs.end()) {
    if (!it->second) return DFK_OK;  // known not capturable: caller runs eagerly
    cudaError_t e = cudaGraphLaunch(it->second, s);
    if (!e) e = cudaStreamSynchronize(s);
    if (e) {
      cudaGetLastError();
      return cuda_fail(e, "forward graph replay");
    }
    *done = true;
    return DFK_OK;
  }
  cudaStream_t &cs = g_capture_streams[dev];
  cudaError_t e = cudaSuccess;
  if (!cs) e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
  cudaEvent_t ready = nullptr;
  if (!e) e = cudaEventCreateWithFlags(&ready, cudaEventDisableTiming);
  if (!e) e = cudaEventRecord(ready, s);  // after the caller's earlier work on s
  if (!e) e = cudaStreamWaitEvent(cs, ready, 0);
  if (ready) cudaEventDestroy(ready);
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "forward graph set-up");
  }
  // eager run on the capture stream: this call's result
  int rc = forward_host_enqueue(a, cs);
  if (!rc && (e = cudaStreamSynchronize(cs))) {
    cudaGetLastError();
    rc = cuda_fail(e, "forward on the capture stream");
  }
  if (rc) return rc;
  *done = true;
  // capture the same step for the next calls
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (!e) {
    rc = forward_host_enqueue(a, cs);
    cudaError_t e2 = cudaStreamEndCapture(cs, &graph);
    if (!rc && !e2 && graph) e = cudaGraphInstantiate(&exec, graph, 0);
    else e = e2 ? e2 : cudaErrorUnknown;
  }
  if (graph) cudaGraphDestroy(graph);
  if (e || rc) {
    cudaGetLastError();
    exec = nullptr;
    log_msg("forward graph capture failed; this argument set runs eagerly");
  }
  if (g_host_graphs.size() >= 64) {  // bounded cache
    for (auto &kv : g_host_graphs)
      if (kv.second) cudaGraphExecDestroy(kv.second);
    g_host_graphs.clear();
  }
  g_host_graphs[key] = exec;
  return DFK_OK;
}

}  // namespace dfk

extern "C" {

int dfk_mlp_forward_host(const void *x_host, const void *gamma, float eps, const void *w_gate,
                         const void *w_up, int layout, const void *w_down, void *y_host,
                         void *x_dev, void *h_dev, void *y_dev, int B, int d_model, int d_ff,
                         void *stream) {
  if (B < 0) return fail(DFK_ERR_INVALID_ARG, "negative batch");
  if (B == 0) return DFK_OK;
  if (!x_host || !y_host || !x_dev || !h_dev || !y_dev || !w_down)
    return fail(DFK_ERR_INVALID_ARG, "null pointer argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const HostCall a{x_host, gamma, eps, w_gate, w_up, layout, w_down, y_host, x_dev, h_dev,
                   y_dev, B, d_model, d_ff};
  DeviceState *ds;
  int dev;
  int rc = current_device(&ds, &dev);
  if (rc) return rc;
  if (env_flag("DFK_HOST_GRAPH", true) && !stream_capturing(s) && pinned_host(x_host) &&
      pinned_host(y_host)) {
    bool done = false;
    if ((rc = forward_host_graph(a, dev, s, &done))) return rc;
    if (done) return DFK_OK;
  }
  if ((rc = forward_host_enqueue(a, s))) return rc;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "forward synchronise");
  }
  return DFK_OK;
}

const char *dfk_status_string(int status) {
  switch (status) {
    case DFK_OK: return "ok";
    case DFK_ERR_INVALID_ARG: return "invalid argument";
    case DFK_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DFK_ERR_UNSUPPORTED_LAYOUT: return "unsupported layout";
    case DFK_ERR_MISALIGNED: return "misaligned pointer";
    case DFK_ERR_CUDA: return "CUDA error";
    case DFK_ERR_ARCH: return "no sm_100 device";
    case DFK_ERR_TIMEOUT: return "device pipeline wait timed out";
    case DFK_ERR_NO_VARIANT: return "no variant fits this shape";
    case DFK_ERR_BOUNDS: return "a kernel's bounds check failed";
    default: return "unknown status";
  }
}

const char *dfk_last_error(void) { return t_last_error.c_str(); }

int dfk_device_error(int *code) {
  if (!code) return fail(DFK_ERR_INVALID_ARG, "code is NULL");
  DeviceState *ds;
  int rc = current_device(&ds);
  if (rc) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  unsigned v[2] = {0u, 0u};
  if (!e) e = cudaMemcpyFromSymbol(v, g_dfk_err, sizeof v);
  const unsigned zero[2] = {0u, 0u};
  if (!e) e = cudaMemcpyToSymbol(g_dfk_err, zero, sizeof zero);
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "reading the device error word");
  }
  *code = static_cast<int>(v[0]);
  if (v[0] & dfk::ERR_BOUNDS)
    return fail(DFK_ERR_BOUNDS, "bounds check failed (first at site %u, source line %u)",
                v[1] >> 16, v[1] & 0xffffu);
  if (v[0]) return fail(DFK_ERR_TIMEOUT, "a kernel's pipeline wait gave up");
  return DFK_OK;
}

int dfk_set_wait_limit(unsigned long long ns) {
  DeviceState *ds;
  int rc = current_device(&ds);
  if (rc) return rc;
  // words 2-3 of the status block; a plain copy, ordered after work already
  // queued on the legacy default stream
  cudaError_t e = cudaMemcpyToSymbol(g_dfk_err, &ns, sizeof ns, 2 * sizeof(unsigned));
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "setting the wait limit");
  }
  return DFK_OK;
}

int dfk_selftest_bounded_wait(void *elapsed_ns, void *stream) {
  if (!elapsed_ns) return fail(DFK_ERR_INVALID_ARG, "elapsed_ns is NULL");
  if (reinterpret_cast<uintptr_t>(elapsed_ns) & 7u)
    return fail(DFK_ERR_MISALIGNED, "elapsed_ns must be 8-byte aligned");
  DeviceState *ds;
  int rc = current_device(&ds);
  if (rc) return rc;
  cudaError_t e = dfk::launch_wait_selftest(ds->err, static_cast<unsigned long long *>(elapsed_ns),
                                            static_cast<cudaStream_t>(stream));
  if (e) {
    cudaGetLastError();
    return cuda_fail(e, "wait self-test launch");
  }
  return DFK_OK;
}

const char *dfk_version(void) { return "dfk 0.1.0 sm_100a"; }

}  // extern "C"
