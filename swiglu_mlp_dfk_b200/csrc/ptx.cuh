// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor
// loads, programmatic dependent launch, bounded waits.
#pragma once
#include <cuda.h>
#include <cstdint>

namespace dfk {

// Device status block (one per device, read by dfk_device_error): word 0
// holds the error bits, word 1 the site of the first failed bounds check
// (checked builds), words 2-3 the pipeline-wait limit in ns as a 64-bit
// value (0 = the default), set by dfk_set_wait_limit.  Every kernel gets a
// pointer to word 0 (`err`).
constexpr unsigned ERR_WAIT_TIMEOUT = 1u;
constexpr unsigned ERR_BOUNDS = 2u;
constexpr int STATUS_WORDS = 4;

// Checked builds (-DDFK_CHECKED): the kernels test the index of every global
// store of a result and of the activation loads against the tensor's extent
// first; a failed test skips the access, records the first failing check in
// word 1 of the status block (site number << 16 | source line) and sets
// ERR_BOUNDS -- never a trap.  In ordinary builds the test compiles away.
#ifdef DFK_CHECKED
static __device__ __noinline__ void bounds_failed(unsigned *err, unsigned site_line) {
  if (err) {
    atomicCAS(err + 1, 0u, site_line);
    atomicOr(err, 2u);
  }
}
#define DFK_IN_BOUNDS(cond, site, err)                                                  \
  ((cond) || (::dfk::bounds_failed((err), (static_cast<unsigned>(site) << 16) |          \
                                              (static_cast<unsigned>(__LINE__) & 0xffffu)), \
              false))
#else
#define DFK_IN_BOUNDS(cond, site, err) true
#endif

// A pipeline wait gives up after this long by default (the data it waits
// for arrives in microseconds in a healthy run).
constexpr unsigned long long WAIT_TIMEOUT_NS = 4000000000ull;

// The wait limit in force for kernels given the status block `err`.
__device__ __forceinline__ unsigned long long wait_limit_ns(const unsigned *err) {
  if (!err) return WAIT_TIMEOUT_NS;
  const unsigned long long v =
      *reinterpret_cast<const volatile unsigned long long *>(err + 2);
  return v ? v : WAIT_TIMEOUT_NS;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// (returns false) when *abort_flag becomes non-zero, or after the wait
// limit, in which case it sets *abort_flag and the device error word.
// Pipeline waits (abort_flag given) use the limit set for the device
// (dfk_set_wait_limit, default WAIT_TIMEOUT_NS); the waits at exit for
// copies and MMAs still in flight (abort_flag == nullptr) always allow the
// default, so a short limit never lets a CTA leave while its shared memory
// is still being written.  Never spins unboundedly.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort_flag, unsigned *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long limit = abort_flag ? wait_limit_ns(err) : WAIT_TIMEOUT_NS;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (global_timer_ns() - t0 > limit || it > (1u << 30)) {
        if (abort_flag) *abort_flag = 1;
        if (err) atomicOr(err, ERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// System-scope release store / acquire load of a 64-bit flag (peer memory
// over NVLink included).
__device__ __forceinline__ void st_release_sys_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_sys_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Wait until each of the n flags fl[0 .. n) holds a value >= want.  Bounded
// like mbar_wait_bounded: gives up when *abort_flag becomes non-zero or after
// the device's wait limit (then sets *abort_flag and the error word).
__device__ __forceinline__ bool flags_wait_bounded(const unsigned long long *fl, int n,
                                                   unsigned long long want,
                                                   volatile int *abort_flag, unsigned *err) {
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long limit = wait_limit_ns(err);
  for (int s = 0; s < n; ++s) {
    for (uint32_t it = 1; ld_acquire_sys_u64(fl + s) < want; ++it) {
      if ((it & 15u) == 0) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit || it > (1u << 30)) {
          *abort_flag = 1;
          if (err) atomicOr(err, ERR_WAIT_TIMEOUT);
          return false;
        }
      }
      __nanosleep(32);
    }
  }
  return true;
}

// Bulk tensor copy global -> shared, 2-D tile, completion counted on `bar`.
// The innermost coordinate c0 times the element size must be a multiple of
// 16 bytes (callers pass multiples of 8 bf16 elements).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

// Bulk tensor prefetch global -> L2 of the box a tma_load_2d with the same map
// and coordinates would copy (no shared memory, no barrier; boxes past the
// tensor bounds are clipped by the map).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// L2 policy: weights are streamed once per call -> evict first.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Programmatic dependent launch: allow the next kernel in the stream to
// start its prologue, and wait for the previous kernel's memory.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Named barrier over `nthreads` threads (multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Read-only 16-byte global load that bypasses L1 allocation.
__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// bf16 halves of a 32-bit word -> fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Four FP8 E4M3 codes (byte i of w = element i) -> their fp32 values.  Each
// pair goes through the hardware E4M3x2 -> f16x2 conversion and then f16 ->
// f32; both steps are exact (every E4M3 value, subnormals included, is an
// f16 value), so f[i] is the code's value with no rounding.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float (&f)[4]) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(h01), "=r"(h23)
      : "r"(w));
  asm("{\n\t.reg .b16 a, b, c, d;\n\t"
      "mov.b32 {a, b}, %4;\n\t"
      "mov.b32 {c, d}, %5;\n\t"
      "cvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t"
      "cvt.f32.f16 %2, c;\n\t"
      "cvt.f32.f16 %3, d;\n\t}"
      : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3])
      : "r"(h01), "r"(h23));
}

// FP8 E4M3 -> bf16 without the conversion unit (whose throughput is a
// quarter of the ALU's): for a code c = s.eeee.mmm, the 16 bits
// (c & 0x7F) << 4 read as bf16 have exponent field e and mantissa mmm0000,
// i.e. the value |E4M3(c)| * 2^-120 exactly (e = 0 gives the bf16 subnormal
// m * 2^-129); one bf16x2 multiply by 2^120 (exact) restores the scale and
// the sign bit is or-ed in.  Per pair of codes: a byte permute, a shift, a
// mask, a multiply and an or.  The NaN code S.1111.111 is not special:
// it comes out as +-480.
__device__ __forceinline__ uint32_t e4m3x2_bits_to_bf16x2(uint32_t b) {
  // b holds code 0 in bits 15..8 and code 1 in bits 31..24 (other bits 0)
  const uint32_t mag = (b >> 4) & 0x07F007F0u;
  uint32_t v;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(v) : "r"(mag), "r"(0x7B807B80u));  // x 2^120
  return v | (b & 0x80008000u);
}

__device__ __forceinline__ void e4m3x4_to_bf16x2_alu(uint32_t w, uint32_t &lo, uint32_t &hi) {
  lo = e4m3x2_bits_to_bf16x2(__byte_perm(w, 0u, 0x1404));  // [c1, 0, c0, 0]
  hi = e4m3x2_bits_to_bf16x2(__byte_perm(w, 0u, 0x3424));  // [c3, 0, c2, 0]
}

// Two fp32 values in one 64-bit register (lo = first element).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Packed fused multiply-add: each lane computes fma(a, b, c) with one
// rounding, exactly as fmaf does.
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// fp32 -> bf16 bits, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

__device__ __forceinline__ float round_bf16(float f) {
  return __uint_as_float(static_cast<uint32_t>(f32_to_bf16_bits(f)) << 16);
}

// Output element (b, j): row j of the one output, or of its q / k / v part.
template <typename P>
__device__ __forceinline__ void store_out(const P &p, int b, int j, uint16_t v) {
  if (!DFK_IN_BOUNDS(b >= 0 && b < p.B && j >= 0 && j < p.N, 1, p.err)) return;
  if (p.outs[0] == nullptr) {
    p.out[static_cast<size_t>(b) * p.N + j] = v;
  } else if (j < p.split[0]) {
    p.outs[0][static_cast<size_t>(b) * p.split[0] + j] = v;
  } else if (j < p.split[1]) {
    p.outs[1][static_cast<size_t>(b) * (p.split[1] - p.split[0]) + (j - p.split[0])] = v;
  } else {
    p.outs[2][static_cast<size_t>(b) * (p.N - p.split[1]) + (j - p.split[1])] = v;
  }
}

// Split-K tail for output row `row` of row block `blk`: adds the kslices
// (<= 8) fp32 partial sums of tokens 0 .. B-1 in slice order (slice 0
// first) and hands each total to emit(n, total).  The loads of a batch of
// tokens x all slices (64 values: 16 tokens at up to 4 slices, 8 at up to 8)
// are issued before any add, so the tail costs a few L2 round trips rather
// than one per token.  part: [kslices][nblocks][bnp][128].
constexpr int SPLITK_MAX = 8;

template <int KSM, typename Emit>
__device__ __forceinline__ void splitk_reduce_row_n(const float *part, int kslices, int nblocks,
                                                    int blk, int bnp, int B, int row,
                                                    Emit emit) {
  constexpr int TB = 64 / KSM;
  for (int n0 = 0; n0 < B; n0 += TB) {
    float v[TB][KSM];
#pragma unroll
    for (int i = 0; i < TB; ++i)
#pragma unroll
      for (int sl = 0; sl < KSM; ++sl)
        v[i][sl] = (n0 + i < B && sl < kslices)
                       ? __ldcg(part + ((static_cast<size_t>(sl) * nblocks + blk) * bnp + n0 + i) *
                                           128 + row)
                       : 0.f;
#pragma unroll
    for (int i = 0; i < TB; ++i) {
      if (n0 + i < B) {
        float acc = v[i][0];
#pragma unroll
        for (int sl = 1; sl < KSM; ++sl)
          if (sl < kslices) acc = acc + v[i][sl];
        emit(n0 + i, acc);
      }
    }
  }
}

template <typename Emit>
__device__ __forceinline__ void splitk_reduce_row(const float *part, int kslices, int nblocks,
                                                  int blk, int bnp, int B, int row, Emit emit) {
  splitk_reduce_row_n<SPLITK_MAX>(part, kslices, nblocks, blk, bnp, B, row, emit);
}

}  // namespace dfk
