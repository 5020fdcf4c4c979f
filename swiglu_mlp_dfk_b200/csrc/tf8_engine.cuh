// tf8_engine.cuh -- tensor-core weight-streaming kernel for FP8 E4M3 weights
// with one fp32 scale per output row (W[j][k] = s[j] * E4M3(q[j][k])).
//
// The operation is the one of the bf16 kernels ("Deep Kernel Fusion for
// Transformer Decoding", episode description: gate, up, SiLU and multiply in
// one decode kernel; the down projection is the NMAT = 1 instance), with the
// dequantisation fused into the matrix product as GPULlama3.java PR #78 does
// for its quantised matrix-vector kernels: codes stream from HBM at one byte
// per weight and are widened on chip, never written back.
//
// Why the dequantised weights go to TMEM: kind::f16 needs A and B of one
// type, and the activations are bf16, so the codes become bf16 (exactly, by
// integer bit placement and one bf16 multiply: the conversion unit would
// bound the kernel at a third of HBM speed).  Writing them to shared memory for
// the MMA would cost 1 (TMA) + 1 (read) + 2 (write) + 2 (MMA read) bytes of
// shared-memory traffic per weight, about the whole shared-memory bandwidth
// at HBM speed; with A in TMEM (tcgen05.st, then an MMA that reads A from
// TMEM) shared memory carries 2 bytes per weight.
//
// Work split: a CTA owns r <= 128 consecutive output rows (one M = 128 MMA
// tile; TMEM lane m = row m) over its reduction range (the whole K, or one
// of `kslices` slices for the split-K GEMV).  One ring stage holds one
// 128-wide k tile: the codes of every matrix (TMA, 128-byte swizzle) and the
// activations as two 64-wide bf16 sub-tiles (TMA, 128-byte swizzle).
//
// Warp roles (576 threads): warp 0 issues TMA copies; warp 1 owns TMEM and
// issues the MMAs (one elected lane); warps 2-17 dequantise -- the four warps of a
// TMEM lane quarter split a tile's 128 codes per row into parts of 32, each
// thread converts its row's 32 codes and stores 16 columns with tcgen05.st
// into one of two A buffers -- and with the RMSNorm prologue also split x *
// gamma into bf16 hi + lo (exact) and accumulate sum x^2, as the bf16
// tensor-core kernel does.  Warps 2-5 then run the epilogue: accumulator ->
// registers, times r_b (RMSNorm) and the row scale s[j], SiLU(gate) * up,
// one bf16 store.  Split-K slices leave fp32 partial sums; the last CTA of a
// row block adds them in slice order, scales and stores.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "tc_engine.cuh"
#include "tc_ptx.cuh"

namespace dfk {

constexpr int TF8_XFORM = 512;                 // dequantise / transform threads
constexpr int TF8_THREADS = 64 + TF8_XFORM;    // + TMA warp + MMA warp
constexpr int TF8_TILE_K = 128;  // reduction elements per ring stage (one 128-byte code row)

struct Tf8Params {
  uint16_t *out;          // [B][N] bf16
  const uint16_t *gamma;  // [K] bf16 (NORM)
  const float *scale[2];  // per-row scales [N] of each matrix
  unsigned *err;          // device error word
  int B, K, N;
  float eps;
  int rbase, rextra;      // rows per row block: rbase, +1 for the first rextra blocks
  int hmax;               // code box height of map 0; map 1 is hmax - 1
  int r8;                 // rows reserved per code tile in shared memory (multiple of 8)
  int bn;                 // tokens on N: 16, 32 or 64
  int stages, stage_bytes;
  int a8_bytes;           // code bytes of one stage: NMAT * r8 * 128
  int xt_bytes;           // bytes of one 64-wide activation sub-tile: bn * 128 (x2 with NORM)
  int tmem_cols;          // allocated TMEM columns
  int acol;               // first TMEM column of the two A buffers
  int g_off, bar_off;     // shared-memory offsets from the 1024-byte aligned base
  int ntiles;             // 128-wide k tiles covering K
  int kslices;            // split-K slices (GEMV only; 1 = none)
  float *part;            // [kslices][nblocks][bn][128] fp32 partial sums
  unsigned *counters;     // [nblocks], 0 between calls
  int nblocks;            // row blocks
};

// w[m][0]: codes of matrix m, box {128, hmax}; w[m][1]: box {128, hmax - 1};
// x: activations, box {64, bn}.  All with 128-byte swizzle.
struct Tf8Maps {
  CUtensorMap w[2][2];
  CUtensorMap x;
};

template <int NMAT, bool NORM>
__global__ void __launch_bounds__(TF8_THREADS, 1)
    tf8_gemv_kernel(const __grid_constant__ Tf8Maps maps, const Tf8Params p) {
  static_assert(NMAT == 1 || NMAT == 2, "NMAT");
  static_assert(!NORM || NMAT == 2, "the RMSNorm prologue belongs to the gate/up kernel");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.stages, BN = p.bn;
  const int WN = NORM ? 2 * BN : BN;

  uint64_t *fullb = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = fullb + S;
  constexpr int NAB = 2;
  uint64_t *aready = empty + S;     // [NAB]: A buffer written (and x transformed)
  uint64_t *aempty = aready + NAB;  // [NAB]: MMAs reading the A buffer have completed
  uint64_t *accfull = aempty + NAB;
  volatile int *s_abort = reinterpret_cast<volatile int *>(accfull + 1);
  int *s_issued = reinterpret_cast<int *>(accfull + 1) + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(accfull + 1) + 2;
  volatile int *s_last = reinterpret_cast<volatile int *>(accfull + 1) + 3;
  float *s_rinv = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(accfull + 1) + 16);
  uint16_t *gs = reinterpret_cast<uint16_t *>(smem + p.g_off);

  // ---- this CTA's rows [j0, j0 + r) and k tiles [tile0, tile1)
  const int cta = blockIdx.x;
  const int blk = cta / p.kslices, slc = cta - blk * p.kslices;
  const int j0 = blk * p.rbase + min(blk, p.rextra);
  const int r = p.rbase + (blk < p.rextra ? 1 : 0);
  const int mi = (r == p.hmax) ? 0 : 1;
  const int tile0 = (slc * p.ntiles) / p.kslices;
  const int tile1 = ((slc + 1) * p.ntiles) / p.kslices;
  const int nsteps = tile1 - tile0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullb[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NAB; ++b) {
      mbar_init(&aready[b], TF8_XFORM);
      mbar_init(&aempty[b], 1);
    }
    mbar_init(accfull, 1);
    *s_abort = 0;
    *s_issued = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  pdl_launch_dependents();

  if (warp == 0) {
    // ================= TMA producer (one lane)
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_normal();
      const int S0 = min(S, nsteps);
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S;
        if (i >= S && !mbar_wait_bounded(&empty[st], ((i / S) - 1) & 1, s_abort, p.err)) break;
        uint8_t *sb = smem + static_cast<size_t>(st) * p.stage_bytes;
        const int k0 = (tile0 + i) * TF8_TILE_K;
        const int nx = (p.K - k0 > 64) ? 2 : 1;  // activation sub-tiles inside K
        mbar_arrive_expect_tx(&fullb[st], static_cast<uint32_t>(NMAT * r * 128 + nx * BN * 128));
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
          tma_load_2d(sb + m * p.r8 * 128, &maps.w[m][mi], &fullb[st], k0, j0, pol_w);
        // activations: only after the previous kernel's results are visible
        if (i >= S0)
          for (int h = 0; h < nx; ++h)
            tma_load_2d(sb + p.a8_bytes + h * p.xt_bytes, &maps.x, &fullb[st], k0 + 64 * h, 0,
                        pol_x);
        if (i == S0 - 1) {
          pdl_wait();
          for (int ii = 0; ii < S0; ++ii) {
            const int k0i = (tile0 + ii) * TF8_TILE_K;
            const int nxi = (p.K - k0i > 64) ? 2 : 1;
            for (int h = 0; h < nxi; ++h)
              tma_load_2d(smem + static_cast<size_t>(ii) * p.stage_bytes + p.a8_bytes +
                              h * p.xt_bytes,
                          &maps.x, &fullb[ii], k0i + 64 * h, 0, pol_x);
          }
        }
        issued = i + 1;
      }
      *s_issued = issued;
    }
  } else if (warp == 1) {
    // ================= MMA issuer: per stage, the k-slices of 16 inside K,
    // A from TMEM buffer (i mod NAB), B from the activation sub-tile (k-slice
    // kk: sub-tile kk / 4, 32 bytes per slice inside its swizzled rows).  The
    // whole warp walks the ring (warp-uniform descriptors); one elected lane
    // issues.
    __syncwarp();
    const uint32_t leader = elect_one_sync();
    {
      const uint32_t idesc = umma_idesc_bf16_f32(128, WN);
      const uint64_t desc0 = umma_desc_sw128(sbase);
      const uint32_t x_enc = static_cast<uint32_t>(p.a8_bytes) >> 4;
      const uint32_t xt_enc = static_cast<uint32_t>(p.xt_bytes) >> 4;
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S, slot = i % NAB;
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(&aready[slot], (i / NAB) & 1, s_abort, p.err)))
          break;
        tc_fence_after();
        const int k0 = (tile0 + i) * TF8_TILE_K;
        const int nk = min(8, (p.K - k0) / 16);
        const uint64_t bx = desc0 + (static_cast<uint32_t>(st * p.stage_bytes) >> 4) + x_enc;
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t b = bx + (kk >> 2) * xt_enc + 2 * (kk & 3);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint32_t a = tmem + static_cast<uint32_t>(p.acol + (slot * NMAT + m) * 64 + 8 * kk);
            if (leader)
              umma_bf16_ts(tmem + static_cast<uint32_t>(m * WN), a, b, idesc,
                           (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (leader) {
          umma_commit(&empty[st]);     // the stage's activations have been read
          umma_commit(&aempty[slot]);  // and so has the A buffer
        }
        __syncwarp();
      }
      if (leader) umma_commit(accfull);  // every MMA issued above has completed
    }
  } else {
    // ================= dequantise / x * gamma transform: warps 2..17
    const int et = tid - 64;           // 0 .. TF8_XFORM - 1
    const int q = warp & 3;            // TMEM lane quarter this warp may address
    const int part = (warp - 2) >> 2;  // 32-code part of a tile row: k 32 part .. 32 part + 31
    const int row = 32 * q + lane;     // A row (TMEM lane) this thread widens
    if (NORM) {
      pdl_wait();
      const int kpad = p.ntiles * TF8_TILE_K;
      for (int idx = et; idx < kpad / 8; idx += TF8_XFORM) {
        const int k = idx * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k < p.K) v = ld_nc_v4(p.gamma + k);
        *reinterpret_cast<uint4 *>(gs + k) = v;
      }
      named_barrier(1, TF8_XFORM);
    }
    // x * gamma: thread et < 8 bn owns 16-byte chunk pc = et & 7 of token row
    // n = et >> 3 in every 64-wide sub-tile; the 8 lanes of a row reduce its
    // sum of squares (the order of the bf16 tensor-core kernel)
    const int pc = et & 7, xn_row = et >> 3;
    float ss = 0.f;
    for (int i = 0; i < nsteps; ++i) {
      const int st = i % S, slot = i % NAB;
      bool ok = mbar_wait_bounded(&fullb[st], (i / S) & 1, s_abort, p.err);
      if (ok && i >= NAB)
        ok = mbar_wait_bounded(&aempty[slot], ((i / NAB) - 1) & 1, s_abort, p.err);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.st below is warp-collective
      tc_fence_after();
      if (ok) {
        uint8_t *sb = smem + static_cast<size_t>(st) * p.stage_bytes;
        const int k0 = (tile0 + i) * TF8_TILE_K;
        if (NORM && xn_row < BN) {
          const int nx = (p.K - k0 > 64) ? 2 : 1;
          for (int h = 0; h < nx; ++h) {
            uint8_t *xt = sb + p.a8_bytes + h * p.xt_bytes;
            uint8_t *lt = xt + BN * 128;
            const int n = xn_row;
            const int lc = pc ^ (n & 7);        // 128-byte swizzle: logical chunk
            const int k = k0 + 64 * h + 8 * lc;
            const uint4 xv = *reinterpret_cast<const uint4 *>(xt + n * 128 + pc * 16);
            const uint4 gv = *reinterpret_cast<const uint4 *>(gs + k);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t hwd[4], lwd[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float x0 = bf16_lo(xw[u]), x1 = bf16_hi(xw[u]);
              ss = fmaf(x0, x0, ss);
              ss = fmaf(x1, x1, ss);
              const float p0 = x0 * bf16_lo(gw[u]), p1 = x1 * bf16_hi(gw[u]);  // exact
              const uint16_t h0 = f32_to_bf16_bits(p0), h1 = f32_to_bf16_bits(p1);
              const float r0 = p0 - __uint_as_float(static_cast<uint32_t>(h0) << 16);
              const float r1 = p1 - __uint_as_float(static_cast<uint32_t>(h1) << 16);
              hwd[u] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
              lwd[u] = static_cast<uint32_t>(f32_to_bf16_bits(r0)) |
                       (static_cast<uint32_t>(f32_to_bf16_bits(r1)) << 16);
            }
            *reinterpret_cast<uint4 *>(xt + n * 128 + pc * 16) =
                make_uint4(hwd[0], hwd[1], hwd[2], hwd[3]);
            *reinterpret_cast<uint4 *>(lt + n * 128 + pc * 16) =
                make_uint4(lwd[0], lwd[1], lwd[2], lwd[3]);
          }
          fence_proxy_async_smem();
        }
        // codes of this thread's row, logical 16-byte chunks 2 part, 2 part + 1
        // (stored at chunk c ^ (row & 7) by the swizzled copy), widened to
        // bf16 and written to A buffer `slot`, columns 16 part .. 16 part + 15
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const uint8_t *cr = sb + m * p.r8 * 128 + row * 128;
          uint32_t v[16];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (row < r)
              w = *reinterpret_cast<const uint4 *>(cr + (((2 * part + c) ^ (row & 7)) * 16));
            e4m3x4_to_bf16x2_alu(w.x, v[8 * c + 0], v[8 * c + 1]);
            e4m3x4_to_bf16x2_alu(w.y, v[8 * c + 2], v[8 * c + 3]);
            e4m3x4_to_bf16x2_alu(w.z, v[8 * c + 4], v[8 * c + 5]);
            e4m3x4_to_bf16x2_alu(w.w, v[8 * c + 6], v[8 * c + 7]);
          }
          tmem_st_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) +
                                 static_cast<uint32_t>(p.acol + (slot * NMAT + m) * 64 + 16 * part),
                             v);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&aready[slot]);
    }
    if (NORM) {
      // sum of squares of each token row: its 8 chunks sit in 8 adjacent lanes
      float v = ss;
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (xn_row < BN && pc == 0)
        s_rinv[xn_row] =
            (xn_row < p.B) ? 1.0f / sqrtf(v / static_cast<float>(p.K) + p.eps) : 0.f;
      named_barrier(1, TF8_XFORM);
    }

    // ---- epilogue (warps 2..5, one per TMEM lane quarter): TMEM -> registers
    // -> r_b, s[j] -> SiLU(gate) * up -> bf16 h (or a split-K partial sum)
    if (part == 0) {
      const bool okw = mbar_wait_bounded(accfull, 0, s_abort, p.err);
      tc_fence_after();
      const bool go = __all_sync(0xffffffffu, okw && !*s_abort);
      if (go) {
        const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16);
        const int j = j0 + row;
        float sg = 0.f, su = 0.f;
        if (p.kslices == 1 && row < r) {
          sg = __ldg(p.scale[0] + j);
          if (NMAT == 2) su = __ldg(p.scale[1] + j);
        }
        for (int c = 0; c < BN; c += 16) {
          float g[16], u[16];
          tmem_sum_banks(base + c, 1, WN, NORM ? BN : 0, g);
          if (NMAT == 2) tmem_sum_banks(base + WN + c, 1, WN, NORM ? BN : 0, u);
          if (p.kslices > 1) {
            float *mine = p.part + (static_cast<size_t>(slc) * p.nblocks + blk) * BN * 128;
#pragma unroll
            for (int e = 0; e < 16; ++e) mine[(c + e) * 128 + row] = g[e];
          } else if (row < r) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int n = c + e;
              if (n < p.B) {
                float res;
                if (NMAT == 2) {
                  const float sc = NORM ? s_rinv[n] : 1.0f;
                  const float a = (g[e] * sc) * sg, uu = (u[e] * sc) * su;
                  res = (a / (1.0f + expf(-a))) * uu;
                } else {
                  res = g[e] * sg;
                }
                if (DFK_IN_BOUNDS(j < p.N, 9, p.err))
                  p.out[static_cast<size_t>(n) * p.N + j] = f32_to_bf16_bits(res);
              }
            }
          }
        }
      }
      if (p.kslices > 1) {
        // every CTA of the row block takes part in the count (also after an
        // abort, so the counter stays consistent); the last one reduces
        __threadfence();
        named_barrier(2, 128);
        if (et == 0) {
          const unsigned old = atomicAdd(&p.counters[blk], 1u);
          *s_last = (old == static_cast<unsigned>(p.kslices - 1)) ? 1 : 0;
        }
        named_barrier(2, 128);
        if (*s_last) {
          __threadfence();
          if (row < r && !*s_abort) {
            const float sd = __ldg(p.scale[0] + j0 + row);
            splitk_reduce_row(p.part, p.kslices, p.nblocks, blk, BN, p.B, row,
                              [&](int n, float acc) {
                                if (DFK_IN_BOUNDS(n < p.B && j0 + row < p.N, 10, p.err))
                                p.out[static_cast<size_t>(n) * p.N + j0 + row] =
                                    f32_to_bf16_bits(acc * sd);
                              });
          }
          named_barrier(2, 128);
          if (et == 0) p.counters[blk] = 0u;
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    // every MMA has completed before TMEM is released (bounded wait)
    if (lane == 0) mbar_wait_bounded(accfull, 0, nullptr, p.err);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if (tid == 0 && *s_abort) {
    // after an aborted pipeline, wait (bounded) for copies still in flight
    const int issued = *s_issued;
    for (int st = 0; st < S; ++st) {
      int last = -1;
      for (int i = issued - 1; i >= 0 && i >= issued - S; --i)
        if (i % S == st) { last = i; break; }
      if (last >= 0) mbar_wait_bounded(&fullb[st], (last / S) & 1, nullptr, p.err);
    }
  }
}

}  // namespace dfk
