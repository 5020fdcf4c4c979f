// cc_engine.cuh -- CUDA-core weight-streaming GEMV engine for sm_100a.
//
// One kernel template covers
//   * the fused gate/up kernel (NMAT = 2): h = SiLU(xn . Wg^T) * (xn . Wu^T),
//     optionally with the RMSNorm prologue (NORM) -- "Deep Kernel Fusion for
//     Transformer Decoding", episode description (gate, up, SiLU and multiply
//     in one decode kernel) and GPULlama3.java PR #78 (`rms_ffn_gate_up`);
//   * a plain GEMV (NMAT = 1): out = x . W^T, used for the separate down
//     projection and for the unfused baseline.
//
// Data flow per CTA (one CTA per SM, persistent over its share of outputs):
//   - a producer warp streams weight tiles [rows x 64 k] of every matrix
//     through an S-stage shared-memory ring with TMA (cp.async.bulk.tensor),
//     each tile read from HBM exactly once for all B tokens and both
//     projections; mbarriers carry the full/empty hand-off;
//   - consumer warps hold the (normalised) activations in shared memory,
//     multiply-accumulate in fp32 registers, reduce across the 8 slots of a
//     tile row, apply SiLU(a)*u in registers and store h once as bf16.
//
// Canonical summation order (shared by every layout and every tile, thread
// and pipeline choice of the CUDA-core family, so that row-major,
// column-major and interleaved weights give bit-identical results):
//   k = 64 t + 8 s + e  (tile t, slot s in [0,8), element e in [0,8));
//   with KSPLIT teams, team c owns the tiles t with floor(t / nt) = c
//   (mod KSPLIT), nt = tiles per ring stage (KSPLIT = 1: one team, all tiles).
//   p[c][s] = fp32 chain from +0 over its tiles t ascending, then e
//             ascending:  p = fma(a[b][k], W[j][k], p);
//   q[c]    = ((p0 + p4) + (p2 + p6)) + ((p1 + p5) + (p3 + p7));
//   total   = left fold q[0] + q[1] + ... + q[KSPLIT-1].
// Without the RMSNorm a = x (bf16, every product exact in fp32).  With it
// a = x * gamma, the product of two bf16 values and so exact in fp32, and the
// epilogue multiplies total by r_b = 1 / sqrt(mean_k x[b][k]^2 + eps) (the
// sum of squares in the order of the standalone RMSNorm): RMSNorm(x) * W
// = r_b * sum_k (x gamma)[k] W[k], with r_b out of the dot product as in the
// tensor-core family, so the first FMA does not wait for the reduction.
// Either way the result is fixed by the order above.
//
// FP8 weights (W8, row-major only): W[j][k] = s[j] * Q[j][k] with Q in FP8
// E4M3 and one fp32 scale per output row (GPULlama3.java PR #78: dequantize
// inside the matrix-vector product instead of a separate pass).  A 128-byte
// tile row then holds 128 codes, so the order becomes k = 128 t + 16 s + e
// (e in [0, 16)); each code is converted to its exact fp32 value in
// registers, the chains are the same fp32 fmas, and the row scale multiplies
// the reduced sum once in the epilogue: out = s[j] * sum_k xn[k] Q[j][k].  Tokens never interact, so row b of the
// output is independent of the batch size.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"

namespace dfk {

constexpr int TILE_K = 64;          // reduction elements per tile row (128 bytes)
constexpr int NSLOT = 8;            // 16-byte slots per tile row
constexpr int CC_MAX_THREADS = 512; // consumers + one producer warp

enum : int { LAYOUT_ROW = 0, LAYOUT_COL = 1, LAYOUT_IL = 2 };

struct CcParams {
  const uint16_t *x;      // [B][K] bf16 activations
  const uint16_t *gamma;  // [K] bf16 RMSNorm weight (NORM only)
  uint16_t *out;          // [B][N] bf16
  uint16_t *outs[3];      // split output (packed QKV) when outs[0] != nullptr: rows
  int split[2];           // [0, split0) -> outs[0], [split0, split1) -> outs[1], rest -> outs[2]
  const float *scale[2];  // W8: per-output-row scales of each matrix [N] fp32
  unsigned *err;          // device error word
  int B, K, N;
  float eps;
  int nt;           // consecutive 64-wide tiles per team per ring stage (1, 2 or 4)
  int nsteps;       // ring steps per pass = ceil(ceil(K/TK) / (KSPLIT * nt)), TK = 64
                    // reduction elements per tile (128 with FP8 weights)
  int kpad;         // nsteps * KSPLIT * nt * TK: activation row pitch in shared memory
  int granule;      // output rows per partition unit
  int ubase, uextra;// units per CTA: ubase, +1 for the first uextra CTAs
  int r_hi;         // largest row count of any CTA (shared-memory slot size)
  int stages;       // ring depth
  int stage_bytes;  // KSPLIT * NMAT * r_hi * 128 * nt
  int npass;        // ceil(B / BT)
  int tpt;          // consumer threads per K team (multiple of 32)
  int xs_off;       // shared-memory offset of the activation / reduction area
  int g_off;        // (unused)
  int bar_off;      // shared-memory offset of the barrier area
  int pf_steps;     // ring steps after the first fill whose weight boxes are prefetched into L2
};

// Tensor maps: index matrix * 2 + (CTA has the short row count ? 1 : 0).
struct CcMaps {
  CUtensorMap m[4];
};

template <int NMAT, int JPT, int BT>
struct CcAcc {
  float v[NMAT][JPT][BT];
};

// PAIR: issue the FMAs two at a time with fma.rn.f32x2 -- the gate and up
// accumulators of one row (NMAT = 2) or two adjacent rows (NMAT = 1) share a
// packed register, the activation is broadcast into both lanes.  Each lane
// performs the same fma sequence as the scalar path: results are identical.
template <int LAYOUT, int NMAT, int JPT, int BT, int KSPLIT, bool XF32, bool NORM, bool PAIR,
          bool W8 = false>
__global__ void __launch_bounds__(CC_MAX_THREADS, 1)
    cc_gemv_kernel(const __grid_constant__ CcMaps maps, const CcParams p) {
  static_assert(LAYOUT != LAYOUT_IL || NMAT == 2, "interleaved layout holds both matrices");
  static_assert(!W8 || LAYOUT == LAYOUT_ROW, "FP8 weights are row-major");
  constexpr int TK = W8 ? 2 * TILE_K : TILE_K;  // reduction elements per 128-byte tile row
  static_assert(XF32 || !NORM, "normalised activations are kept in fp32");
  constexpr int NPAIR = PAIR ? (NMAT == 2 ? JPT : JPT / 2) : 1;
  static_assert(JPT == 2 || JPT == 4, "JPT");
  extern __shared__ __align__(1024) uint8_t smem[];

  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int ncons = nthr - 32 - (NORM ? 32 : 0);  // consumer threads (then [norm warp], producer)
  const int warp = tid >> 5, lane = tid & 31;
  const int S = p.stages;

  uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = full + S;
  volatile int *s_abort = reinterpret_cast<volatile int *>(empty + S);
  int *s_issued = reinterpret_cast<int *>(empty + S) + 1;
  float *s_rinv = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(empty + S) + 16);

  // ---- this CTA's contiguous share of output rows [j0, j0 + r)
  const int cta = blockIdx.x;
  const int u0 = cta * p.ubase + min(cta, p.uextra);
  const int nu = p.ubase + (cta < p.uextra ? 1 : 0);
  const int j0 = u0 * p.granule;
  const int r = nu * p.granule;
  const int mi = (r == p.r_hi) ? 0 : 1;
  const int nt = p.nt;
  const uint32_t slot_bytes = static_cast<uint32_t>(p.r_hi) * TILE_K * 2 * nt;
  const int rowb = TILE_K * 2 * nt;  // bytes per row of a row-major / interleaved tile

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncons / 32);
    }
    *s_abort = 0;
    *s_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  const int total_steps = p.npass * p.nsteps;

  if (warp == (nthr >> 5) - 1) {
    // ================= producer warp: one lane issues all TMA traffic
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      const uint32_t tile_bytes = static_cast<uint32_t>(r) * TILE_K * 2 * nt;
      const uint32_t tx = tile_bytes * NMAT * KSPLIT;
      int issued = 0;
      for (int i = 0; i < total_steps; ++i) {
        const int st = i % S;
        if (i >= S && !mbar_wait_bounded(&empty[st], ((i / S) - 1) & 1, s_abort, p.err)) break;
        const int step = i % p.nsteps;
        uint8_t *base = smem + static_cast<size_t>(st) * p.stage_bytes;
        mbar_arrive_expect_tx(&full[st], tx);
#pragma unroll
        for (int kt = 0; kt < KSPLIT; ++kt) {
          const int k0 = (step * KSPLIT + kt) * nt * TK;
          uint8_t *tb = base + static_cast<size_t>(kt) * NMAT * slot_bytes;
          if (LAYOUT == LAYOUT_ROW) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              tma_load_2d(tb + m * slot_bytes, &maps.m[m * 2 + mi], &full[st], k0, j0, pol);
          } else if (LAYOUT == LAYOUT_COL) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              tma_load_2d(tb + m * slot_bytes, &maps.m[m * 2 + mi], &full[st], j0, k0, pol);
          } else {
            // interleaved rows [2 j0, 2 j0 + 2r) as two boxes of r rows
            tma_load_2d(tb, &maps.m[mi], &full[st], k0, 2 * j0, pol);
            tma_load_2d(tb + tile_bytes, &maps.m[mi], &full[st], k0, 2 * j0 + r, pol);
          }
        }
        issued = i + 1;
        if (i == S - 1) {
          // ring full: pull the next pf_steps steps' boxes into L2 while the
          // consumers wait for the previous kernel's activations
          const int pf_end = min(total_steps, S + p.pf_steps);
          for (int ii = S; ii < pf_end; ++ii) {
            const int pstep = ii % p.nsteps;
#pragma unroll
            for (int kt = 0; kt < KSPLIT; ++kt) {
              const int k0 = (pstep * KSPLIT + kt) * nt * TK;
              if (LAYOUT == LAYOUT_ROW) {
#pragma unroll
                for (int m = 0; m < NMAT; ++m) tma_prefetch_2d(&maps.m[m * 2 + mi], k0, j0);
              } else if (LAYOUT == LAYOUT_COL) {
#pragma unroll
                for (int m = 0; m < NMAT; ++m) tma_prefetch_2d(&maps.m[m * 2 + mi], j0, k0);
              } else {
                tma_prefetch_2d(&maps.m[mi], k0, 2 * j0);
                tma_prefetch_2d(&maps.m[mi], k0, 2 * j0 + r);
              }
            }
          }
        }
      }
      *s_issued = issued;
    }
  } else if (NORM && warp == (nthr >> 5) - 2) {
    // ================= norm warp: r_b = 1 / sqrt(mean(x^2) + eps) of each token
    // of each pass, beside the consumers (r_b multiplies the row sums in the
    // epilogue, so no FMA waits for it).  Fixed order: lane l chains k = 8 l + e
    // + 256 c (c, then e ascending), then a xor butterfly over the 32 lanes (the
    // order of the standalone RMSNorm).  x comes from global memory (L2), eight
    // chunks a lane in flight; s_rinv alternates between two halves by pass.
    pdl_wait();  // x comes from the previous kernel in the stream
    for (int pass = 0; pass < p.npass; ++pass) {
      const int b0 = pass * BT;
      for (int bb = 0; bb < BT; ++bb) {
        float ss = 0.f;
        const bool real = b0 + bb < p.B;
        const uint16_t *xr = p.x + static_cast<size_t>(real ? b0 + bb : 0) * p.K;
        for (int k0 = 8 * lane; real && k0 < p.K; k0 += 8 * 256) {
          uint4 xv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int k = k0 + 256 * c;
            xv[c] = (k < p.K && DFK_IN_BOUNDS(k + 8 <= p.K, 3, p.err))
                        ? ld_nc_v4(xr + k) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (k0 + 256 * c >= p.K) break;
            const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float e0 = bf16_lo(w4[h]), e1 = bf16_hi(w4[h]);
              ss = fmaf(e0, e0, ss);
              ss = fmaf(e1, e1, ss);
            }
          }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        if (lane == 0)
          s_rinv[(pass & 1) * BT + bb] =
              real ? 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps) : 0.f;
      }
      named_barrier(2, ncons + 32);  // the consumers read this pass's r_b after it
    }
  } else {
    // ================= consumer warps
    const int team = tid / p.tpt;
    const int lt = tid - team * p.tpt;
    int s, q;
    if (LAYOUT == LAYOUT_COL) {
      s = (lt >> 5) & 7;                  // a warp shares one slot
      q = (lt >> 8) * 32 + (lt & 31);     // lanes walk consecutive column groups
    } else {
      s = lt & 7;                         // 8 lanes cover one 128-byte tile row
      q = lt >> 3;
    }
    const int jl0 = q * JPT;              // first local output row of this thread
    const bool active = jl0 < r;
    const int cw = tid >> 5, ncw = ncons >> 5;

    float *xs_f = reinterpret_cast<float *>(smem + p.xs_off);
    uint16_t *xs_h = reinterpret_cast<uint16_t *>(smem + p.xs_off);
    float *red = reinterpret_cast<float *>(smem + p.xs_off);  // reused after the K loop

    pdl_wait();  // activations come from the previous kernel in the stream

    for (int pass = 0; pass < p.npass; ++pass) {
      const int b0 = pass * BT;

      // ---- prologue: the activations into shared memory -- x, or with the
      // RMSNorm xg = x * gamma (the product of two bf16 values, exact in fp32;
      // r_b multiplies the row sums in the epilogue).  Every consumer thread
      // issues its 16-byte loads back to back, so the prologue costs one L2
      // round trip; x is read only after pdl_wait().
      {
        const int c8n = p.kpad >> 3;  // 8-element chunks per activation row
        const int nx = BT * c8n;      // activation chunks
        // chunks a thread has in flight: 8 without the RMSNorm (one round trip
        // for the 1792 chunks of a 14336-long row), 4 with it (x and gamma)
        constexpr int PB = NORM ? 4 : 8;
        for (int base = tid; base < nx; base += PB * ncons) {
          uint4 v[PB], g[PB];
#pragma unroll
          for (int u = 0; u < PB; ++u) {
            const int idx = base + u * ncons;
            v[u] = g[u] = make_uint4(0u, 0u, 0u, 0u);
            if (idx < nx) {
              const int bb = idx / c8n, k = (idx - bb * c8n) * 8;
              if (b0 + bb < p.B && k < p.K)
                if (DFK_IN_BOUNDS(b0 + bb < p.B && k + 8 <= p.K, 2, p.err)) {
                  v[u] = ld_nc_v4(p.x + static_cast<size_t>(b0 + bb) * p.K + k);
                  if (NORM) g[u] = ld_nc_v4(p.gamma + k);
                }
            }
          }
#pragma unroll
          for (int u = 0; u < PB; ++u) {
            const int idx = base + u * ncons;
            if (idx >= nx) continue;
            const int bb = idx / c8n, k = (idx - bb * c8n) * 8;
            if (XF32) {
              // within a 64-wide tile, element 8s + 4h + i sits at 32h + 4s + i
              float *row = xs_f + static_cast<size_t>(bb) * p.kpad + (k & ~63);
              const int s8 = (k >> 3) & 7;
              float4 lo = make_float4(bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y),
                                      bf16_hi(v[u].y));
              float4 hi = make_float4(bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w),
                                      bf16_hi(v[u].w));
              if (NORM) {
                lo.x *= bf16_lo(g[u].x); lo.y *= bf16_hi(g[u].x);
                lo.z *= bf16_lo(g[u].y); lo.w *= bf16_hi(g[u].y);
                hi.x *= bf16_lo(g[u].z); hi.y *= bf16_hi(g[u].z);
                hi.z *= bf16_lo(g[u].w); hi.w *= bf16_hi(g[u].w);
              }
              *reinterpret_cast<float4 *>(row + 4 * s8) = lo;
              *reinterpret_cast<float4 *>(row + 32 + 4 * s8) = hi;
            } else {
              *reinterpret_cast<uint4 *>(xs_h + static_cast<size_t>(bb) * p.kpad + k) = v[u];
            }
          }
        }
        named_barrier(1, ncons);
      }

      // ---- main loop over the weight stream
      CcAcc<NMAT, JPT, BT> acc;
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int jj = 0; jj < JPT; ++jj)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) acc.v[m][jj][bb] = 0.f;
      uint64_t acc2[NPAIR][BT];  // PAIR only: packed accumulators, +0 in both lanes
#pragma unroll
      for (int pr = 0; pr < NPAIR; ++pr)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) acc2[pr][bb] = 0ull;

      for (int step = 0; step < p.nsteps; ++step) {
        const int i = pass * p.nsteps + step;
        const int st = i % S;
        const bool ok = mbar_wait_bounded(&full[st], (i / S) & 1, s_abort, p.err);
        for (int tt = 0; ok && active && tt < nt; ++tt) {
          const int t = (step * KSPLIT + team) * nt + tt;
          const uint8_t *tb = smem + static_cast<size_t>(st) * p.stage_bytes +
                              static_cast<size_t>(team) * NMAT * slot_bytes;
          if constexpr (W8) {
            // slot s of 128-wide tile t: k = 128 t + 16 s + e, taken as two halves
            // of 8 (e ascending); 16 codes per row per thread
            uint32_t wq[NMAT][JPT][4];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
              for (int jj = 0; jj < JPT; ++jj) {
                const uint4 v = *reinterpret_cast<const uint4 *>(
                    tb + m * slot_bytes + (jl0 + jj) * rowb + tt * (TILE_K * 2) + s * 16);
                wq[m][jj][0] = v.x; wq[m][jj][1] = v.y; wq[m][jj][2] = v.z; wq[m][jj][3] = v.w;
              }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              float xv[BT][8];
#pragma unroll
              for (int bb = 0; bb < BT; ++bb) {
                if (XF32) {
                  // 64-wide tile 2 t + s / 4, 8-element chunk (2 s + hf) mod 8
                  const int c = (2 * s + hf) & 7;
                  const float *row =
                      xs_f + static_cast<size_t>(bb) * p.kpad + (2 * t + (s >> 2)) * TILE_K;
                  const float4 lo = *reinterpret_cast<const float4 *>(row + 4 * c);
                  const float4 hi = *reinterpret_cast<const float4 *>(row + 32 + 4 * c);
                  xv[bb][0] = lo.x; xv[bb][1] = lo.y; xv[bb][2] = lo.z; xv[bb][3] = lo.w;
                  xv[bb][4] = hi.x; xv[bb][5] = hi.y; xv[bb][6] = hi.z; xv[bb][7] = hi.w;
                } else {
                  const uint4 v = *reinterpret_cast<const uint4 *>(
                      xs_h + static_cast<size_t>(bb) * p.kpad + t * TK + 16 * s + 8 * hf);
                  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                  for (int ii = 0; ii < 4; ++ii) {
                    xv[bb][2 * ii] = bf16_lo(w[ii]);
                    xv[bb][2 * ii + 1] = bf16_hi(w[ii]);
                  }
                }
              }
#pragma unroll
              for (int wi = 0; wi < 2; ++wi) {  // code word 2 hf + wi: elements 4 wi .. 4 wi + 3
                float wf[NMAT][JPT][4];
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                  for (int jj = 0; jj < JPT; ++jj) e4m3x4_to_f32(wq[m][jj][2 * hf + wi], wf[m][jj]);
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                  const int e = 4 * wi + e4;
                  if constexpr (PAIR) {
                    uint64_t xd[BT];
#pragma unroll
                    for (int bb = 0; bb < BT; ++bb) xd[bb] = pack_f32x2(xv[bb][e], xv[bb][e]);
#pragma unroll
                    for (int pr = 0; pr < NPAIR; ++pr) {
                      const int m1 = NMAT - 1, j0r = (NMAT == 2) ? pr : 2 * pr;
                      const int j1r = (NMAT == 2) ? pr : 2 * pr + 1;
                      const uint64_t wp = pack_f32x2(wf[0][j0r][e4], wf[m1][j1r][e4]);
#pragma unroll
                      for (int bb = 0; bb < BT; ++bb)
                        acc2[pr][bb] = fma_f32x2(xd[bb], wp, acc2[pr][bb]);
                    }
                  } else {
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                      for (int jj = 0; jj < JPT; ++jj)
#pragma unroll
                        for (int bb = 0; bb < BT; ++bb)
                          acc.v[m][jj][bb] = fmaf(xv[bb][e], wf[m][jj][e4], acc.v[m][jj][bb]);
                  }
                }
              }
            }
            continue;
          }
          float xv[BT][8];
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            if (XF32) {
              const float *row = xs_f + static_cast<size_t>(bb) * p.kpad + t * TILE_K;
              const float4 lo = *reinterpret_cast<const float4 *>(row + 4 * s);
              const float4 hi = *reinterpret_cast<const float4 *>(row + 32 + 4 * s);
              xv[bb][0] = lo.x; xv[bb][1] = lo.y; xv[bb][2] = lo.z; xv[bb][3] = lo.w;
              xv[bb][4] = hi.x; xv[bb][5] = hi.y; xv[bb][6] = hi.z; xv[bb][7] = hi.w;
            } else {
              const uint4 v = *reinterpret_cast<const uint4 *>(
                  xs_h + static_cast<size_t>(bb) * p.kpad + t * TILE_K + 8 * s);
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int ii = 0; ii < 4; ++ii) {
                xv[bb][2 * ii] = bf16_lo(w[ii]);
                xv[bb][2 * ii + 1] = bf16_hi(w[ii]);
              }
            }
          }
          if (LAYOUT != LAYOUT_COL) {
            // thread reads 8 consecutive k of each of its rows (one 16-byte slot)
            uint32_t wv[NMAT][JPT][4];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
              for (int jj = 0; jj < JPT; ++jj) {
                const int row = (LAYOUT == LAYOUT_IL) ? 2 * (jl0 + jj) + m : jl0 + jj;
                const uint8_t *bse = (LAYOUT == LAYOUT_IL) ? tb : tb + m * slot_bytes;
                const uint4 v =
                    *reinterpret_cast<const uint4 *>(bse + row * rowb + tt * (TILE_K * 2) + s * 16);
                wv[m][jj][0] = v.x; wv[m][jj][1] = v.y; wv[m][jj][2] = v.z; wv[m][jj][3] = v.w;
              }
            if constexpr (PAIR) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                uint64_t xd[BT];
#pragma unroll
                for (int bb = 0; bb < BT; ++bb) xd[bb] = pack_f32x2(xv[bb][e], xv[bb][e]);
#pragma unroll
                for (int pr = 0; pr < NPAIR; ++pr) {
                  // NMAT = 2: (gate, up) of row pr; NMAT = 1: rows (2 pr, 2 pr + 1)
                  const int m1 = NMAT - 1, j0r = (NMAT == 2) ? pr : 2 * pr;
                  const int j1r = (NMAT == 2) ? pr : 2 * pr + 1;
                  const uint32_t w0 = wv[0][j0r][e >> 1], w1 = wv[m1][j1r][e >> 1];
                  const uint64_t wp = (e & 1) ? pack_f32x2(bf16_hi(w0), bf16_hi(w1))
                                              : pack_f32x2(bf16_lo(w0), bf16_lo(w1));
#pragma unroll
                  for (int bb = 0; bb < BT; ++bb)
                    acc2[pr][bb] = fma_f32x2(xd[bb], wp, acc2[pr][bb]);
                }
              }
            } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
              for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int jj = 0; jj < JPT; ++jj) {
                  const uint32_t w = wv[m][jj][e >> 1];
                  const float wf = (e & 1) ? bf16_hi(w) : bf16_lo(w);
#pragma unroll
                  for (int bb = 0; bb < BT; ++bb)
                    acc.v[m][jj][bb] = fmaf(xv[bb][e], wf, acc.v[m][jj][bb]);
                }
            }
          } else {
            // column-major tile [64 k][r j]: thread reads JPT consecutive j per k row
            const int pitch = r * 2;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int krow = tt * TILE_K + 8 * s + e;
              uint32_t w[NMAT][JPT / 2];
#pragma unroll
              for (int m = 0; m < NMAT; ++m) {
                const uint8_t *src = tb + m * slot_bytes + krow * pitch + jl0 * 2;
                if constexpr (JPT == 4) {
                  const uint2 v = *reinterpret_cast<const uint2 *>(src);
                  w[m][0] = v.x;
                  w[m][1] = v.y;
                } else {
                  w[m][0] = *reinterpret_cast<const uint32_t *>(src);
                }
              }
              if constexpr (PAIR) {
                uint64_t xd[BT];
#pragma unroll
                for (int bb = 0; bb < BT; ++bb) xd[bb] = pack_f32x2(xv[bb][e], xv[bb][e]);
#pragma unroll
                for (int pr = 0; pr < NPAIR; ++pr) {
                  const int m1 = NMAT - 1, j0r = (NMAT == 2) ? pr : 2 * pr;
                  const int j1r = (NMAT == 2) ? pr : 2 * pr + 1;
                  const float f0 = (j0r & 1) ? bf16_hi(w[0][j0r >> 1]) : bf16_lo(w[0][j0r >> 1]);
                  const float f1 = (j1r & 1) ? bf16_hi(w[m1][j1r >> 1]) : bf16_lo(w[m1][j1r >> 1]);
                  const uint64_t wp = pack_f32x2(f0, f1);
#pragma unroll
                  for (int bb = 0; bb < BT; ++bb)
                    acc2[pr][bb] = fma_f32x2(xd[bb], wp, acc2[pr][bb]);
                }
              } else {
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                  for (int jj = 0; jj < JPT; ++jj) {
                    const float wf =
                        (jj & 1) ? bf16_hi(w[m][jj >> 1]) : bf16_lo(w[m][jj >> 1]);
#pragma unroll
                    for (int bb = 0; bb < BT; ++bb)
                      acc.v[m][jj][bb] = fmaf(xv[bb][e], wf, acc.v[m][jj][bb]);
                  }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }

      if constexpr (PAIR) {
#pragma unroll
        for (int pr = 0; pr < NPAIR; ++pr)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            if constexpr (NMAT == 2)
              unpack_f32x2(acc2[pr][bb], acc.v[0][pr][bb], acc.v[NMAT - 1][pr][bb]);
            else
              unpack_f32x2(acc2[pr][bb], acc.v[0][2 * pr][bb], acc.v[0][2 * pr + 1][bb]);
          }
      }

      // ---- reduce over the 8 slots, fold the K teams, SwiGLU epilogue
      if (LAYOUT != LAYOUT_COL) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
          for (int jj = 0; jj < JPT; ++jj)
#pragma unroll
            for (int bb = 0; bb < BT; ++bb) {
              float v = acc.v[m][jj][bb];
              v += __shfl_xor_sync(0xffffffffu, v, 4);
              v += __shfl_xor_sync(0xffffffffu, v, 2);
              v += __shfl_xor_sync(0xffffffffu, v, 1);
              acc.v[m][jj][bb] = v;
            }
      }
      if (NORM) named_barrier(2, ncons + 32);  // this pass's r_b from the norm warp
      named_barrier(1, ncons);  // activation reads done: `red` aliases them
      const int rh = p.r_hi;
      if (active) {
        if (LAYOUT != LAYOUT_COL) {
          if (s == 0) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
              for (int jj = 0; jj < JPT; ++jj)
#pragma unroll
                for (int bb = 0; bb < BT; ++bb)
                  red[((team * NMAT + m) * BT + bb) * rh + jl0 + jj] = acc.v[m][jj][bb];
          }
        } else {
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int jj = 0; jj < JPT; ++jj)
#pragma unroll
              for (int bb = 0; bb < BT; ++bb)
                red[(((team * NSLOT + s) * NMAT + m) * BT + bb) * rh + jl0 + jj] =
                    acc.v[m][jj][bb];
        }
      }
      named_barrier(1, ncons);
      const bool aborted = *s_abort != 0;
      for (int o = tid; o < BT * r; o += ncons) {
        const int bb = o / r;
        const int jl = o - bb * r;
        const int b = b0 + bb, j = j0 + jl;
        float v[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          float tot = 0.f;
#pragma unroll
          for (int kt = 0; kt < KSPLIT; ++kt) {
            float tk;
            if (LAYOUT == LAYOUT_COL) {
              const float *pp = red + ((kt * NSLOT * NMAT + m) * BT + bb) * rh + jl;
              const int ss = NMAT * BT * rh;  // slot stride
              tk = ((pp[0] + pp[4 * ss]) + (pp[2 * ss] + pp[6 * ss])) +
                   ((pp[1 * ss] + pp[5 * ss]) + (pp[3 * ss] + pp[7 * ss]));
            } else {
              tk = red[((kt * NMAT + m) * BT + bb) * rh + jl];
            }
            tot = (kt == 0) ? tk : tot + tk;
          }
          v[m] = tot;
        }
        if (!aborted && b < p.B && j < p.N) {
          if constexpr (NORM) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) v[m] *= s_rinv[(pass & 1) * BT + bb];
          }
          if constexpr (W8) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) v[m] *= __ldg(p.scale[m] + j);
          }
          float res;
          if (NMAT == 2) {
            const float a = v[0];
            res = (a / (1.0f + expf(-a))) * v[NMAT - 1];
          } else {
            res = v[0];
          }
          store_out(p, b, j, f32_to_bf16_bits(res));
        }
      }
      named_barrier(1, ncons);  // `red` / activations are rewritten by the next pass
    }
  }

  __syncthreads();
  // After an aborted pipeline, wait (bounded) for this CTA's copies still in
  // flight before shared memory is released.
  if (tid == nthr - 32 && *s_abort) {
    const int issued = *s_issued;
    for (int st = 0; st < S; ++st) {
      int last = -1;
      for (int i = issued - 1; i >= 0 && i >= issued - S; --i)
        if (i % S == st) { last = i; break; }
      if (last >= 0) mbar_wait_bounded(&full[st], (last / S) & 1, nullptr, p.err);
    }
  }
}

}  // namespace dfk
