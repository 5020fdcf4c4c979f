// tc_engine.cuh -- tensor-core (tcgen05 / TMEM) weight-streaming kernel for
// the decode MLP at larger decode batches (8 <= B <= 64), where fp32 FMA on
// CUDA cores can no longer keep up with HBM.
//
// Same operation as the CUDA-core engine ("Deep Kernel Fusion for
// Transformer Decoding", episode description: gate projection, up
// projection, SiLU and elementwise multiply in one decode kernel; the down
// projection is the NMAT = 1 instance), formulated for the MMA with the
// weight rows on M and the tokens on N:
//     D_gate[j][n] = sum_k Wg[j][k] * X[n][k],  D_up likewise,
// accumulated in fp32 in TMEM, then h[n][j] = SiLU(D_gate) * D_up.
//
// Work split: one CTA per SM owns a contiguous range of r ~ F / #SMs output
// rows over the whole reduction (no split-K, no scratch memory); the range
// is cut into MT sub-tiles of at most 128 rows, each one M = 128 MMA tile.
// Rows of a sub-tile beyond its height come from neighbouring shared memory
// and produce ignored accumulator rows (the MMA reads 128 rows; only the
// loaded ones are stored).
//
// RMSNorm prologue (NORM): r_b = 1/sqrt(mean_k x[b][k]^2 + eps) is a
// per-token scalar, so it factors out of the dot product:
//     a[b][j] = r_b * sum_k (x[b][k] * gamma[k]) * Wg[j][k].
// Four warps turn each streamed x tile into x*gamma, split exactly into two
// bf16 halves (hi = bf16(x*gamma), lo = bf16(x*gamma - hi); the product of
// two bf16 values has at most 16 significant bits, so hi + lo is exact),
// accumulate sum_k x^2 on the way, and scale by r_b in the epilogue.  The hi
// and lo rows sit side by side on N (one MMA of N = 2 * bn reads each weight
// tile once); the epilogue adds the two column halves.  NORM = 1 does this
// transform inside the kernel; NORM = 2 reads tiles that a prep kernel (a
// CTA per token, launched just before) wrote in the same
// layout, with r_b, so the kernel streams them like plain activations (the
// in-kernel transform serialises with the MMAs and costs a third of the time
// at 64 tokens; the host uses NORM = 2 above 32 tokens).
//
// Warp roles (192 threads): warp 0 issues TMA copies into an S-stage ring;
// warp 1 owns TMEM and issues the MMAs (one elected lane) with tcgen05.commit
// releasing ring stages; warps 2-5 run the x*gamma transform (NORM) and the
// epilogue (tcgen05.ld -> SiLU * up -> one bf16 store per output).
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "tc_ptx.cuh"

namespace dfk {

constexpr int TC_THREADS = 192;
constexpr int TC_TILE_K = 64;       // reduction elements per k-tile (one 128-byte swizzle row)
constexpr int TC_ATOM = 1024;       // bytes of an 8-row swizzle atom
constexpr int TP_MAX = 8;           // ranks of a tensor-parallel group

struct TcParams {
  uint16_t *out;          // [B][N] bf16
  uint16_t *outs[3];      // split output (packed QKV) when outs[0] != nullptr
  int split[2];           // row ranges of the q / k / v parts
  const uint16_t *gamma;  // [K] bf16 (NORM = 1)
  const float *rinv;      // [bn] r_b from the prep kernel (NORM = 2)
  unsigned *err;          // device error word
  int B, K, N;
  float eps;
  int nsteps;             // ring steps = ceil(K / (64 * nt))
  int nt;                 // k-tiles per ring stage
  int rbase, rextra;      // rows per CTA: rbase, +1 for the first rextra CTAs
  int hmax;               // height of the taller sub-tile box (map 0); map 1 is hmax - 1
  int rc;                 // rows reserved per A tile in shared memory (multiple of 8)
  int bn;                 // tokens on N: 16, 32 or 64
  int stages, stage_bytes;
  int a_bytes;            // A-tile bytes of one stage
  int xt_bytes;           // bytes of one k-tile's activation rows (bn * 128, x2 with NORM)
  int tmem_cols;
  int nbank;              // independent TMEM accumulators per output (1, 2 or 4)
  int g_off, bar_off;     // shared-memory offsets from the 1024-byte aligned base
  // split-K (single-matrix GEMV only): CTA c handles row block c / kslices and
  // reduction slice c % kslices; partial sums go to `part`, the last CTA to
  // arrive on a row block (counter) adds the slices in order 0, 1, ... and
  // stores the output, then resets the counter to 0.
  int ntiles;             // 64-wide k-tiles covering K
  int kslices;            // 1 = no split
  float *part;            // [kslices][row blocks][bn][128] fp32
  unsigned *counters;     // [row blocks], 0 between calls
  int nblocks;            // row blocks (split-K)
  int full;               // 1: every CTA owns 128 rows (the last one fewer); boxes of 128 rows
  int pf_steps;           // ring steps after the first fill whose weight boxes are prefetched
                          // into L2 before the wait on the previous kernel
  // Tensor-parallel down projection with the all-reduce fused in (GEMV,
  // no split-K; tp_world = 0: off).  The reduction dimension is sharded over
  // tp_world ranks; this grid computes the shards of ranks tp_rank0 ..
  // tp_rank0 + (grid / tp_blocks) - 1 (one rank on a multi-GPU run; all of
  // them when the ranks are emulated on one device), tp_blocks row blocks
  // each.  Rank r's weights are rows r * N .. of the weight map and its
  // activations rows r * B .. of the activation map.  Each CTA writes its
  // fp32 partial rows into every rank's receive buffer, raises its flag
  // there, waits (bounded) for every rank's flag of its row block, adds the
  // ranks' partials in rank order and stores bf16 y of its own rank.
  int tp_world;
  int tp_rank0;
  int tp_blocks;
  float *tp_recv[TP_MAX];               // per rank: [2][tp_world][tp_bmax][N] fp32
  unsigned long long *tp_flags[TP_MAX]; // per rank: [row blocks][tp_world]
  unsigned long long *tp_seq;           // this grid's call counter (calls completed)
  unsigned *tp_exit;                    // CTAs of this grid that finished (0 between calls)
  int tp_bmax;                          // token capacity of the receive buffers
};

// wg/wu: [0] box height hmax, [1] box height hmax - 1; x: activations box {64, bn}.
// Interleaved weights use wg for both matrices (3-D map {k, gate|up, row}).
struct TcMaps {
  CUtensorMap wg[2];
  CUtensorMap wu[2];
  CUtensorMap x;
};

// Loads 16 columns of `nb` accumulator banks (bank stride `bank_cols`
// columns) for this warp's 32 TMEM lanes and adds them in a fixed order; with
// lo_off > 0 each bank also holds a second column block lo_off columns
// further (the lo products), added to its first block before the banks are
// combined: v = ((b0.hi + b0.lo) + (b1.hi + b1.lo)) + ...
__device__ __forceinline__ void tmem_sum_banks(uint32_t taddr, int nb, int bank_cols, int lo_off,
                                               float (&v)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = 0.f;
  float part[4][16];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    if (b < nb) {  // nb is warp-uniform: the loads stay converged
      float hi[16];
      tmem_ld_32x32b_x16(taddr + b * bank_cols, hi);
      if (lo_off > 0) {
        float lo[16];
        tmem_ld_32x32b_x16(taddr + b * bank_cols + lo_off, lo);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) part[b][e] = hi[e] + lo[e];
      } else {
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) part[b][e] = hi[e];
      }
    }
  }
  if (nb == 1) {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = part[0][e];
  } else if (nb == 2) {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = part[0][e] + part[1][e];
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = (part[0][e] + part[1][e]) + (part[2][e] + part[3][e]);
  }
}

// WL (weight layout): 0 row-major [N][K] (K-major A), 1 column-major [K][N]
// (MN-major A; each CTA owns 128 columns, loaded as two 64-column boxes),
// 2 interleaved [N][2][K].
// NORM: 0 none, 1 x * gamma transform in the kernel, 2 prepared tiles.
template <int NMAT, int NORM, int WL, int MT>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_gemv_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  constexpr bool IL = WL == 2, COLM = WL == 1;
  static_assert(NMAT == 1 || NMAT == 2, "NMAT");
  static_assert(!IL || NMAT == 2, "interleaved layout holds both matrices");
  static_assert(!COLM || MT == 1, "column-major: one 128-column tile per CTA");
  static_assert(NORM >= 0 && NORM <= 2, "NORM");
  constexpr int XROWS = NORM == 2 ? 2 : 1;  // activation rows per token loaded by TMA
  static_assert(MT == 1 || MT == 2, "MT");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (the host reserves the slack)
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.stages, NT = p.nt, BN = p.bn;

  uint64_t *fullb = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = fullb + S;
  uint64_t *xready = empty + S;
  uint64_t *xfull = xready + S;  // NORM = 1: a stage's activation tiles have landed
  uint64_t *accfull = xfull + S;
  volatile int *s_abort = reinterpret_cast<volatile int *>(accfull + 1);
  int *s_issued = reinterpret_cast<int *>(accfull + 1) + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(accfull + 1) + 2;
  volatile int *s_last = reinterpret_cast<volatile int *>(accfull + 1) + 3;
  float *s_rinv = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(accfull + 1) + 16);
  uint16_t *gs = reinterpret_cast<uint16_t *>(smem + p.g_off);

  // ---- this CTA's rows [j0, j0 + r), cut into MT sub-tiles, and its
  // reduction range: k-tiles [tile0, tile1)
  const int cta = blockIdx.x;
  int blk = cta / p.kslices;
  const int slc = cta - blk * p.kslices;
  // tensor-parallel: this CTA computes rank tp_rank0 + tpl's shard; its rows
  // and activations sit at these offsets of the (stacked) maps
  const int tpl = (NMAT == 1 && p.tp_world) ? blk / p.tp_blocks : 0;
  blk -= tpl * p.tp_blocks;
  const int wrow = tpl * p.N, xrow = tpl * p.B;
  const int j0 = blk * p.rbase + min(blk, p.rextra);
  const bool full = COLM || p.full;  // 128-row boxes, zero-filled past the last row
  const int r = full ? min(p.rbase, p.N - j0) : p.rbase + (blk < p.rextra ? 1 : 0);
  const int tile0 = (slc * p.ntiles) / p.kslices;
  const int tile1 = ((slc + 1) * p.ntiles) / p.kslices;
  const int nsteps = (tile1 - tile0 + NT - 1) / NT;
  int h[MT], rs[MT];
  h[0] = (r + MT - 1) / MT;
  rs[0] = 0;
  if constexpr (MT == 2) {
    h[1] = r - h[0];
    rs[1] = h[0];
  }

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullb[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&xready[s], 128);
      mbar_init(&xfull[s], 1);
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
        const int nv = min(NT, tile1 - (tile0 + i * NT));  // k-tiles of this step in range
        // (column-major boxes are always 64 x 64, zero-filled past the last column)
        const uint32_t wbytes = static_cast<uint32_t>(nv) * NMAT * (full ? 128 : r) * 128u;
        const uint32_t xbytes = static_cast<uint32_t>(nv) * XROWS * BN * 128u;
        // with the in-kernel transform the activation tiles have a barrier of
        // their own: they come from L2 and land long before the weights, so
        // the transform is done by the time the weights arrive
        if (NORM == 1) {
          mbar_arrive_expect_tx(&xfull[st], xbytes);
          mbar_arrive_expect_tx(&fullb[st], wbytes);
        } else {
          mbar_arrive_expect_tx(&fullb[st], wbytes + xbytes);
        }
        uint64_t *xbar = NORM == 1 ? &xfull[st] : &fullb[st];
        for (int kt = 0; kt < nv; ++kt) {
          const int k0 = (tile0 + i * NT + kt) * TC_TILE_K;
          // activations: only after the previous kernel's results are visible
          // (prepared tiles: rows tile * 2 bn .. of the prep kernel's buffer)
          if (i >= S0) {
            const int tl = tile0 + i * NT + kt;
            tma_load_2d(sb + p.a_bytes + kt * p.xt_bytes, &maps.x, xbar,
                        NORM == 2 ? 0 : k0, NORM == 2 ? tl * 2 * BN : xrow, pol_x);
          }
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int mi = (full || h[t] == p.hmax) ? 0 : 1;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              uint8_t *dst = sb + ((kt * MT + t) * NMAT + m) * p.rc * 128;
              const CUtensorMap *wm = m == 0 ? &maps.wg[mi] : &maps.wu[mi];
              if (IL) {
                tma_load_3d(dst, &maps.wg[mi], &fullb[st], k0, m, j0 + rs[t], pol_w);
              } else if (COLM) {
                // columns j0 .. j0 + 63 and j0 + 64 .. j0 + 127, 64 k rows each
                tma_load_2d(dst, wm, &fullb[st], j0, k0, pol_w);
                tma_load_2d(dst + 8192, wm, &fullb[st], j0 + 64, k0, pol_w);
              } else {
                tma_load_2d(dst, wm, &fullb[st], k0, wrow + j0 + rs[t], pol_w);
              }
            }
          }
        }
        if (i == S0 - 1) {
          // the weights never depend on the previous kernel: pull the next
          // pf_steps steps' boxes into L2 while it finishes
          const int pf_end = min(nsteps, S0 + p.pf_steps);
          for (int ii = S0; ii < pf_end; ++ii) {
            const int nvi = min(NT, tile1 - (tile0 + ii * NT));
            for (int kt = 0; kt < nvi; ++kt) {
              const int k0 = (tile0 + ii * NT + kt) * TC_TILE_K;
#pragma unroll
              for (int t = 0; t < MT; ++t) {
                const int mi = (full || h[t] == p.hmax) ? 0 : 1;
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                  const CUtensorMap *wm = m == 0 ? &maps.wg[mi] : &maps.wu[mi];
                  if (IL) {
                    tma_prefetch_3d(&maps.wg[mi], k0, m, j0 + rs[t]);
                  } else if (COLM) {
                    tma_prefetch_2d(wm, j0, k0);
                    tma_prefetch_2d(wm, j0 + 64, k0);
                  } else {
                    tma_prefetch_2d(wm, k0, wrow + j0 + rs[t]);
                  }
                }
              }
            }
          }
          pdl_wait();
          for (int ii = 0; ii < S0; ++ii) {
            const int nvi = min(NT, tile1 - (tile0 + ii * NT));
            for (int kt = 0; kt < nvi; ++kt) {
              const int tl = tile0 + ii * NT + kt;
              tma_load_2d(smem + static_cast<size_t>(ii) * p.stage_bytes + p.a_bytes +
                              kt * p.xt_bytes,
                          &maps.x, NORM == 1 ? &xfull[ii] : &fullb[ii],
                          NORM == 2 ? 0 : tl * TC_TILE_K,
                          NORM == 2 ? tl * 2 * BN : xrow, pol_x);
            }
          }
        }
        issued = i + 1;
      }
      *s_issued = issued;
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    // The whole warp walks the ring, so every descriptor below is a
    // warp-uniform value; one elected lane issues the MMAs and commits.
    // (Issued from a single-lane branch each MMA cost ~50 cycles of issue,
    // holding its ring stage for that long.)
    // Each output may accumulate into NB independent TMEM banks (k-slice kk
    // of a tile goes to bank kk % NB); the epilogue adds the banks in a fixed
    // order.  One MMA covers N = bn tokens, or with the prologue N = 2 bn
    // (the hi rows, then the lo rows).
    __syncwarp();
    const uint32_t leader = elect_one_sync();
    {
      const int WN = NORM ? 2 * BN : BN;
      const uint32_t idesc = umma_idesc_bf16_f32(128, WN, COLM);
      const int NB = p.nbank;
      // descriptors are built once; the address field (bits 0-13, 16-byte
      // units) is then advanced by plain addition (shared memory < 256 KB)
      const uint64_t desc0 = umma_desc_sw128(sbase);
      const uint32_t tile_enc = static_cast<uint32_t>(p.rc * 128) >> 4;
      const uint32_t x_enc = static_cast<uint32_t>(p.a_bytes) >> 4;
      const uint32_t xt_enc = static_cast<uint32_t>(p.xt_bytes) >> 4;
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S;
        bool ok = mbar_wait_bounded(&fullb[st], (i / S) & 1, s_abort, p.err);
        if (NORM == 1 && ok) ok = mbar_wait_bounded(&xready[st], (i / S) & 1, s_abort, p.err);
        if (!__all_sync(0xffffffffu, ok)) break;  // the warp leaves together
        tc_fence_after();
        const uint64_t ds = desc0 + (static_cast<uint32_t>(st * p.stage_bytes) >> 4);
        const int nv = min(NT, tile1 - (tile0 + i * NT));
        for (int kt = 0; kt < nv; ++kt) {
          const uint64_t bx = ds + x_enc + kt * xt_enc;
          const uint64_t at = ds + static_cast<uint64_t>(kt * MT * NMAT) * tile_enc;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int b = kk % NB;
            const uint32_t acc = (i > 0 || kt > 0 || kk >= NB) ? 1u : 0u;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
#pragma unroll
              for (int m = 0; m < NMAT; ++m) {
                // K-major: the 16-element k-slice kk starts 32 bytes into each
                // swizzled row; MN-major: it is the atom pair 2 kk, 2 kk + 1
                // (2048 bytes per slice), with atoms 8192 bytes apart along M
                const uint64_t a =
                    COLM ? umma_desc_sw128_mn(0u, 8192u, 1024u) +
                               (((at + static_cast<uint64_t>(t * NMAT + m) * tile_enc) &
                                 0x3FFFull) +
                                (2048u >> 4) * kk)
                         : at + static_cast<uint64_t>(t * NMAT + m) * tile_enc + 2 * kk;
                const uint32_t d = tmem + static_cast<uint32_t>(((t * NMAT + m) * NB + b) * WN);
                if (leader) umma_bf16(d, a, bx + 2 * kk, idesc, acc);
              }
            }
          }
        }
        if (leader) umma_commit(&empty[st]);  // the stage is free once these MMAs have read it
        __syncwarp();
      }
      if (leader) umma_commit(accfull);       // every MMA issued above has completed
    }
  } else {
    // ================= x*gamma transform (NORM = 1) and epilogue: warps 2..5
    const int et = tid - 64;
    if (NORM == 2) pdl_wait();  // r_b comes from the prep kernel
    if (NORM == 1) {
      // gamma is a weight: read before the dependency on the previous kernel
      // resolves, every thread's loads in flight together
      const int kpad = ((p.ntiles + NT - 1) / NT) * NT * TC_TILE_K;
      for (int base = et; base < kpad / 8; base += 4 * 128) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = (base + 128 * u) * 8;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (k < p.K && DFK_IN_BOUNDS(k + 8 <= p.K, 4, p.err)) v[u] = ld_nc_v4(p.gamma + k);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (base + 128 * u < kpad / 8)
            *reinterpret_cast<uint4 *>(gs + (base + 128 * u) * 8) = v[u];
      }
      pdl_wait();
      named_barrier(1, 128);
      // task t = et + 128 c (c < BN / 16) is 16-byte chunk (t & 7) of token row
      // t >> 3: the 8 lanes of a shared-memory phase cover the 8 chunks of one
      // row (conflict-free), and the 8 lanes of a row reduce its sum of squares
      const int cpt = BN / 16;        // rows (chunks) per thread per k-tile: 1, 2 or 4
      const int pc = et & 7;          // physical 16-byte chunk
      float ss[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S;
        const bool ok = mbar_wait_bounded(&xfull[st], (i / S) & 1, s_abort, p.err);
        if (ok) {
          uint8_t *sb = smem + static_cast<size_t>(st) * p.stage_bytes;
          const int nv = min(NT, tile1 - (tile0 + i * NT));
          for (int kt = 0; kt < nv; ++kt) {
            uint8_t *xt = sb + p.a_bytes + kt * p.xt_bytes;
            uint8_t *lt = xt + BN * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (c >= cpt) break;
              const int n = (et >> 3) + 16 * c;       // token row
              const int lc = pc ^ (n & 7);            // 128-byte swizzle: logical chunk
              const int k = (tile0 + i * NT + kt) * TC_TILE_K + 8 * lc;
              const uint4 xv = *reinterpret_cast<const uint4 *>(xt + n * 128 + pc * 16);
              const uint4 gv = *reinterpret_cast<const uint4 *>(gs + k);
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float x0 = bf16_lo(xw[q]), x1 = bf16_hi(xw[q]);
                ss[c] = fmaf(x0, x0, ss[c]);
                ss[c] = fmaf(x1, x1, ss[c]);
                const float p0 = x0 * bf16_lo(gw[q]), p1 = x1 * bf16_hi(gw[q]);  // exact
                const uint16_t h0 = f32_to_bf16_bits(p0), h1 = f32_to_bf16_bits(p1);
                const float r0 = p0 - __uint_as_float(static_cast<uint32_t>(h0) << 16);
                const float r1 = p1 - __uint_as_float(static_cast<uint32_t>(h1) << 16);
                hw[q] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
                lw[q] = static_cast<uint32_t>(f32_to_bf16_bits(r0)) |
                        (static_cast<uint32_t>(f32_to_bf16_bits(r1)) << 16);
              }
              *reinterpret_cast<uint4 *>(xt + n * 128 + pc * 16) =
                  make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4 *>(lt + n * 128 + pc * 16) =
                  make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&xready[st]);
      }
      // sum of squares of each row: its 8 chunks sit in 8 adjacent lanes
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v = ss[c];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        const int n = (et >> 3) + 16 * c;
        if (c < cpt && pc == 0)
          s_rinv[n] = (n < p.B) ? 1.0f / sqrtf(v / static_cast<float>(p.K) + p.eps) : 0.f;
      }
      named_barrier(1, 128);
    }

    // ---- epilogue: TMEM -> registers -> SiLU(gate) * up -> bf16 h
    const bool ok = mbar_wait_bounded(accfull, 0, s_abort, p.err);
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, ok && !*s_abort);
    const int q = warp & 3;               // TMEM lanes 32q .. 32q + 31 belong to this warp
    const int row = 32 * q + lane;
    const bool tp = NMAT == 1 && p.tp_world > 0;
    const int tp_src = p.tp_rank0 + tpl;  // this CTA's rank
    unsigned long long tp_seq = 0;
    int tp_set = 0;
    if (tp) {
      // the previous call's counter update is visible once the grids before
      // this one have completed
      pdl_wait();
      tp_seq = *reinterpret_cast<volatile unsigned long long *>(p.tp_seq) + 1;
      tp_set = static_cast<int>(tp_seq & 1);
    }
    if (go) {
      const int NB = p.nbank;
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        for (int c = 0; c < BN; c += 16) {
          float g[16], u[16];
          const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16);
          // fixed order: per bank (hi + lo), then ((b0 + b1) + (b2 + b3))
          const int WN = NORM ? 2 * BN : BN;
          tmem_sum_banks(base + (t * NMAT) * NB * WN + c, NB, WN, NORM ? BN : 0, g);
          if (NMAT == 2)
            tmem_sum_banks(base + (t * NMAT + 1) * NB * WN + c, NB, WN, NORM ? BN : 0, u);
          if (p.kslices > 1) {
            // split-K: this slice's partial sums, [n][row] so a warp's stores coalesce
            float *mine = p.part + (static_cast<size_t>(slc) * p.nblocks + blk) * BN * 128;
#pragma unroll
            for (int e = 0; e < 16; ++e) mine[(c + e) * 128 + row] = g[e];
          } else if (tp) {
            // tensor-parallel: this rank's fp32 partial rows into slot tp_src
            // of every rank's receive buffer (peer stores over NVLink)
            if (row < h[t]) {
              const int j = j0 + rs[t] + row;
              for (int d = 0; d < p.tp_world; ++d) {
                float *dst = p.tp_recv[d] +
                             (static_cast<size_t>(tp_set * p.tp_world + tp_src) * p.tp_bmax) * p.N +
                             j;
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  if (c + e < p.B &&
                      DFK_IN_BOUNDS(j < p.N && c + e < p.tp_bmax && d < p.tp_world, 5, p.err))
                    dst[static_cast<size_t>(c + e) * p.N] = g[e];
              }
            }
          } else if (row < h[t]) {
            const int j = j0 + rs[t] + row;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int n = c + e;
              if (n < p.B) {
                float res;
                const float sc = NORM == 1 ? s_rinv[n] : (NORM == 2 ? p.rinv[n] : 1.0f);
                if (NMAT == 2) {
                  const float a = g[e] * sc, uu = u[e] * sc;
                  res = (a / (1.0f + expf(-a))) * uu;
                } else {
                  res = NORM ? g[e] * sc : g[e];
                }
                store_out(p, n, j, f32_to_bf16_bits(res));
              }
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
          auto emit = [&](int n, float acc) {
            // RMSNorm with split-K only in mode 2 (r_b over all of K)
            if (NORM == 2) acc *= p.rinv[n];
            store_out(p, n, j0 + row, f32_to_bf16_bits(acc));
          };
          // up to four slices: 16 tokens per batch of loads, else 8
          if (p.kslices <= 4)
            splitk_reduce_row_n<4>(p.part, p.kslices, p.nblocks, blk, BN, p.B, row, emit);
          else
            splitk_reduce_row(p.part, p.kslices, p.nblocks, blk, BN, p.B, row, emit);
        }
        named_barrier(2, 128);
        if (et == 0) p.counters[blk] = 0u;
      }
    }
    if (tp) {
      // publish: every thread's partial rows are visible system-wide before
      // this CTA's flag is raised in each rank's flag array
      __threadfence_system();
      named_barrier(2, 128);
      if (et == 0 && go) {
        for (int d = 0; d < p.tp_world; ++d)
          st_release_sys_u64(p.tp_flags[d] + static_cast<size_t>(blk) * p.tp_world + tp_src,
                             tp_seq);
        // every rank's partial of this row block has arrived (bounded wait)
        flags_wait_bounded(p.tp_flags[tp_src] + static_cast<size_t>(blk) * p.tp_world,
                           p.tp_world, tp_seq, s_abort, p.err);
      }
      named_barrier(2, 128);
      if (go && !*s_abort) {
        // y = the ranks' partial sums added in rank order 0, 1, ..., the same
        // order (and so the same bits) on every rank
        const float *src = p.tp_recv[tp_src] +
                           static_cast<size_t>(tp_set) * p.tp_world * p.tp_bmax * p.N;
        uint16_t *y = p.out + static_cast<size_t>(tpl) * p.B * p.N;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (row < h[t]) {
            const int j = j0 + rs[t] + row;
            for (int n = 0; n < p.B; ++n) {
              const float *v = src + static_cast<size_t>(n) * p.N + j;
              float acc = __ldcg(v);
              for (int r = 1; r < p.tp_world; ++r)
                acc = acc + __ldcg(v + static_cast<size_t>(r) * p.tp_bmax * p.N);
              if (DFK_IN_BOUNDS(j < p.N && n < p.B, 6, p.err))
                y[static_cast<size_t>(n) * p.N + j] = f32_to_bf16_bits(acc);
            }
          }
        }
      }
      // the grid's last CTA to get here advances the call counter (every CTA
      // has read it above) and re-arms the exit count
      named_barrier(2, 128);
      if (et == 0) {
        __threadfence();
        if (atomicAdd(p.tp_exit, 1u) == gridDim.x - 1) {
          *reinterpret_cast<volatile unsigned long long *>(p.tp_seq) = tp_seq;
          *reinterpret_cast<volatile unsigned *>(p.tp_exit) = 0u;
          __threadfence();
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
      if (last >= 0) {
        mbar_wait_bounded(&fullb[st], (last / S) & 1, nullptr, p.err);
        if (NORM == 1) mbar_wait_bounded(&xfull[st], (last / S) & 1, nullptr, p.err);
      }
    }
  }
}

// ---- prep for NORM = 2: one CTA per token slot b = blockIdx.x, one pass
// over x.  x * gamma (exact in fp32) is split into bf16 hi + lo and written
// as rows tile * 2 bn + b (hi) and tile * 2 bn + bn + b (lo) of 64 bf16 per
// k tile -- zeros past K and for b >= B -- as each chunk of 8 elements
// arrives (the split does not depend on r_b); sum x^2 in a fixed order (each
// thread chains its chunks c = t + TC_PREP_THREADS * i, i then e ascending;
// a xor butterfly per warp; the warps in order) gives r_b.  Defined in the
// one file that instantiates the kernels.
struct TcPrepParams {
  const uint16_t *x;      // [B][K] bf16
  const uint16_t *gamma;  // [K] bf16
  uint16_t *xg;           // [ntiles][2 bn][64] bf16
  float *rinv;            // [bn]
  int B, K, bn, ntiles;
  float eps;
  unsigned *err;          // device status block (checked builds)
};

constexpr int TC_PREP_THREADS = 512;

#ifdef DFK_TC_KERNELS
// At most 40 registers a thread (three CTAs' worth per SM): a prep CTA must
// fit in the register file beside one CTA of the main kernel (192 threads,
// up to 216 registers).
__global__ void __launch_bounds__(TC_PREP_THREADS, 3) tc_norm_prep_kernel(const TcPrepParams p) {
  __shared__ float s_wss[TC_PREP_THREADS / 32];
  pdl_launch_dependents();
  pdl_wait();  // x comes from the previous kernel
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool real = b < p.B;
  const int nchunk = p.ntiles * TC_TILE_K / 8, kchunks = p.K / 8;
  float ss = 0.f;
  for (int c0 = tid; c0 < nchunk; c0 += 2 * TC_PREP_THREADS) {
    uint4 xv[2], gv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {  // two chunks' loads in flight per thread
      const int c = c0 + i * TC_PREP_THREADS;
      xv[i] = gv[i] = make_uint4(0u, 0u, 0u, 0u);
      if (real && c < kchunks && DFK_IN_BOUNDS(8 * c + 8 <= p.K, 7, p.err)) {
        xv[i] = ld_nc_v4(p.x + static_cast<size_t>(b) * p.K + 8 * c);
        gv[i] = ld_nc_v4(p.gamma + 8 * c);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = c0 + i * TC_PREP_THREADS;
      if (c >= nchunk) continue;
      const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
      const uint32_t gw[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x0 = bf16_lo(xw[u]), x1 = bf16_hi(xw[u]);
        ss = fmaf(x0, x0, ss);
        ss = fmaf(x1, x1, ss);
        const float p0 = x0 * bf16_lo(gw[u]);  // exact
        const float p1 = x1 * bf16_hi(gw[u]);
        const uint16_t h0 = f32_to_bf16_bits(p0), h1 = f32_to_bf16_bits(p1);
        const float r0 = p0 - __uint_as_float(static_cast<uint32_t>(h0) << 16);
        const float r1 = p1 - __uint_as_float(static_cast<uint32_t>(h1) << 16);
        hw[u] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
        lw[u] = static_cast<uint32_t>(f32_to_bf16_bits(r0)) |
                (static_cast<uint32_t>(f32_to_bf16_bits(r1)) << 16);
      }
      const int k = 8 * c, tile = k / TC_TILE_K, kk = k % TC_TILE_K;
      if (!DFK_IN_BOUNDS(tile < p.ntiles && b < p.bn, 8, p.err)) continue;
      uint16_t *hrow = p.xg + (static_cast<size_t>(tile) * 2 * p.bn + b) * TC_TILE_K;
      *reinterpret_cast<uint4 *>(hrow + kk) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(hrow + static_cast<size_t>(p.bn) * TC_TILE_K + kk) =
          make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  if (lane == 0) s_wss[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < TC_PREP_THREADS / 32; ++w) t += s_wss[w];
    p.rinv[b] = real ? 1.0f / sqrtf(t / static_cast<float>(p.K) + p.eps) : 0.f;
  }
}
#endif  // DFK_TC_KERNELS

}  // namespace dfk
