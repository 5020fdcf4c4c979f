// pstack_engine.cuh -- one decode step of a stack of SwiGLU MLP layers as a
// single persistent kernel (tcgen05 / TMEM).
//
// A decode step streams every layer's weights once: for layer l the fused
// RMSNorm + gate/up + SiLU * up (h_l = SiLU(xn W_gate_l^T) * (xn W_up_l^T),
// xn = RMSNorm(x_l; gamma_l)) and then the separate down projection
// (y_l = h_l W_down_l^T, x_{l+1} = y_l), and after the last layer the
// per-row rescale x_next = y / sqrt(mean(y^2) + eps) ("Deep Kernel Fusion
// for Transformer Decoding", episode description: gate/up/SiLU/multiply in
// one kernel, the down projection separate -- here they are separate
// phases of one launch; the whole-model single kernel for low-batch
// inference is the FlashFormer idea on the paper-listing page).
//
// Why one launch: with one kernel per projection every layer boundary
// drains the weight stream -- the next kernel's CTAs cannot start streaming
// until the previous kernel's CTAs have left their SMs.  The weights never
// depend on the activations, so here a producer warp per SM streams the
// weights of phase after phase (gate/up of layer 0, down of layer 0, gate/up
// of layer 1, ...) into its shared-memory ring without ever waiting for an
// activation; only the consumers wait, at each phase boundary, for every
// CTA to have finished the previous phase (a grid-wide counter; the grid is
// a cooperative launch, so every CTA is resident).
//
// Work split (one CTA per SM, G CTAs):
//   gate/up phase: CTA c owns ~F / G rows of both matrices over the whole
//     reduction (d_model), one 128-row MMA tile, like the tensor-core gate/up
//     kernel with the in-kernel RMSNorm transform;
//   down phase: G / 4 row blocks x 4 reduction slices; every CTA writes its
//     fp32 partial rows, the last to arrive on a row block adds the four
//     slices in order 0, 1, 2, 3 and stores y (the split-K tensor-core GEMV).
// The arithmetic -- the MMA k order, the hi + lo split of x * gamma, the
// order of the sum of squares for r_b, the epilogues, the slice order, and
// the final rescale's order -- is that of the separate kernels
// (tc_engine.cuh mode 1 with 16 token slots, the split-K GEMV with four
// slices, the rescale kernel), so a step gives the same bits as the 2L + 1
// kernel launches with those variants.
//
// Warp roles (192 threads):
//   warp 0     producer (one lane): for every ring step of every phase it
//              issues the weight tiles at once -- weights never depend on
//              the activations -- and the step's activation tiles (x or the
//              previous layer's y, and gamma, for gate/up; h for the down
//              projection) as soon as the phase's grid-wide count shows the
//              previous phase done; steps issued before that get their
//              activation tiles back-filled when it does;
//   warp 1     MMA issuer (one elected lane): per step, waits for the
//              weights and for the activation tiles to be ready, issues the
//              MMAs into the phase's TMEM buffer (two buffers, alternating
//              phases) and frees the slot with a commit;
//   warps 2-5  transform and epilogue: turn each gate/up activation tile
//              into x * gamma split into bf16 hi and lo rows in place (the
//              sum of squares on the way), then read the accumulators and
//              store h (SiLU(a) * u) or the down projection's partial sums,
//              and count the phase as done.
// Outputs that a later phase loads with TMA are written by ordinary stores:
// the writer fences them toward the async proxy before counting its phase,
// and the producer fences after seeing the count.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "tc_engine.cuh"
#include "tc_ptx.cuh"

namespace dfk {

constexpr int PS_THREADS = 192;
constexpr int PS_BN = 16;       // token slots on the MMA's N (x hi rows; + 16 lo rows)
constexpr int PS_KSPLIT = 4;    // reduction slices of the down projection
constexpr int PS_TILE_K = 64;   // reduction elements per k tile (one 128-byte row)
constexpr int PS_ATILE = 2 * PS_BN * 128;   // gate/up activation tile: hi rows then lo rows
constexpr int PS_DTILE = PS_BN * 128;       // down activation tile (h rows)
constexpr int PS_TMEM_COLS = 128;           // two buffers of 64 columns

struct PsMaps {
  CUtensorMap wg[2];  // stacked W_gate [L * F][D]: box {64, gu_hmax}, {64, gu_hmax - 1};
                      // column-major [L * D][F]: box {64 columns, 64 k rows} in wg[0]
  CUtensorMap wu[2];  // stacked W_up, same boxes
  CUtensorMap wd[2];  // stacked W_down [L * D][F]: box {64, dn_hmax}, {64, dn_hmax - 1}
  CUtensorMap x;      // step input [B][D]: box {64, 16}
  CUtensorMap y;      // every layer's y [L * B][D]: box {64, 16}
  CUtensorMap h;      // every layer's h [L * B][F]: box {64, 16}
  CUtensorMap gam;    // gammas [L][D]: box {64, 1}, no swizzle
};

// Orders this thread's generic-proxy global writes before later async-proxy
// (TMA) accesses, and the reverse.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

struct PsParams {
  const uint16_t *gamma;  // [L][D] bf16
  uint16_t *x;            // [B][D] bf16 step input; receives the rescaled output
  uint16_t *h;            // [L][B][F] bf16, every layer's h
  uint16_t *y;            // [L][B][D] bf16, every layer's y
  float *part;            // [PS_KSPLIT][dn_nblk][PS_BN][128] fp32 partial sums
  unsigned *ctl;          // [0] launch epoch, [1] CTAs done, [2 .. 2 + 2L) CTAs done per
                          // phase (cumulative over launches), then [dn_nblk] row-block counts
  unsigned *err;          // device status block
  int L, B, D, F;
  float eps;
  int gu_rbase, gu_rextra, gu_hmax, gu_rc, gu_tiles, gu_nt;
  int gu_col;             // 1: W_gate / W_up column-major, 128 columns per CTA (MN-major A)
  int dn_nblk, dn_rbase, dn_rextra, dn_hmax, dn_rc, dn_tiles, dn_nt;
  // (nt: k tiles per ring step -- consecutive 128-byte pieces of each weight
  // row in one step, for DRAM locality)
  int S, slot_bytes;      // ring: S slots of slot_bytes
  int x_off;              // offset of a slot's activation tiles
  int g_off;              // offset of a slot's gamma slices (gate/up steps)
  int bar_off;            // barriers, from the 1024-byte aligned base
};

#ifdef DFK_PSTACK_KERNELS

// Wait until *ctr >= want (a grid-wide phase count), bounded like the
// pipeline waits.
__device__ __forceinline__ bool ps_grid_wait(const unsigned *ctr, unsigned want,
                                             volatile int *abort_flag, unsigned *err) {
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long limit = wait_limit_ns(err);
  for (uint32_t it = 1;; ++it) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (static_cast<int>(v - want) >= 0) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit || it > (1u << 30)) {
        *abort_flag = 1;
        atomicOr(err, ERR_WAIT_TIMEOUT);
        return false;
      }
    }
    __nanosleep(64);
  }
}

__global__ void __launch_bounds__(PS_THREADS, 1)
    pstack_kernel(const __grid_constant__ PsMaps maps, const PsParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.S;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nphase = 2 * p.L;

  uint64_t *wfull = reinterpret_cast<uint64_t *>(smem + p.bar_off);  // weights landed
  uint64_t *afull = wfull + S;        // activation tiles (and gamma) landed
  uint64_t *xready = afull + S;       // activation tiles ready for the MMA
  uint64_t *wempty = xready + S;      // slot read by the MMAs
  uint64_t *accfull = wempty + S;     // [2]
  uint64_t *tmempty = accfull + 2;    // [2]
  uint64_t *mmadone = tmempty + 2;
  volatile int *s_abort = reinterpret_cast<volatile int *>(mmadone + 1);
  int *s_issued = reinterpret_cast<int *>(mmadone + 1) + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(mmadone + 1) + 2;
  volatile int *s_last = reinterpret_cast<volatile int *>(mmadone + 1) + 3;
  unsigned *s_epoch = reinterpret_cast<unsigned *>(mmadone + 1) + 4;
  int *s_aissued = reinterpret_cast<int *>(mmadone + 1) + 5;
  float *s_rinv = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(mmadone + 1) + 32);

  // ---- partitions
  // gate/up rows: row-major ~F / G rows per CTA; column-major 128 columns per
  // CTA (the CTAs past the last column have no gate/up work)
  const int gu_j0 = p.gu_col ? cta * 128 : cta * p.gu_rbase + min(cta, p.gu_rextra);
  const int gu_r = p.gu_col ? max(0, min(128, p.F - gu_j0))
                            : p.gu_rbase + (cta < p.gu_rextra ? 1 : 0);
  const int dn_blk = cta / PS_KSPLIT, dn_slc = cta - dn_blk * PS_KSPLIT;
  const int dn_j0 = dn_blk * p.dn_rbase + min(dn_blk, p.dn_rextra);
  const int dn_r = p.dn_rbase + (dn_blk < p.dn_rextra ? 1 : 0);
  const int dn_t0 = (dn_slc * p.dn_tiles) / PS_KSPLIT;
  const int dn_t1 = ((dn_slc + 1) * p.dn_tiles) / PS_KSPLIT;
  // k tiles and ring steps of a phase
  auto phase_tiles = [&](bool gu) { return gu ? (gu_r > 0 ? p.gu_tiles : 0) : dn_t1 - dn_t0; };
  auto phase_nt = [&](bool gu) { return gu ? p.gu_nt : p.dn_nt; };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&afull[s], 1);
      mbar_init(&xready[s], 128);
      mbar_init(&wempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&tmempty[b], 4);
    }
    mbar_init(mmadone, 1);
    *s_abort = 0;
    *s_issued = 0;
    *s_aissued = 0;
    *s_epoch = *reinterpret_cast<volatile unsigned *>(p.ctl);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, PS_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const unsigned target = (*s_epoch + 1u) * static_cast<unsigned>(G);  // phase counts this launch
  unsigned *done = p.ctl + 2;
  unsigned *blkctr = p.ctl + 2 + nphase;

  if (warp == 0) {
    // ================= producer (one lane)
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_normal();
      // activation tiles of step (phase ph, step i) into ring slot st
      auto issue_act = [&](int ph, int i, int st) {
        const int l = ph >> 1;
        const bool gu = (ph & 1) == 0;
        const int nt = phase_nt(gu), ntl = phase_tiles(gu);
        const int nv = min(nt, ntl - nt * i);
        uint8_t *xa = smem + static_cast<size_t>(st) * p.slot_bytes + p.x_off;
        const CUtensorMap *map = gu ? (l == 0 ? &maps.x : &maps.y) : &maps.h;
        const int row0 = gu ? (l == 0 ? 0 : (l - 1) * p.B) : l * p.B;
        mbar_arrive_expect_tx(&afull[st],
                              static_cast<uint32_t>(nv) * (PS_BN * 128u + (gu ? 128u : 0u)));
        for (int kt = 0; kt < nv; ++kt) {
          const int k0 = ((gu ? 0 : dn_t0) + nt * i + kt) * PS_TILE_K;
          tma_load_2d(xa + kt * (gu ? PS_ATILE : PS_DTILE), map, &afull[st], k0, row0, pol_x);
          if (gu)
            tma_load_2d(smem + static_cast<size_t>(st) * p.slot_bytes + p.g_off + kt * 128,
                        &maps.gam, &afull[st], k0, l, pol_x);
        }
      };
      // the previous phase is done grid-wide (checked without waiting); its
      // outputs are then visible to this thread's TMA loads
      auto phase_open = [&](int ph) {
        if (ph == 0) return true;
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(done + ph - 1)
                     : "memory");
        if (static_cast<int>(v - target) < 0) return false;
        fence_proxy_async_global();
        return true;
      };
      int open_ph = 0;              // phases up to this one have their activations open
      int pend_q[8], pend_ph[8], pend_i[8];
      int npend = 0, head = 0;      // steps issued without activation tiles (FIFO)
      int q = 0;
      bool ok = true;
      const unsigned long long limit = wait_limit_ns(p.err);
      // issue the pending activation tiles once their phase opens
      auto flush = [&]() {
        while (npend > 0) {
          const int ph = pend_ph[head];
          if (ph > open_ph) {
            if (!phase_open(ph)) return;
            open_ph = ph;
          }
          issue_act(ph, pend_i[head], pend_q[head] % S);
          *s_aissued = pend_q[head] + 1;
          head = (head + 1) & 7;
          --npend;
        }
      };
      for (int ph = 0; ph < nphase && ok; ++ph) {
        const int l = ph >> 1;
        const bool gu = (ph & 1) == 0;
        const int nt = phase_nt(gu), ntl = phase_tiles(gu);
        const int nsteps = (ntl + nt - 1) / nt;
        for (int i = 0; i < nsteps; ++i, ++q) {
          const int st = q % S;
          if (q >= S) {
            // wait for the slot, opening pending activations meanwhile
            const unsigned long long t0 = global_timer_ns();
            for (uint32_t it = 1; !mbar_try_wait(&wempty[st], ((q / S) - 1) & 1); ++it) {
              if (npend) flush();
              if ((it & 15u) == 0) {
                if (*s_abort || global_timer_ns() - t0 > limit) {
                  if (!*s_abort) atomicOr(p.err, ERR_WAIT_TIMEOUT);
                  *s_abort = 1;
                  ok = false;
                  break;
                }
              }
            }
            if (!ok) break;
          }
          uint8_t *slot = smem + static_cast<size_t>(st) * p.slot_bytes;
          const int nv = min(nt, ntl - nt * i);  // k tiles of this step
          if (gu && p.gu_col) {
            // weight tiles [kt][gate | up], each two boxes of 64 columns x 64 k rows
            mbar_arrive_expect_tx(&wfull[st], static_cast<uint32_t>(nv) * 2u * 16384u);
            for (int kt = 0; kt < nv; ++kt) {
              const int krow = l * p.D + (nt * i + kt) * PS_TILE_K;
#pragma unroll
              for (int m = 0; m < 2; ++m) {
                uint8_t *tile = slot + (2 * kt + m) * 16384;
                const CUtensorMap *wm = m == 0 ? &maps.wg[0] : &maps.wu[0];
                tma_load_2d(tile, wm, &wfull[st], gu_j0, krow, pol_w);
                tma_load_2d(tile + 8192, wm, &wfull[st], gu_j0 + 64, krow, pol_w);
              }
            }
          } else if (gu) {
            // weight tiles [kt][gate | up], gu_rc rows each
            const int mi = gu_r == p.gu_hmax ? 0 : 1;
            mbar_arrive_expect_tx(&wfull[st], static_cast<uint32_t>(nv) * 2u * gu_r * 128u);
            const int row = l * p.F + gu_j0;
            for (int kt = 0; kt < nv; ++kt) {
              const int k0 = (nt * i + kt) * PS_TILE_K;
              tma_load_2d(slot + (2 * kt) * p.gu_rc * 128, &maps.wg[mi], &wfull[st], k0, row,
                          pol_w);
              tma_load_2d(slot + (2 * kt + 1) * p.gu_rc * 128, &maps.wu[mi], &wfull[st], k0,
                          row, pol_w);
            }
          } else {
            const int mi = dn_r == p.dn_hmax ? 0 : 1;
            mbar_arrive_expect_tx(&wfull[st], static_cast<uint32_t>(nv) * dn_r * 128u);
            for (int kt = 0; kt < nv; ++kt)
              tma_load_2d(slot + kt * p.dn_rc * 128, &maps.wd[mi], &wfull[st],
                          (dn_t0 + nt * i + kt) * PS_TILE_K, l * p.D + dn_j0, pol_w);
          }
          *s_issued = q + 1;
          // the activation tiles now, or when the phase opens
          pend_q[(head + npend) & 7] = q;
          pend_ph[(head + npend) & 7] = ph;
          pend_i[(head + npend) & 7] = i;
          ++npend;
          flush();
        }
      }
      // the last steps' activations (bounded wait for their phase)
      const unsigned long long t0 = global_timer_ns();
      for (uint32_t it = 1; ok && npend > 0; ++it) {
        flush();
        if (npend && (it & 15u) == 0 && (*s_abort || global_timer_ns() - t0 > limit)) {
          if (!*s_abort) atomicOr(p.err, ERR_WAIT_TIMEOUT);
          *s_abort = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer: the warp walks the ring, one lane issues
    __syncwarp();
    const uint32_t leader = elect_one_sync();
    const uint32_t idesc_gu = umma_idesc_bf16_f32(128, 2 * PS_BN, p.gu_col != 0);
    const uint32_t idesc_dn = umma_idesc_bf16_f32(128, PS_BN);
    const uint64_t desc0 = umma_desc_sw128(sbase);
    int q = 0;  // ring steps consumed over all phases
    bool ok = true;
    for (int ph = 0; ph < nphase && ok; ++ph) {
      const bool gu = (ph & 1) == 0;
      const int buf = ph & 1;
      if (ph >= 2) ok = mbar_wait_bounded(&tmempty[buf], ((ph >> 1) - 1) & 1, s_abort, p.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int nt = phase_nt(gu), ntl = phase_tiles(gu);
      const int nsteps = (ntl + nt - 1) / nt;
      for (int i = 0; i < nsteps && ok; ++i, ++q) {
        const int st = q % S;
        ok = mbar_wait_bounded(&wfull[st], (q / S) & 1, s_abort, p.err);
        if (ok) ok = mbar_wait_bounded(&xready[st], (q / S) & 1, s_abort, p.err);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        const uint64_t ws = desc0 + (static_cast<uint32_t>(st * p.slot_bytes) >> 4);
        const uint64_t xs = ws + (static_cast<uint32_t>(p.x_off) >> 4);
        const int nv = min(nt, ntl - nt * i);
        for (int kt = 0; kt < nv; ++kt) {
          const uint64_t bx = xs + (static_cast<uint32_t>(kt * (gu ? PS_ATILE : PS_DTILE)) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (i > 0 || kt > 0 || kk > 0) ? 1u : 0u;
            if (gu) {
#pragma unroll
              for (int m = 0; m < 2; ++m) {
                // K-major rows: the 16-element k slice kk starts 32 bytes into
                // each swizzled row; MN-major (column-major weights): it is the
                // atom pair 2 kk, 2 kk + 1 (2048 bytes per slice), atoms 8 KB
                // apart along M
                const uint64_t a =
                    p.gu_col
                        ? umma_desc_sw128_mn(0u, 8192u, 1024u) +
                              ((((ws + (static_cast<uint32_t>((2 * kt + m) * 16384) >> 4)) &
                                 0x3FFFull)) +
                               (2048u >> 4) * kk)
                        : ws + (static_cast<uint32_t>((2 * kt + m) * p.gu_rc * 128) >> 4) +
                              2 * kk;
                if (leader)
                  umma_bf16(tmem + buf * 64 + m * 2 * PS_BN, a, bx + 2 * kk, idesc_gu, acc);
              }
            } else {
              const uint64_t a = ws + (static_cast<uint32_t>(kt * p.dn_rc * 128) >> 4) + 2 * kk;
              if (leader) umma_bf16(tmem + buf * 64, a, bx + 2 * kk, idesc_dn, acc);
            }
          }
        }
        if (leader) umma_commit(&wempty[st]);  // the slot is free once these MMAs read it
        __syncwarp();
      }
      if (ok && leader) umma_commit(&accfull[buf]);
      __syncwarp();
    }
    if (leader) umma_commit(mmadone);  // every MMA issued above has completed
    __syncwarp();
  } else {
    // ================= transform and epilogue: warps 2..5 (128 threads)
    const int et = tid - 64;
    const int q4 = warp & 3;            // TMEM lanes 32 q4 .. 32 q4 + 31
    const int row = 32 * q4 + lane;     // accumulator row (output row of the CTA)
    const int n = et >> 3;              // token slot this thread converts (0 .. 15)
    const int pc = et & 7;              // physical 16-byte chunk of the 128-byte row
    int q = 0;                          // ring steps seen over all phases
    for (int ph = 0; ph < nphase; ++ph) {
      const int l = ph >> 1;
      const bool gu = (ph & 1) == 0;
      const int buf = ph & 1;
      const int nt = phase_nt(gu), ntl = phase_tiles(gu);
      const int nsteps = (ntl + nt - 1) / nt;
      float ss = 0.f;
      for (int i = 0; i < nsteps; ++i, ++q) {
        const int st = q % S;
        // every step's activations pass through here, so each slot's barrier
        // phases are waited for in order
        if (!mbar_wait_bounded(&afull[st], (q / S) & 1, s_abort, p.err)) break;
        if (gu) {
          uint8_t *xa = smem + static_cast<size_t>(st) * p.slot_bytes + p.x_off;
          const int nv = min(nt, ntl - nt * i);
          for (int kt = 0; kt < nv; ++kt) {
            // x * gamma (exact in fp32) split into bf16 hi + lo; sum of x^2
            uint8_t *xt = xa + kt * PS_ATILE;
            const int lc = pc ^ (n & 7);  // logical chunk (128-byte swizzle)
            const uint4 gv = *reinterpret_cast<const uint4 *>(
                smem + static_cast<size_t>(st) * p.slot_bytes + p.g_off + kt * 128 + 16 * lc);
            const uint4 xv = *reinterpret_cast<const uint4 *>(xt + n * 128 + pc * 16);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float x0 = bf16_lo(xw[qq]), x1 = bf16_hi(xw[qq]);
              ss = fmaf(x0, x0, ss);
              ss = fmaf(x1, x1, ss);
              const float p0 = x0 * bf16_lo(gw[qq]), p1 = x1 * bf16_hi(gw[qq]);
              const uint16_t h0 = f32_to_bf16_bits(p0), h1 = f32_to_bf16_bits(p1);
              const float r0 = p0 - __uint_as_float(static_cast<uint32_t>(h0) << 16);
              const float r1 = p1 - __uint_as_float(static_cast<uint32_t>(h1) << 16);
              hw[qq] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
              lw[qq] = static_cast<uint32_t>(f32_to_bf16_bits(r0)) |
                       (static_cast<uint32_t>(f32_to_bf16_bits(r1)) << 16);
            }
            *reinterpret_cast<uint4 *>(xt + n * 128 + pc * 16) =
                make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(xt + (PS_BN + n) * 128 + pc * 16) =
                make_uint4(lw[0], lw[1], lw[2], lw[3]);
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&xready[st]);
      }
      if (gu) {
        // r_b: each token row's 8 chunks sit in 8 adjacent lanes
        float v = ss;
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if (pc == 0)
          s_rinv[n] = n < p.B ? 1.0f / sqrtf(v / static_cast<float>(p.D) + p.eps) : 0.f;
        named_barrier(1, 128);
      }

      // ---- epilogue: TMEM -> registers
      const bool okw = mbar_wait_bounded(&accfull[buf], (ph >> 1) & 1, s_abort, p.err);
      tc_fence_after();
      const bool go = __all_sync(0xffffffffu, okw && !*s_abort);
      const uint32_t base = tmem + (static_cast<uint32_t>(32 * q4) << 16) + buf * 64;
      if (go) {
        float a[16], u[16];
        if (gu) {
          // per output: hi columns + lo columns (tc_engine.cuh's order)
          tmem_sum_banks(base, 1, 2 * PS_BN, PS_BN, a);
          tmem_sum_banks(base + 2 * PS_BN, 1, 2 * PS_BN, PS_BN, u);
          if (row < gu_r) {
            const int j = gu_j0 + row;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (e < p.B) {
                const float sc = s_rinv[e];
                const float aa = a[e] * sc, uu = u[e] * sc;
                if (DFK_IN_BOUNDS(j < p.F, 16, p.err))
                  p.h[(static_cast<size_t>(l) * p.B + e) * p.F + j] =
                      f32_to_bf16_bits((aa / (1.0f + expf(-aa))) * uu);
              }
            }
          }
        } else {
          tmem_sum_banks(base, 1, PS_BN, 0, a);
          float *mine =
              p.part + (static_cast<size_t>(dn_slc) * p.dn_nblk + dn_blk) * PS_BN * 128;
#pragma unroll
          for (int e = 0; e < 16; ++e) mine[e * 128 + row] = a[e];
        }
      }
      // the accumulators of this buffer are free for phase ph + 2
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmempty[buf]);
      if (!gu) {
        // split-K: every CTA of the row block counts (also after an abort);
        // the last one adds the slices in order and stores y_l
        __threadfence();
        named_barrier(2, 128);
        if (et == 0) {
          const unsigned old = atomicAdd(&blkctr[dn_blk], 1u);
          *s_last = (old == static_cast<unsigned>(PS_KSPLIT - 1)) ? 1 : 0;
        }
        named_barrier(2, 128);
        if (*s_last) {
          __threadfence();
          if (row < dn_r && !*s_abort)
            splitk_reduce_row_n<PS_KSPLIT>(p.part, PS_KSPLIT, p.dn_nblk, dn_blk, PS_BN, p.B, row,
                              [&](int nn, float acc) {
                                if (DFK_IN_BOUNDS(nn < p.B && dn_j0 + row < p.D, 17, p.err))
                                  p.y[(static_cast<size_t>(l) * p.B + nn) * p.D + dn_j0 +
                                      row] = f32_to_bf16_bits(acc);
                              });
          named_barrier(2, 128);
          if (et == 0) blkctr[dn_blk] = 0u;
        }
      }
      // this CTA's share of the phase is in memory: count it (the next phase
      // reads it with TMA, through the async proxy)
      fence_proxy_async_global();
      __threadfence();
      named_barrier(2, 128);
      if (et == 0) atomicAdd(&done[ph], 1u);
    }

    // ---- after the last layer: x_next[b] = y[b] / sqrt(mean(y[b]^2) + eps),
    // one warp per token row (the order of the rescale kernel: lane l sums
    // k = 8 l + 256 c + e, c then e ascending, then a xor butterfly)
    if (et == 0) ps_grid_wait(done + nphase - 1, target, s_abort, p.err);
    named_barrier(1, 128);
    if (!*s_abort) {
      const int wq = et >> 5;
      for (int b = cta * 4 + wq; b < p.B; b += G * 4) {
        const uint16_t *yr = p.y + (static_cast<size_t>(p.L - 1) * p.B + b) * p.D;
        float s2 = 0.f;
        for (int k = 8 * lane; k < p.D; k += 256) {
          const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(yr + k));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float f0 = bf16_lo(w[i]), f1 = bf16_hi(w[i]);
            s2 = fmaf(f0, f0, s2);
            s2 = fmaf(f1, f1, s2);
          }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, m);
        const float r = 1.0f / sqrtf(s2 / static_cast<float>(p.D) + p.eps);
        uint16_t *xr = p.x + static_cast<size_t>(b) * p.D;
        for (int k = 8 * lane; k < p.D; k += 256) {
          const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(yr + k));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = f32_to_bf16_bits((bf16_lo(w[i]) * r) * 1.0f);
            const uint32_t hi = f32_to_bf16_bits((bf16_hi(w[i]) * r) * 1.0f);
            o[i] = lo | (hi << 16);
          }
          if (DFK_IN_BOUNDS(k + 8 <= p.D, 18, p.err))
            *reinterpret_cast<uint4 *>(xr + k) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    // every MMA has completed before TMEM is released (bounded wait)
    if (lane == 0) mbar_wait_bounded(mmadone, 0, nullptr, p.err);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, PS_TMEM_COLS);
  }
  if (tid == 0) {
    if (*s_abort) {
      // after an aborted pipeline, wait (bounded) for copies in flight
      const int issued = *s_issued, aissued = *s_aissued;
      for (int q = issued - 1; q >= 0 && q >= issued - S; --q)
        mbar_wait_bounded(&wfull[q % S], (q / S) & 1, nullptr, p.err);
      for (int q = aissued - 1; q >= 0 && q >= aissued - S; --q)
        mbar_wait_bounded(&afull[q % S], (q / S) & 1, nullptr, p.err);
    }
    // the grid's last CTA starts the next launch's epoch
    __threadfence();
    if (atomicAdd(p.ctl + 1, 1u) == static_cast<unsigned>(G - 1)) {
      *reinterpret_cast<volatile unsigned *>(p.ctl + 1) = 0u;
      *reinterpret_cast<volatile unsigned *>(p.ctl) = *s_epoch + 1u;
      __threadfence();
    }
  }
}

#endif  // DFK_PSTACK_KERNELS

}  // namespace dfk
