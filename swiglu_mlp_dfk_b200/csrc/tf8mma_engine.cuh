// tf8mma_engine.cuh -- FP8 weights on the E4M3 tensor-core MMA
// (tcgen05.mma kind::f8f6f4): the weight codes are the MMA's A operand as
// they arrive from HBM, with no per-weight work on the CUDA cores.
//
// Same operation as the other FP8 kernels (W[j][k] = s[j] * E4M3(q[j][k]);
// "Deep Kernel Fusion for Transformer Decoding", episode description, with
// the dequantisation inside the product as GPULlama3.java PR #78 does).  The
// MMA multiplies E4M3 by E4M3, so the activations are written as a short sum
// of E4M3 terms per token b (a prep kernel does this once per call):
//   v[k] = x[b][k] * gamma[k]  (RMSNorm; exact in fp32)  or  x[b][k],
//   u[k] = v[k] * 2^e_b         (e_b puts max_k |u| in [128, 256)),
//   c_0 = E4M3(u), c_t = E4M3((u - sum_{i<t} c_i 16^-i) 16^t)  (t < T),
// so u = sum_t c_t 16^-t up to the last residual.  Two terms carry a bf16
// value exactly (8 significant bits, 4 per E4M3 term) and four terms the
// 16-bit x * gamma products, for every element within 2^17 of the token's
// largest (smaller ones are carried to about 2^-21 of it).  Term t of token
// b is row t * bnp + b of the MMA's B operand, so one MMA of N = T * bnp
// reads each weight tile once for all terms and tokens, and
//   sum_k W[j][k] v[k] = s[j] * 2^-e_b * sum_t 16^-t D[j][t * bnp + b],
// the terms combined smallest first (Horner in 1/16, exact scalings).
// The prep kernel (one CTA per token and reduction slice, a single pass
// over its part of x held in registers: the x-dependent chain between the
// previous kernel and this one is one L2 round trip and one block
// reduction) also computes r_b = 1 / sqrt(mean x^2 + eps) for the RMSNorm
// and stores f_b = r_b * 2^-e_b (1 * 2^-e_b without it).  With a k split
// (the down projection, no RMSNorm) each slice of each token has its own
// scale 2^e_b from the slice's largest element, as with the in-kernel
// terms, and each slice's partial sums are multiplied by its f_b before
// they are added (exact: a power of two).
//
// Main kernel: one CTA per SM owns r <= 128 weight rows (the MMA's M) over its
// reduction range (split-K slices for the down projection); a TMA ring
// carries 128-wide k tiles of codes (128-byte swizzle) and of the activation
// terms; one elected lane issues 4 MMAs (K = 32) per matrix per tile; warps 2-5
// read the accumulators, combine the terms, apply f_b, s[j], SiLU(gate) * up
// and store bf16.  Rows of the 128-row MMA beyond r read neighbouring shared
// memory and give ignored accumulator rows.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "tc_ptx.cuh"

namespace dfk {

constexpr int TM8_THREADS = 192;
constexpr int TM8_TILE_K = 128;
// in-kernel activation terms (no prep kernel): 8 more warps write the terms
// of the CTA's whole k range into shared memory once
constexpr int TM8_XF_THREADS = 256;
constexpr int TM8_INK_THREADS = TM8_THREADS + TM8_XF_THREADS;
constexpr int TM8_PREP_THREADS = 512;
constexpr int TM8_PREP_CPT = 2;  // chunks per prep thread kept in registers

// kind::f8f6f4 instruction descriptor: E4M3 A and B (format 0), fp32 D,
// both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc], one CTA, kind::f8f6f4 (K = 32).
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Two fp32 values -> two E4M3 codes (round to nearest even, saturating to
// +-448), lo in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Exact value of the E4M3 code in byte 0 / byte 1 of a 16-bit pair.
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t pair, float &lo, float &hi) {
  asm("{\n\t.reg .b16 c, a, b;\n\t.reg .b32 h;\n\t"
      "cvt.u16.u32 c, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 h, c;\n\t"
      "mov.b32 {a, b}, h;\n\t"
      "cvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(pair));
}

// One E4M3 term of 8 scaled activations u (codes packed little-endian into
// w0, w1); u becomes the residual times 16, the next term's input (exact:
// |residual| <= half an E4M3 step of u, and times 16 stays below 448).
__device__ __forceinline__ void tm8_encode_term(float (&u)[8], uint32_t &w0, uint32_t &w1) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t c01 = f32x2_to_e4m3x2(u[4 * h + 0], u[4 * h + 1]);
    const uint32_t c23 = f32x2_to_e4m3x2(u[4 * h + 2], u[4 * h + 3]);
    w[h] = c01 | (c23 << 16);
    float d0, d1, d2, d3;
    e4m3x2_to_f32(c01, d0, d1);
    e4m3x2_to_f32(c23, d2, d3);
    u[4 * h + 0] = (u[4 * h + 0] - d0) * 16.f;
    u[4 * h + 1] = (u[4 * h + 1] - d1) * 16.f;
    u[4 * h + 2] = (u[4 * h + 2] - d2) * 16.f;
    u[4 * h + 3] = (u[4 * h + 3] - d3) * 16.f;
  }
  w0 = w[0];
  w1 = w[1];
}

struct Tm8PrepParams {
  const uint16_t *x;      // [B][K] bf16
  const uint16_t *gamma;  // [K] bf16 or nullptr (no RMSNorm; then kslices may exceed 1)
  uint8_t *terms;         // [ntiles][T * bnp][128] E4M3 codes
  float *fac;             // [kslices][bnp]: f_b of each reduction slice (0 for padding tokens)
  int B, K, bnp, T, ntiles;
  int kslices;            // the main kernel's reduction slices: one scale per token and slice
  float eps;
  unsigned *err;          // device status block (checked builds)
};

// One CTA per token slot b = blockIdx.x and reduction slice blockIdx.y,
// one pass over the slice's part of x: thread t holds chunks c = c_lo + t +
// TM8_PREP_THREADS * i (8 elements each) in registers for i < TM8_PREP_CPT
// and re-reads any further ones.  max |v| and sum x^2 in a
// fixed order (each thread chains its chunks, i then e ascending; a xor
// butterfly per warp; the warps in order), then the T term codes of every
// chunk (zeros past K and for b >= B).  Defined in the one file that
// instantiates the kernels.
#ifdef DFK_TF8MMA_KERNELS
__device__ __forceinline__ void tm8_load_chunk(const Tm8PrepParams &p, int b, int c, uint4 &xv,
                                               uint4 &gv) {
  xv = gv = make_uint4(0u, 0u, 0u, 0u);
  if (!DFK_IN_BOUNDS(b < p.B && 8 * c + 8 <= p.K, 13, p.err)) return;
  xv = ld_nc_v4(p.x + static_cast<size_t>(b) * p.K + 8 * c);
  gv = p.gamma ? ld_nc_v4(p.gamma + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
}

// v = x (or x * gamma, exact in fp32) of one chunk
__device__ __forceinline__ void tm8_chunk_values(const Tm8PrepParams &p, const uint4 &xv,
                                                 const uint4 &gv, float (&v)[8]) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float x0 = bf16_lo(xw[u]), x1 = bf16_hi(xw[u]);
    v[2 * u] = p.gamma ? x0 * bf16_lo(gw[u]) : x0;
    v[2 * u + 1] = p.gamma ? x1 * bf16_hi(gw[u]) : x1;
  }
}

__device__ __forceinline__ void tm8_chunk_stats(const uint4 &xv, const float (&v)[8], float &mx,
                                                float &ss) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float x0 = bf16_lo(xw[u]), x1 = bf16_hi(xw[u]);
    ss = fmaf(x0, x0, ss);
    ss = fmaf(x1, x1, ss);
    mx = fmaxf(mx, fmaxf(fabsf(v[2 * u]), fabsf(v[2 * u + 1])));
  }
}

// The T term codes of one chunk (u = v * 2^e, already scaled) at k = 8 c.
__device__ __forceinline__ void tm8_write_terms(const Tm8PrepParams &p, int b, int c,
                                                float (&u)[8]) {
  const int k = 8 * c, tile = k / TM8_TILE_K, kk = k % TM8_TILE_K;
  const int rows = p.T * p.bnp;
  for (int t = 0; t < p.T; ++t) {
    uint32_t w0, w1;
    if (t + 1 < p.T) {
      tm8_encode_term(u, w0, w1);
    } else {  // the last term: no residual needed
      w0 = f32x2_to_e4m3x2(u[0], u[1]) | (f32x2_to_e4m3x2(u[2], u[3]) << 16);
      w1 = f32x2_to_e4m3x2(u[4], u[5]) | (f32x2_to_e4m3x2(u[6], u[7]) << 16);
    }
    if (!DFK_IN_BOUNDS(tile < p.ntiles && b < p.bnp, 14, p.err)) return;
    uint8_t *dst = p.terms + (static_cast<size_t>(tile) * rows + t * p.bnp + b) * TM8_TILE_K + kk;
    *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
  }
}

// At most 64 registers a thread: a prep CTA must fit in the register file
// beside one CTA of the main kernel (192 threads x 128 registers).
__global__ void __launch_bounds__(TM8_PREP_THREADS, 2) tf8mma_prep_kernel(const Tm8PrepParams p) {
  __shared__ float s_wmax[TM8_PREP_THREADS / 32], s_wss[TM8_PREP_THREADS / 32];
  __shared__ float s_scale;
  pdl_launch_dependents();
  pdl_wait();  // x comes from the previous kernel
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this CTA's range: the 128-wide k tiles of reduction slice blockIdx.y, as
  // the main kernel splits them (the whole of K without a split)
  const int slc = blockIdx.y;
  const int c_lo = ((slc * p.ntiles) / p.kslices) * (TM8_TILE_K / 8);
  const int nchunk = (((slc + 1) * p.ntiles) / p.kslices) * (TM8_TILE_K / 8);  // range end,
                                                                                // padding incl.
  const int kchunks = min(nchunk, p.K / 8);  // end of the chunks inside K
  float *fac = p.fac + static_cast<size_t>(slc) * p.bnp + b;
  constexpr int NT = TM8_PREP_THREADS, CPT = TM8_PREP_CPT;
  if (b >= p.B) {  // padding token slot: zero codes, zero factor
    float z[8];
    for (int c = c_lo + tid; c < nchunk; c += NT) {
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = 0.f;
      tm8_write_terms(p, b, c, z);
    }
    if (tid == 0) *fac = 0.f;
    return;
  }
  uint4 xr[CPT], gr[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) {  // every load issued before any use
    const int c = c_lo + tid + NT * i;
    xr[i] = gr[i] = make_uint4(0u, 0u, 0u, 0u);
    if (c < kchunks) tm8_load_chunk(p, b, c, xr[i], gr[i]);
  }
  float mx = 0.f, ss = 0.f;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    float v[8];
    tm8_chunk_values(p, xr[i], gr[i], v);
    tm8_chunk_stats(xr[i], v, mx, ss);
  }
  for (int c = c_lo + tid + NT * CPT; c < kchunks; c += NT) {
    uint4 xv, gv;
    tm8_load_chunk(p, b, c, xv, gv);
    float v[8];
    tm8_chunk_values(p, xv, gv, v);
    tm8_chunk_stats(xv, v, mx, ss);
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    ss += __shfl_xor_sync(0xffffffffu, ss, m);
  }
  if (lane == 0) {
    s_wmax[warp] = mx;
    s_wss[warp] = ss;
  }
  __syncthreads();
  if (tid == 0) {
    float m = 0.f, t = 0.f;
    for (int w = 0; w < NT / 32; ++w) {
      m = fmaxf(m, s_wmax[w]);
      t += s_wss[w];
    }
    int e = 0;
    if (m > 0.f) {
      int E;
      frexpf(m, &E);                   // m = f * 2^E, f in [0.5, 1)
      e = min(max(8 - E, -126), 126);  // m * 2^e in [128, 256)
    }
    s_scale = ldexpf(1.0f, e);
    const float r = p.gamma ? 1.0f / sqrtf(t / static_cast<float>(p.K) + p.eps) : 1.0f;
    *fac = r * ldexpf(1.0f, -e);
  }
  __syncthreads();
  const float sc = s_scale;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = c_lo + tid + NT * i;
    if (c < nchunk) {
      float u[8];
      tm8_chunk_values(p, xr[i], gr[i], u);  // zeros past K
#pragma unroll
      for (int q = 0; q < 8; ++q) u[q] *= sc;
      tm8_write_terms(p, b, c, u);
    }
  }
  for (int c = c_lo + tid + NT * CPT; c < nchunk; c += NT) {
    uint4 xv = make_uint4(0u, 0u, 0u, 0u), gv = make_uint4(0u, 0u, 0u, 0u);
    if (c < kchunks) tm8_load_chunk(p, b, c, xv, gv);
    float u[8];
    tm8_chunk_values(p, xv, gv, u);
#pragma unroll
    for (int q = 0; q < 8; ++q) u[q] *= sc;
    tm8_write_terms(p, b, c, u);
  }
}
#endif  // DFK_TF8MMA_KERNELS

struct Tm8Params {
  uint16_t *out;          // [B][N] bf16
  const float *scale[2];  // per-row scales [N]
  const float *fac;       // [kslices][bnp] factors f_b of each slice (prep kernel)
  unsigned *err;
  int B, K, N;
  int rbase, rextra, hmax, r8;
  int bnp, T, np;         // tokens per term block, terms, np = T * bnp (the MMA's N)
  int nt;                 // 128-wide k tiles per ring stage (1 or 2)
  int stages, stage_bytes, a8_bytes;  // a8_bytes: code bytes of one tile (NMAT * r8 * 128)
  int tmem_cols;
  int bar_off;
  int ntiles, kslices, nblocks;
  float *part;            // split-K partial sums [kslices][nblocks][bnp][128]
  unsigned *counters;     // [nblocks]
  int term_off;           // prep terms: offset of the term tiles within a stage;
                          // in-kernel terms: offset of the resident term area
                          // ([tiles of this CTA][np rows][128], after the ring)
  const uint16_t *x;      // in-kernel terms: [B][K] bf16 activations
  const uint16_t *gamma;  // in-kernel terms: [K] bf16, or nullptr (no RMSNorm)
  float eps;
};

// w[m][0]: codes of matrix m, box {128, hmax}; w[m][1]: box {128, hmax - 1};
// x: the term codes [ntiles * np][128], box {128, np} (prep terms only).
// 128-byte swizzle.
struct Tm8Maps {
  CUtensorMap w[2][2];
  CUtensorMap x;
};

// IBP > 0: in-kernel terms, no prep kernel.  IBP token slots (4, 8 or 16)
// and IT terms per token (IR = IBP * IT = 16 or 32 MMA columns).  Warps
// 6..13 wait for the previous kernel, read this CTA's k range of x once,
// derive each token's scale 2^e_b (and r_b) from it, and write the terms of
// the whole range into a resident shared-memory area (128-byte swizzle, as
// TMA would write them), then release it to the MMA thread (tready).  The
// TMA ring carries only the weight codes, so the producer never waits for
// the previous kernel.  With a k split each slice's partial sums are scaled
// by the slice's own 2^-e before they are added.
template <int NMAT, int IBP, int IT>
__global__ void __launch_bounds__(IBP > 0 ? TM8_INK_THREADS : TM8_THREADS, 1)
    tf8mma_kernel(const __grid_constant__ Tm8Maps maps, const Tm8Params p) {
  static_assert(NMAT == 1 || NMAT == 2, "NMAT");
  constexpr bool INK = IBP > 0;
  constexpr int IR = IBP * IT;  // B-operand rows / TMEM columns per matrix (INK)
  static_assert(!INK || (IR == 16 || IR == 32), "in-kernel terms: 16 or 32 MMA columns");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.stages, NP = p.np;

  uint64_t *fullb = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = fullb + S;
  uint64_t *accfull = empty + S;
  uint64_t *tready = accfull + 1;  // INK: the resident term area is written
  uint64_t *bend = tready + 1;
  volatile int *s_abort = reinterpret_cast<volatile int *>(bend);
  int *s_issued = reinterpret_cast<int *>(bend) + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bend) + 2;
  volatile int *s_last = reinterpret_cast<volatile int *>(bend) + 3;
  float *s_fac = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bend) + 16);  // [16]
  float *s_sc = s_fac + 16;                                                             // [16]
  float *s_rmx = s_sc + 16, *s_rss = s_rmx + 8;  // per-warp partials of the term warps

  const int cta = blockIdx.x;
  const int blk = cta / p.kslices, slc = cta - blk * p.kslices;
  const int j0 = blk * p.rbase + min(blk, p.rextra);
  const int r = p.rbase + (blk < p.rextra ? 1 : 0);
  const int mi = (r == p.hmax) ? 0 : 1;
  const int tile0 = (slc * p.ntiles) / p.kslices;
  const int tile1 = ((slc + 1) * p.ntiles) / p.kslices;
  const int NT = p.nt;
  const int nsteps = (tile1 - tile0 + NT - 1) / NT;
  // stage layout: code tiles [tt][m] (r8 rows each), then (prep terms) the
  // term tiles [tt] (np rows)

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullb[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(tready, TM8_XF_THREADS);
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
    // ================= TMA producer (one lane): codes; the term tiles (prep
    // terms) only after the prep kernel's results are visible
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_normal();
      const int S0 = min(S, nsteps);
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S;
        if (i >= S && !mbar_wait_bounded(&empty[st], ((i / S) - 1) & 1, s_abort, p.err)) break;
        uint8_t *sb = smem + static_cast<size_t>(st) * p.stage_bytes;
        const int nv = min(NT, tile1 - (tile0 + i * NT));  // k tiles of this stage
        mbar_arrive_expect_tx(&fullb[st],
                              static_cast<uint32_t>(nv * (NMAT * r + (INK ? 0 : NP)) * 128));
        for (int tt = 0; tt < nv; ++tt) {
          const int tile = tile0 + i * NT + tt;
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
            tma_load_2d(sb + tt * p.a8_bytes + m * p.r8 * 128, &maps.w[m][mi], &fullb[st],
                        tile * TM8_TILE_K, j0, pol_w);
          if (!INK && i >= S0)
            tma_load_2d(sb + p.term_off + tt * NP * 128, &maps.x, &fullb[st], 0, tile * NP,
                        pol_x);
        }
        if (!INK && i == S0 - 1) {
          pdl_wait();
          for (int ii = 0; ii < S0; ++ii) {
            const int nvi = min(NT, tile1 - (tile0 + ii * NT));
            for (int tt = 0; tt < nvi; ++tt)
              tma_load_2d(smem + static_cast<size_t>(ii) * p.stage_bytes + p.term_off +
                              tt * NP * 128,
                          &maps.x, &fullb[ii], 0, (tile0 + ii * NT + tt) * NP, pol_x);
          }
        }
        issued = i + 1;
      }
      *s_issued = issued;
    }
  } else if (warp == 1) {
    // ================= MMA issuer: per tile and matrix, 4 MMAs of K = 32
    // (32 bytes further into each swizzled 128-byte row).  The whole warp
    // walks the ring (warp-uniform descriptors); one elected lane issues.
    __syncwarp();
    const uint32_t leader = elect_one_sync();
    {
      const uint32_t idesc = umma_idesc_e4m3_f32(128, INK ? IR : NP);
      const uint64_t desc0 = umma_desc_sw128(sbase);
      const uint32_t tile_enc = static_cast<uint32_t>(p.r8 * 128) >> 4;
      const uint32_t a_enc = static_cast<uint32_t>(p.a8_bytes) >> 4;
      const uint32_t x_enc = static_cast<uint32_t>(p.term_off) >> 4;
      const uint32_t xt_enc = static_cast<uint32_t>((INK ? IR : NP) * 128) >> 4;
      bool ok = !INK || mbar_wait_bounded(tready, 0, s_abort, p.err);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
      for (int i = 0; ok && i < nsteps; ++i) {
        const int st = i % S;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&fullb[st], (i / S) & 1, s_abort, p.err)))
          break;
        tc_fence_after();
        const uint64_t ds = desc0 + (static_cast<uint32_t>(st * p.stage_bytes) >> 4);
        const int nv = min(NT, tile1 - (tile0 + i * NT));
        for (int tt = 0; tt < nv; ++tt) {
          // B operand: this stage's term tile, or the resident one of the tile
          const uint64_t bx = INK ? desc0 + x_enc + (i * NT + tt) * xt_enc
                                  : ds + x_enc + tt * xt_enc;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              if (leader)
                umma_e4m3(tmem + static_cast<uint32_t>(m * (INK ? IR : NP)),
                          ds + tt * a_enc + m * tile_enc + 2 * kk, bx + 2 * kk, idesc,
                          (i > 0 || tt > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (leader) umma_commit(&empty[st]);
        __syncwarp();
      }
      if (leader) umma_commit(accfull);
    }
  } else if (warp < 6) {
    // ================= epilogue (warps 2..5, one per TMEM lane quarter)
    const int et = tid - 64;
    const int q = warp & 3;
    const int row = 32 * q + lane;
    if (INK) named_barrier(4, 128 + TM8_XF_THREADS);  // the term warps' s_fac is written
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
      const int cstep = INK ? IBP : 16;  // token slots per pass
      for (int c = 0; c < p.bnp; c += cstep) {
        // terms combined smallest first: S = D_0 + (D_1 + (...) / 16) / 16
        float g[16], u[16];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          float acc[16];
          if constexpr (INK) {
            // columns t * IBP + b of this matrix (IR = 16 or 32; the loops
            // unroll, so every index is a constant)
            float d0[16], d1[16];
            tmem_ld_32x32b_x16(base + m * IR, d0);
            if constexpr (IR == 32) tmem_ld_32x32b_x16(base + m * IR + 16, d1);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (e < IBP) {
                constexpr int top = (IT - 1) * IBP;
                float a = (top + e < 16) ? d0[(top + e) & 15] : d1[(top + e) & 15];
#pragma unroll
                for (int t = IT - 2; t >= 0; --t) {
                  const int col = t * IBP + e;
                  a = ((col < 16) ? d0[col & 15] : d1[col & 15]) + a * 0.0625f;
                }
                acc[e] = a;
              } else {
                acc[e] = 0.f;
              }
            }
          } else {
            for (int t = p.T - 1; t >= 0; --t) {
              float d[16];
              tmem_ld_32x32b_x16(base + m * NP + t * p.bnp + c, d);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) acc[e] = (t == p.T - 1) ? d[e] : d[e] + acc[e] * 0.0625f;
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            if (m == 0) g[e] = acc[e];
            else u[e] = acc[e];
          }
        }
        if (p.kslices > 1) {
          // in-kernel terms: each slice's partial sums at their true scale
          // (times the slice's 2^-e_b; exact)
          float *mine = p.part + (static_cast<size_t>(slc) * p.nblocks + blk) * p.bnp * 128;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (e < cstep)
              mine[(c + e) * 128 + row] =
                  g[e] * (INK ? s_fac[c + e]
                              : __ldg(p.fac + static_cast<size_t>(slc) * p.bnp + c + e));
        } else if (row < r) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int n = c + e;
            if (e < cstep && n < p.B) {
              const float f = INK ? s_fac[n] : __ldg(p.fac + n);
              float res;
              if (NMAT == 2) {
                const float a = (g[e] * f) * sg, uu = (u[e] * f) * su;
                res = (a / (1.0f + expf(-a))) * uu;
              } else {
                res = (g[e] * f) * sg;
              }
              if (DFK_IN_BOUNDS(j < p.N, 11, p.err))
                p.out[static_cast<size_t>(n) * p.N + j] = f32_to_bf16_bits(res);
            }
          }
        }
      }
    }
    if (p.kslices > 1) {
      // every CTA of the row block takes part in the count (also after an
      // abort); the last one adds the slices in order, scales and stores
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
          splitk_reduce_row(p.part, p.kslices, p.nblocks, blk, p.bnp, p.B, row,
                            [&](int n, float acc) {
                              if (DFK_IN_BOUNDS(n < p.B && j0 + row < p.N, 12, p.err))
                              p.out[static_cast<size_t>(n) * p.N + j0 + row] =
                                  f32_to_bf16_bits(acc * sd);
                            });
        }
        named_barrier(2, 128);
        if (et == 0) p.counters[blk] = 0u;
      }
    }
    tc_fence_before();
  } else if (INK) {
    // ================= activation terms (warps 6..13)
    const int xt = tid - TM8_THREADS;  // 0 .. 255
    // the B real token slots share the 256 threads: tpt per slot (256 .. 16)
    const int bp = p.B <= 1 ? 1 : (p.B <= 2 ? 2 : (p.B <= 4 ? 4 : (p.B <= 8 ? 8 : 16)));
    const int tpt = TM8_XF_THREADS / bp;
    const int tok = xt / tpt, sub = xt % tpt;
    const int c_lo = tile0 * (TM8_TILE_K / 8);   // first 8-element chunk of this CTA's range
    const int c_end = tile1 * (TM8_TILE_K / 8);  // past its last chunk (whole tiles)
    const int c_k = min(c_end, p.K / 8);         // chunks inside K
    const bool real = tok < p.B;
    const uint16_t *xr = p.x + static_cast<size_t>(real ? tok : 0) * p.K;
    uint8_t *tarea = smem + p.term_off;
    // chunk c of token slot tok: values v (x, or x * gamma: exact in fp32)
    auto load = [&](int c, uint4 &xv, uint4 &gv) {
      xv = gv = make_uint4(0u, 0u, 0u, 0u);
      if (real && c < c_k) {
        xv = ld_nc_v4(xr + 8 * c);
        if (p.gamma) gv = ld_nc_v4(p.gamma + 8 * c);
      }
    };
    auto values = [&](const uint4 &xv, const uint4 &gv, float (&v)[8]) {
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float x0 = bf16_lo(xw[h]), x1 = bf16_hi(xw[h]);
        v[2 * h] = p.gamma ? x0 * bf16_lo(gw[h]) : x0;
        v[2 * h + 1] = p.gamma ? x1 * bf16_hi(gw[h]) : x1;
      }
    };
    float mx = 0.f, ss = 0.f;
    auto stats = [&](const uint4 &xv, const uint4 &gv) {
      float v[8];
      values(xv, gv, v);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float x0 = bf16_lo(xw[h]), x1 = bf16_hi(xw[h]);
        ss = fmaf(x0, x0, ss);
        ss = fmaf(x1, x1, ss);
        mx = fmaxf(mx, fmaxf(fabsf(v[2 * h]), fabsf(v[2 * h + 1])));
      }
    };
    // the IT term codes of chunk c into the resident area: tile (c - c_lo) / 16,
    // rows t * IBP + tok, 16-byte granule (chunk / 2) xor (row % 8) (128-byte
    // swizzle)
    auto emit = [&](int c, const uint4 &xv, const uint4 &gv, float scb) {
      float u[8];
      values(xv, gv, u);
#pragma unroll
      for (int h = 0; h < 8; ++h) u[h] *= scb;
      const int kl = 8 * (c - c_lo), jc = (kl & (TM8_TILE_K - 1)) >> 3;
      uint8_t *tb = tarea + (kl / TM8_TILE_K) * IR * 128;
#pragma unroll
      for (int t = 0; t < IT; ++t) {
        uint32_t w0, w1;
        if (t + 1 < IT) {
          tm8_encode_term(u, w0, w1);
        } else {  // the last term: no residual needed
          w0 = f32x2_to_e4m3x2(u[0], u[1]) | (f32x2_to_e4m3x2(u[2], u[3]) << 16);
          w1 = f32x2_to_e4m3x2(u[4], u[5]) | (f32x2_to_e4m3x2(u[6], u[7]) << 16);
        }
        const int rw = t * IBP + tok;
        *reinterpret_cast<uint2 *>(tb + rw * 128 + (((jc >> 1) ^ (rw & 7)) << 4) + ((jc & 1) << 3)) =
            make_uint2(w0, w1);
      }
    };
    // rows of the slots past B are zero in every tile (no conversion needed)
    {
      const int ntl = tile1 - tile0, zrows = IBP - p.B;
      constexpr int ITS = IT > 0 ? IT : 1;
      const int nz = ntl * ITS * zrows * 8;  // 16-byte stores
      for (int z = xt; z < nz; z += TM8_XF_THREADS) {
        const int g = z & 7, rz = (z >> 3) % zrows, rest = (z >> 3) / zrows;
        const int t = rest % ITS, tl = rest / ITS;
        *reinterpret_cast<uint4 *>(tarea + tl * IR * 128 + (t * IBP + p.B + rz) * 128 + 16 * g) =
            make_uint4(0u, 0u, 0u, 0u);
      }
    }
    pdl_wait();  // x comes from the previous kernel
    // pass 1: max |v| and sum x^2 of slot tok over [c_lo, c_k); the thread
    // chains its chunks c = c_lo + sub + tpt * i (i, then the 8 elements,
    // ascending)
    constexpr int W = 8;  // chunks per thread in flight
    const bool one = (c_end - c_lo) <= tpt * W;  // the whole range in one window
    uint4 xv[W], gv[W];
    for (int c0 = c_lo + sub; real && c0 < c_end; c0 += tpt * W) {
#pragma unroll
      for (int u = 0; u < W; ++u) load(c0 + tpt * u, xv[u], gv[u]);
#pragma unroll
      for (int u = 0; u < W; ++u) stats(xv[u], gv[u]);
    }
    // combine the tpt threads of the slot: xor butterfly inside the warp (or
    // half warp), then the slot's warps in order
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      if (m < tpt) {  // tpt >= 16: warp-uniform
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
        ss += __shfl_xor_sync(0xffffffffu, ss, m);
      }
    }
    if (tpt > 32) {
      const int w = xt >> 5;
      if (lane == 0) {
        s_rmx[w] = mx;
        s_rss[w] = ss;
      }
      named_barrier(5, TM8_XF_THREADS);
      const int nw = tpt >> 5, w0 = tok * nw;
      mx = s_rmx[w0];
      ss = s_rss[w0];
      for (int q = 1; q < nw; ++q) {
        mx = fmaxf(mx, s_rmx[w0 + q]);
        ss += s_rss[w0 + q];
      }
    }
    if (sub == 0) {
      int e = 0;
      if (mx > 0.f) {
        int E;
        frexpf(mx, &E);                  // mx = f * 2^E, f in [0.5, 1)
        e = min(max(8 - E, -126), 126);  // mx * 2^e in [128, 256)
      }
      s_sc[tok] = ldexpf(1.0f, e);
      const float rr = p.gamma ? 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps) : 1.0f;
      s_fac[tok] = real ? rr * ldexpf(1.0f, -e) : 0.f;
    }
    if (xt < IBP && xt >= bp) s_fac[xt] = 0.f;  // slots no thread group covers
    named_barrier(5, TM8_XF_THREADS);
    const float scb = s_sc[tok];
    // pass 2: the terms of the real slots (from the registers when the range
    // fit in one window)
    if (real) {
      if (one) {
        // term by term over the thread's chunks: the loop over the terms stays
        // rolled, so the conversion is one short stretch of code
        float uu[W][8];
#pragma unroll
        for (int u = 0; u < W; ++u) {
          values(xv[u], gv[u], uu[u]);
#pragma unroll
          for (int h = 0; h < 8; ++h) uu[u][h] *= scb;
        }
#pragma unroll 1
        for (int t = 0; t < IT; ++t) {
          const int rw = t * IBP + tok;
#pragma unroll
          for (int u = 0; u < W; ++u) {
            const int c = c_lo + sub + tpt * u;
            if (c < c_end) {
              uint32_t w0, w1;
              tm8_encode_term(uu[u], w0, w1);  // (the last term's residual is not used)
              const int kl = 8 * (c - c_lo), jc = (kl & (TM8_TILE_K - 1)) >> 3;
              *reinterpret_cast<uint2 *>(tarea + (kl / TM8_TILE_K) * IR * 128 + rw * 128 +
                                         (((jc >> 1) ^ (rw & 7)) << 4) + ((jc & 1) << 3)) =
                  make_uint2(w0, w1);
            }
          }
        }
      } else {
        for (int c0 = c_lo + sub; c0 < c_end; c0 += tpt * W) {
#pragma unroll
          for (int u = 0; u < W; ++u) load(c0 + tpt * u, xv[u], gv[u]);
#pragma unroll
          for (int u = 0; u < W; ++u)
            if (c0 + tpt * u < c_end) emit(c0 + tpt * u, xv[u], gv[u], scb);
        }
      }
    }
    fence_proxy_async_smem();  // the MMA (async proxy) reads these shared-memory writes
    mbar_arrive(tready);
    named_barrier(4, 128 + TM8_XF_THREADS);  // with the epilogue warps: s_fac is written
  }

  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait_bounded(accfull, 0, nullptr, p.err);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if (tid == 0 && *s_abort) {
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
