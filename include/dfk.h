/*
 * dfk.h -- C ABI of libdfk.so, the B200 (sm_100a) decode-stage SwiGLU MLP.
 *
 * The method ("Deep Kernel Fusion for Transformer Decoding", episode
 * description; "Deep Kernel Fusion for Transformers", abstract): at decode
 * time the SwiGLU MLP is a weight-streaming, memory-bandwidth-bound
 * matrix-vector product.  The gate projection, the up projection, the SiLU
 * activation and the elementwise multiply run as ONE kernel, so the gate
 * and up activations never reach HBM; the down projection stays a separate
 * kernel; a profiler-driven runtime scheduler picks among row-major and
 * column-major kernel variants.  The RMSNorm that precedes the MLP can be
 * fused in front of the gate/up projection (GPULlama3.java PR #78, the
 * `rms_ffn_gate_up` task).
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE memory (unless a function says host),
 *     contiguous, bf16 (IEEE binary32 upper halves) unless noted.
 *   - x is [B][d_model] row-major; h is [B][d_ff]; y is [B][d_model].
 *   - Every device pointer must be 16-byte aligned; d_model % 8 == 0; for the
 *     column-major layout also d_ff % 8 == 0.  Violations return
 *     DFK_ERR_MISALIGNED / DFK_ERR_UNSUPPORTED_SHAPE without launching.
 *   - 0 <= B <= 64 (decode batch).  B == 0 is a no-op returning DFK_OK.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: the return code covers argument validation and
 *     launch errors only; a device-side failure (a pipeline wait that gave
 *     up) is recorded in a device error word read by dfk_device_error().
 *   - `variant` = 0 lets the scheduler choose (timed on first use for the
 *     shape, cached; never timed while the stream is being captured);
 *     a positive id forces that variant (dfk_variant_info lists them).
 *   - Accumulation is fp32; every output is rounded once to bf16
 *     (round-to-nearest-even).  CUDA-core variants of one operation give
 *     bit-identical results for every layout, tile and pipeline choice and
 *     for every batch size (row b of the output depends on row b of x only).
 *   - There is no CPU fallback: without an sm_100 device every compute call
 *     returns DFK_ERR_ARCH (or DFK_ERR_CUDA).
 *   - Kernels start while the previous kernel in the stream finishes
 *     (programmatic dependent launch): they read the weights -- W_gate,
 *     W_up, W_down, FP8 codes and scales, gamma -- as soon as they start,
 *     and the activations (x, h) and their outputs only once the previous
 *     kernel's results are visible.  A weight must not be written by work
 *     still running in the same stream (order such writes with an event or
 *     a synchronisation, as loading weights normally does).
 *   - Thread-safe: the variant cache and descriptor cache are locked.
 */
#ifndef DFK_H
#define DFK_H

#if defined(__GNUC__)
#define DFK_API __attribute__((visibility("default")))
#else
#define DFK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dfk_status {
  DFK_OK = 0,
  DFK_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum, bad variant id */
  DFK_ERR_UNSUPPORTED_SHAPE = 2,  /* B > 64, d_model % 8, d_ff % 8 (column-major), too large */
  DFK_ERR_UNSUPPORTED_LAYOUT = 3, /* layout not valid for this entry point */
  DFK_ERR_MISALIGNED = 4,         /* a device pointer is not 16-byte aligned */
  DFK_ERR_CUDA = 5,               /* a CUDA runtime call failed; see dfk_last_error() */
  DFK_ERR_ARCH = 6,               /* no sm_100 device current */
  DFK_ERR_TIMEOUT = 7,            /* a kernel's pipeline wait gave up (dfk_device_error) */
  DFK_ERR_NO_VARIANT = 8,         /* no variant fits this shape (shared memory / threads) */
  DFK_ERR_BOUNDS = 9              /* checked build: a kernel's bounds check failed
                                     (dfk_device_error; the access was skipped)      */
} dfk_status;

/* Storage of W_gate / W_up (as stated in the pages: W_gate, W_up are [d_ff, d_model]). */
typedef enum dfk_wlayout {
  DFK_W_ROW_MAJOR = 0,      /* w_gate, w_up: [d_ff][d_model] each                        */
  DFK_W_COL_MAJOR = 1,      /* w_gate, w_up: [d_model][d_ff] each (the transposes)       */
  DFK_W_GU_INTERLEAVED = 2, /* w_gate: [d_ff][2][d_model], [j][0] = gate row j,
                               [j][1] = up row j; w_up must be NULL                      */
  DFK_W_ANY = -1            /* dfk_select_variant only: time every layout               */
} dfk_wlayout;

typedef enum dfk_op {
  DFK_OP_GATE_UP = 0,         /* dfk_swiglu_gate_up          */
  DFK_OP_RMSNORM_GATE_UP = 1, /* dfk_rmsnorm_swiglu_gate_up  */
  DFK_OP_DOWN = 2,            /* dfk_down_proj               */
  DFK_OP_GATE_UP_FP8 = 3,     /* dfk_swiglu_gate_up_fp8      */
  DFK_OP_RMSNORM_GATE_UP_FP8 = 4, /* dfk_rmsnorm_swiglu_gate_up_fp8 */
  DFK_OP_DOWN_FP8 = 5,        /* dfk_down_proj_fp8           */
  DFK_OP_QKV = 6,             /* dfk_rmsnorm_qkv_proj, gamma == NULL */
  DFK_OP_RMSNORM_QKV = 7      /* dfk_rmsnorm_qkv_proj with RMSNorm   */
} dfk_op;

typedef enum dfk_family {
  DFK_FAMILY_CUDA_CORE = 0,   /* TMA-fed shared-memory ring, fp32 FMA on CUDA cores   */
  DFK_FAMILY_TENSOR_CORE = 1  /* tcgen05 MMA with TMEM accumulators                    */
} dfk_family;

typedef struct dfk_variant {
  int variant_id;   /* id accepted by the `variant` arguments                        */
  int op;           /* dfk_op                                                         */
  int layout;       /* dfk_wlayout the variant reads                                 */
  int family;       /* dfk_family                                                    */
  int j_per_thread; /* output columns per thread (CUDA-core)                         */
  int token_tile;   /* tokens per pass over the weights                              */
  int k_split;      /* thread teams splitting the reduction dimension               */
  int k_tiles_per_stage; /* consecutive 64-wide reduction tiles per ring stage       */
  int acc_banks;    /* tensor core: independent TMEM accumulators per output        */
  int paired_fma;   /* CUDA core: 1 = FMAs issued two at a time (fma.rn.f32x2)      */
  int full_m_tiles; /* tensor core: 1 = each CTA owns 128 output rows (full MMA M) */
  int stages;       /* ring stages used at the queried shape (0 = not resolved)      */
  float measured_us;/* median timed duration; < 0 when chosen without timing        */
  int e4m3_mma;     /* tensor core, FP8 weights only: E4M3 MMA on the codes
                       (kind::f8f6f4, activations as E4M3 terms); 1 = terms
                       written by a prep kernel, 2 = derived inside the kernel
                       (up to 16 tokens); dfk_variant_info reports these under
                       the FP8 ops                                               */
} dfk_variant;

/*
 * h = SiLU(x . W_gate^T) (*) (x . W_up^T)      -- the fused gate/up kernel
 * ("Deep Kernel Fusion for Transformer Decoding", episode description: the
 * up projection, gate projection, SiLU and elementwise multiply fused into
 * one decode kernel).
 *   x       [B][d_model] bf16, device
 *   w_gate  per `layout` (dfk_wlayout), bf16, device
 *   w_up    per `layout`; NULL for DFK_W_GU_INTERLEAVED
 *   h       [B][d_ff] bf16, device, written once
 * SiLU(a) = a / (1 + exp(-a)), applied to the gate branch.
 */
DFK_API int dfk_swiglu_gate_up(const void *x, const void *w_gate, const void *w_up, int layout,
                       void *h, int B, int d_model, int d_ff, int variant, void *stream);

/*
 * Same, with the RMSNorm fused in front (GPULlama3.java PR #78, the
 * `rms_ffn_gate_up` task):
 *   xn[b][k] = x[b][k] * r_b * gamma[k],
 *   r_b = 1 / sqrt( (1/d_model) * sum_k x[b][k]^2 + eps ),
 * then h = SiLU(xn . W_gate^T) (*) (xn . W_up^T).  xn is not rounded to
 * bf16: the CUDA-core kernels keep (x * r_b) * gamma in fp32 in shared
 * memory; the tensor-core kernels split the exact x * gamma into bf16
 * hi + lo MMA operands and apply r_b to the fp32 sums.  xn never reaches
 * HBM.  gamma [d_model] bf16, device.  eps >= 0.
 */
DFK_API int dfk_rmsnorm_swiglu_gate_up(const void *x, const void *gamma, float eps,
                               const void *w_gate, const void *w_up, int layout,
                               void *h, int B, int d_model, int d_ff, int variant,
                               void *stream);

/*
 * y = h . W_down^T, the separate down projection ("Deep Kernel Fusion for
 * Transformer Decoding", episode description: the down projection is left
 * out of the fused kernel).
 *   h       [B][d_ff] bf16, device
 *   w_down  [d_model][d_ff] bf16 row-major, device
 *   y       [B][d_model] bf16, device
 */
DFK_API int dfk_down_proj(const void *h, const void *w_down, void *y, int B, int d_model,
                  int d_ff, int variant, void *stream);

/*
 * y = h . W_down^T without allocating device memory.  (No counterpart in the
 * paper: this serves callers that cannot allocate while they run the MLP --
 * a runtime that has reserved all device memory for its own pool, code that
 * runs inside CUDA stream capture, where allocation calls are not allowed, or
 * a host that lends the library a device it does not own.)
 * Same arguments and result contract as dfk_down_proj; always the split-K
 * tensor-core kernel in a fixed configuration (no scheduler timing).  Its
 * partial sums live in a 6 MiB + 4 KiB array that is part of the library
 * image: every device that loads the library holds it until the process
 * exits.  The first call on a device looks up the array's device address
 * (make that call before any stream capture).  All calls share the array:
 * calls whose executions overlap on the GPU (different streams, or graphs
 * replayed concurrently) race and give wrong results.  A shape whose
 * partial sums exceed the array returns DFK_ERR_UNSUPPORTED_SHAPE.
 */
DFK_API int dfk_down_proj_static_scratch(const void *h, const void *w_down, void *y, int B,
                                         int d_model, int d_ff, void *stream);

/*
 * FP8 weight streaming: the same three operations with weights stored as
 * FP8 E4M3 codes and one fp32 scale per output row, dequantised inside the
 * matrix-vector product (GPULlama3.java PR #78, "fusing dequantize with
 * compute": no separate dequantise pass, no dequantised copy in memory).
 * The weights are half the bytes of bf16, and the decode path is bound by
 * reading them.
 *   W[j][k] = s[j] * E4M3(q[j][k])
 *   E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 *   subnormal (m * 2^-9); S.1111.111 is NaN; no infinities; max 448.
 *   q_gate, q_up  [d_ff][d_model] uint8 codes, row-major, device, 16-byte aligned
 *   s_gate, s_up  [d_ff] fp32, device, 4-byte aligned
 *   q_down        [d_model][d_ff] uint8 codes, row-major; s_down [d_model] fp32
 *   x, gamma, h, y, eps: as for the bf16 entry points.
 * Each code is widened to its exact fp32 value in registers; products and
 * sums are fp32 in a fixed order; the row's sum is multiplied by s[j] once
 * before SiLU and the bf16 rounding.  Variant families: CUDA-core variants
 * (fp32 FMA on the widened codes; at most two k tiles per stage); a
 * widening tensor-core kernel (the tensor-core ids with one k tile per stage
 * and rows spread over the SMs: codes widened to bf16 into TMEM, bf16 MMA
 * with fp32 accumulation); and the E4M3-MMA kernel (ids with e4m3_mma >= 1:
 * the codes feed the E4M3 tensor-core MMA directly, each token's activations
 * are written as E4M3 terms -- two for bf16 x, four for x * gamma, after a
 * power-of-two scale; exact for elements within 2^14 of the token's largest
 * magnitude, smaller ones carried to about 2^-21 of it, so a token spanning
 * more than 2^14 can land outside the bf16 path's accuracy and should use
 * the CUDA-core or widening ids -- either (e4m3_mma = 1) by a small kernel launched
 * before it, into a library-owned buffer per (device, stream) allocated at
 * first use outside stream capture, or (e4m3_mma = 2, B <= 16) inside the
 * kernel from each ring stage's raw activations; with a k split the latter
 * scales each slice's partial sums by the slice's own power of two).  Tensor-core kernels take at most 128 output rows per SM
 * (per SM / k_split for the down projection).  Other ids are rejected with
 * DFK_ERR_INVALID_ARG; E4M3-MMA ids are rejected by the bf16 entry points.
 * Constraints: row-major only; the reduction length (d_model for gate/up,
 * d_ff for the down projection) a multiple of 16; otherwise as for the bf16
 * entry points.
 */
DFK_API int dfk_swiglu_gate_up_fp8(const void *x, const void *q_gate, const float *s_gate,
                                   const void *q_up, const float *s_up, void *h, int B,
                                   int d_model, int d_ff, int variant, void *stream);

DFK_API int dfk_rmsnorm_swiglu_gate_up_fp8(const void *x, const void *gamma, float eps,
                                           const void *q_gate, const float *s_gate,
                                           const void *q_up, const float *s_up, void *h, int B,
                                           int d_model, int d_ff, int variant, void *stream);

DFK_API int dfk_down_proj_fp8(const void *h, const void *q_down, const float *s_down, void *y,
                              int B, int d_model, int d_ff, int variant, void *stream);

/*
 * RMSNorm + packed QKV projection ("Optimizing QKV Projection with Operator
 * Fusion", section "Implementing Fusion: Packed Projections": one wider
 * projection replaces the separate Q, K and V ones and its output is split;
 * the RMSNorm in front as the fusedRmsNormQKVMatmul task of GPULlama3.java
 * PR #78):
 *   xn = RMSNorm(x; gamma, eps) as for dfk_rmsnorm_swiglu_gate_up, or x when
 *        gamma is NULL;
 *   o[b][j] = sum_k xn[b][k] * w_qkv[j][k]  for j < n_q + n_k + n_v;
 *   q[b][j] = o[b][j], k[b][j] = o[b][n_q + j], v[b][j] = o[b][n_q + n_k + j].
 *   x      [B][d_model] bf16, device
 *   w_qkv  [n_q + n_k + n_v][d_model] bf16 row-major (W_q rows, then W_k,
 *          then W_v), device
 *   q, k, v  [B][n_q], [B][n_k], [B][n_v] bf16, device, each written once;
 *          a part of size 0 may be NULL
 * One weight stream for all three parts and every token; the normalised
 * activations never reach HBM.  Runs on the GEMV variants (variant 0 = the
 * scheduler's choice, timed per shape under DFK_OP_QKV / DFK_OP_RMSNORM_QKV;
 * for dfk_select_variant pass d_ff = n_q + n_k + n_v and a packed output).
 * Part sizes >= 0 with a positive sum; otherwise as for dfk_down_proj.
 */
DFK_API int dfk_rmsnorm_qkv_proj(const void *x, const void *gamma, float eps,
                                 const void *w_qkv, void *q, void *k, void *v, int B,
                                 int d_model, int n_q, int n_k, int n_v, int variant,
                                 void *stream);

/*
 * Profiler-driven variant choice ("Deep Kernel Fusion for Transformer
 * Decoding", episode description: runtime scheduling across row-major and
 * column-major kernel variants; "Deep Kernel Fusion for Transformers",
 * abstract: the kernel is paired with a kernel scheduler).
 * Times every feasible variant of `op` for (B, d_model, d_ff, layout) with
 * CUDA events (each sample: L2 flushed, then a burst of 4 back-to-back
 * launches -- or a single launch when one call's weights fit in L2; median
 * of DFK_TUNE_REPS samples), caches the fastest and
 * returns it in *out.  layout == DFK_W_ANY times every layout and reports
 * the fastest layout in out->layout (gate/up ops only).
 *   sample_ptrs  NULL, or the caller's buffers in argument order of the op:
 *                gate_up: {x, w_gate, w_up, h}; rmsnorm_gate_up: {x, gamma,
 *                w_gate, w_up, h}; down: {h, w_down, y}; the FP8 ops put
 *                each scale right after its codes: {x, q_gate, s_gate, q_up,
 *                s_up, h}, {x, gamma, q_gate, s_gate, q_up, s_up, h},
 *                {h, q_down, s_down, y}.  With NULL (or with
 *                DFK_W_ANY) the function allocates throwaway buffers on
 *                `stream` and frees them before returning.
 * Returns DFK_ERR_INVALID_ARG if the stream is being captured.
 * Environment: DFK_TUNE=0 disables timing (heuristic choice),
 * DFK_TUNE_REPS (default 7) sets the timed repetitions, DFK_LOG=1 logs
 * decisions to stderr, DFK_TUNE_CACHE=<file> persists timed decisions (a
 * text file keyed by device name, SM count and driver version; loaded on
 * first use, appended to after each new decision; lines that do not parse
 * are skipped with a warning on stderr), DFK_FAULT=tune makes timing fail
 * (the heuristic is used: a host-side fault injection for tests).
 */
DFK_API int dfk_select_variant(int op, int B, int d_model, int d_ff, int layout,
                       const void *const *sample_ptrs, void *stream, dfk_variant *out);

/* The scheduler's cached choice for (op, B, d_model, d_ff, layout) on the
 * current device: DFK_OK with *out filled, or DFK_ERR_NO_VARIANT when no
 * decision is cached yet (no call of that shape has been made). */
DFK_API int dfk_cached_variant(int op, int B, int d_model, int d_ff, int layout,
                               dfk_variant *out);

/* Number of variant ids (valid ids are 1..count) and their description. */
DFK_API int dfk_variant_count(void);
DFK_API int dfk_variant_info(int variant_id, dfk_variant *out);

/* Forget every cached scheduler decision (all devices). */
DFK_API void dfk_clear_variant_cache(void);

/* ---- one decode step of a layer stack in one launch ------------------------
 * The FlashFormer abstract (paper-listing page) puts a whole model's decode
 * step into one kernel for low-batch inference; here that is applied to a
 * stack of the fused MLP layers.  dfk_mlp_stack_step runs, in ONE persistent
 * kernel (one CTA per SM, a cooperative launch), for l = 0 .. layers-1:
 *   h_l = SiLU(xn_l . W_gate_l^T) (*) (xn_l . W_up_l^T),
 *         xn_l = RMSNorm(x_l; gamma_l, eps)      (as dfk_rmsnorm_swiglu_gate_up)
 *   y_l = h_l . W_down_l^T                       (as dfk_down_proj)
 *   x_{l+1} = y_l,   x_0 = x
 * and then x := y_{L-1} / sqrt(mean(y_{L-1}^2) + eps) per row (as
 * dfk_rms_rescale), in place, ready for the next step.  The weight stream
 * never stops at a layer boundary: each SM's producer streams the next
 * phase's weights while the previous phase finishes on the other SMs.
 *   gammas    [layers][d_model] bf16
 *   w_gate    [layers][d_ff][d_model] bf16 (layout DFK_W_ROW_MAJOR), or
 *             [layers][d_model][d_ff] (DFK_W_COL_MAJOR: the gate/up phases
 *             then take 128 columns per SM, as the column-major tensor-core
 *             kernel does); one allocation
 *   w_up      the same shape as w_gate
 *   w_down    [layers][d_model][d_ff]
 *   x         [B][d_model] bf16, read and overwritten with the next input
 *   h_all     [layers][B][d_ff] bf16, every layer's h (written)
 *   y_all     [layers][B][d_model] bf16, every layer's y (written)
 *   workspace dfk_mlp_stack_workspace_bytes(...) bytes of device memory,
 *             zeroed by the caller once before the first call and then
 *             left to the library (it holds the grid's phase counters);
 *             after a call that reported DFK_ERR_TIMEOUT, zero it again
 * The arithmetic is that of the separate kernels with the tensor-core
 * gate/up (in-kernel RMSNorm, 16 token slots) and the four-slice split-K
 * tensor-core down projection, so one call gives the same bits as those
 * 2 x layers + 1 launches (with the same weight layout).  Constraints: 1 <= B <= 16; d_model, d_ff
 * multiples of 8; d_ff <= 128 rows (or columns) per SM, d_model <= 128 rows
 * per four SMs (the Llama-3-8B shape fits); DFK_ERR_UNSUPPORTED_SHAPE
 * otherwise.  Any other layout: DFK_ERR_UNSUPPORTED_LAYOUT.
 * Calls on one workspace must not overlap on the GPU.  No allocation, so
 * the call can be captured in a CUDA graph.
 */
DFK_API long long dfk_mlp_stack_workspace_bytes(int layers, int B, int d_model, int d_ff);
DFK_API int dfk_mlp_stack_step(const void *gammas, float eps, const void *w_gate,
                               const void *w_up, int layout, const void *w_down, void *x,
                               void *h_all, void *y_all, void *workspace,
                               long long workspace_bytes, int layers, int B, int d_model,
                               int d_ff, void *stream);

/* ---- tensor-parallel MLP ---------------------------------------------------
 * "Deep Kernel Fusion for Transformers" (abstract) keeps the fused kernel
 * adaptable to inference configurations; on several GPUs the MLP shards
 * d_ff: rank r holds rows [f0_r, f1_r) of W_gate and W_up (whole gate/up
 * pairs, so the fused gate/up kernel runs unchanged on the shard and needs
 * no communication) and columns [f0_r, f1_r) of W_down, stored as its own
 * contiguous [d_model][f1_r - f0_r] matrix.  Each rank computes a partial
 * y_r = h_r . W_down_r^T; the full y is the sum over ranks.  The down
 * projection below does that sum inside the kernel: each CTA writes its
 * fp32 partial rows into every rank's receive buffer with plain stores to
 * peer memory (NVLink), raises a flag there, waits (bounded by the device's
 * wait limit) for every rank's flag of its rows, and adds the ranks'
 * partials in rank order 0, 1, ... -- so every rank computes the same bits
 * of bf16 y.  No library collective and no multicast load is involved.
 *
 * One process per GPU.  Setup, on every rank with its device current:
 *   dfk_tp_group_create(world, rank, max_B, d_model, &g, handle)
 *       allocates this rank's buffer (2 x world x max_B x d_model fp32 plus
 *       flags; zeroed) and writes its CUDA IPC handle into `handle`
 *       (DFK_TP_HANDLE_BYTES bytes, host memory);
 *   exchange the handles (e.g. an all-gather over torch.distributed);
 *   dfk_tp_group_connect(g, handles)  -- `handles` = world handles in rank
 *       order (host memory); maps every peer's buffer.
 * Then dfk_tp_down_proj_allreduce on every rank, in the same order of calls
 * on all ranks (a call waits for the same call on the other ranks; each
 * rank counts its calls on the device, so the call can be captured in a
 * CUDA graph).  h [B][d_ff_shard] and w_down_shard [d_model][d_ff_shard]
 * are this rank's, y [B][d_model] receives the full result; B <= max_B,
 * d_ff_shard % 8 == 0 (may differ between ranks), d_model as created.  If a
 * peer never arrives the wait gives up after the wait limit, y is not
 * written and dfk_device_error reports DFK_ERR_TIMEOUT.
 * dfk_tp_group_destroy synchronises the device and frees the buffer.
 * world = 1 is valid (no peers).
 */
#define DFK_TP_HANDLE_BYTES 64
typedef struct dfk_tp_group dfk_tp_group;

DFK_API int dfk_tp_group_create(int world, int rank, int max_B, int d_model,
                                dfk_tp_group **group, void *handle);
DFK_API int dfk_tp_group_connect(dfk_tp_group *group, const void *handles);
DFK_API int dfk_tp_down_proj_allreduce(dfk_tp_group *group, const void *h,
                                       const void *w_down_shard, void *y, int B, int d_model,
                                       int d_ff_shard, void *stream);
DFK_API int dfk_tp_group_destroy(dfk_tp_group *group);

/*
 * The same fused down projection and all-reduce for a group of `world`
 * ranks emulated on the current device: one cooperative grid computes every
 * rank's shard (its CTAs wait on one another's flags, so all of them must be
 * resident at once; shapes needing more CTAs than that are rejected with
 * DFK_ERR_UNSUPPORTED_SHAPE).  Runs the kernel code of the multi-GPU call on
 * one GPU.  h_all [world][B][d_ff_shard], w_all [world][d_model][d_ff_shard]
 * (rank r's shard at index r; equal shard sizes), y_all [world][B][d_model]
 * (every rank's copy of y).  The buffers for the emulated ranks are
 * allocated by the library on the first call per (device, world, d_model),
 * which must not be made during stream capture.
 */
DFK_API int dfk_tp_down_proj_allreduce_emulated(int world, const void *h_all,
                                                const void *w_all, void *y_all, int B,
                                                int d_model, int d_ff_shard, void *stream);

/* ---- building blocks of the unfused baseline and of the decode stack -------
 * These exist to measure what the fusion saves (separate RMSNorm, GEMV,
 * SiLU and multiply kernels with bf16 intermediates in HBM) and to run a
 * multi-layer decode loop; they are not part of the fused path. */

/* xn[b][k] = bf16(x[b][k] * r_b * gamma[k]), r_b as in the fused prologue. */
DFK_API int dfk_rmsnorm(const void *x, const void *gamma, float eps, void *xn, int B, int d,
                void *stream);

/* out[b][n] = bf16( sum_k x[b][k] * w[n][k] ), w [N][K] row-major bf16. */
DFK_API int dfk_gemv(const void *x, const void *w, void *out, int B, int K, int N, int variant,
             void *stream);

/* out[i] = bf16( SiLU(a[i]) ), n elements. */
DFK_API int dfk_silu(const void *a, void *out, long long n, void *stream);

/* out[i] = bf16( a[i] * b[i] ), n elements. */
DFK_API int dfk_mul(const void *a, const void *b, void *out, long long n, void *stream);

/* x_next[b][k] = bf16( y[b][k] / sqrt(mean_k y[b][k]^2 + eps) ). */
DFK_API int dfk_rms_rescale(const void *y, float eps, void *x_next, int B, int d, void *stream);

/*
 * One MLP layer end to end from HOST memory: copies x_host (pinned or
 * pageable, [B][d_model] bf16) to the device, runs the fused RMSNorm+gate/up
 * kernel (gamma may be NULL: no RMSNorm) and the down projection, and copies
 * y back to y_host ([B][d_model] bf16).  Weights are device-resident.
 * x_dev, h_dev, y_dev are caller-owned device work buffers of the sizes of
 * x, h and y.  Synchronises `stream` before returning.  Pinned host
 * buffers (device-addressable, 16-byte aligned): the copies are small
 * kernels chained to the MLP kernels by programmatic dependent launch, and
 * the whole sequence is captured once per argument set and replayed as one
 * CUDA graph; pageable buffers use copy-engine transfers, eagerly.
 */
DFK_API int dfk_mlp_forward_host(const void *x_host, const void *gamma, float eps,
                         const void *w_gate, const void *w_up, int layout,
                         const void *w_down, void *y_host, void *x_dev, void *h_dev,
                         void *y_dev, int B, int d_model, int d_ff, void *stream);

/* ---- status --------------------------------------------------------------- */

/* Static text for a dfk_status value. */
DFK_API const char *dfk_status_string(int status);

/* Text of the last error seen by this thread (CUDA error string or a
 * description of the rejected argument); "" when none. */
DFK_API const char *dfk_last_error(void);

/* Reads the current device's error word into *code and clears it
 * (0 = none; bit 0 = a pipeline wait gave up; bit 1 = a bounds check of the
 * checked build failed).  Synchronises the device.  Returns DFK_OK when the
 * word was 0, DFK_ERR_BOUNDS when bit 1 was set (dfk_last_error names the
 * first failing check), else DFK_ERR_TIMEOUT. */
DFK_API int dfk_device_error(int *code);

/*
 * Failure detection (no counterpart in the pages): every wait of a kernel's
 * pipeline on an mbarrier is bounded.  When a wait gives up the kernel sets
 * bit 0 of the device error word, stops issuing work, waits (with the
 * default limit) for its own copies and MMAs in flight, releases its tensor
 * memory and returns; the context stays usable and dfk_device_error reports
 * DFK_ERR_TIMEOUT.
 *
 * dfk_set_wait_limit sets the limit of the pipeline waits for kernels
 * launched afterwards on the current device: ns > 0, or 0 for the default
 * of 4 s.  A limit shorter than a call's own duration makes healthy calls
 * give up; it exists so that tests and health checks need not wait 4 s.
 * The waits at a kernel's exit for its own copies always allow the default.
 */
DFK_API int dfk_set_wait_limit(unsigned long long ns);

/*
 * Self-test of the bounded wait: launches one warp on `stream` that waits
 * on an mbarrier no one ever completes.  The wait gives up after the current
 * limit, sets bit 0 of the device error word, stores the time it waited (ns)
 * in *elapsed_ns (device memory, 8-byte aligned, caller-owned) and the
 * kernel returns.  A health check: afterwards dfk_device_error must report
 * DFK_ERR_TIMEOUT and the device must still run the MLP kernels.
 */
DFK_API int dfk_selftest_bounded_wait(void *elapsed_ns, void *stream);

/* Library version, e.g. "dfk 0.1.0 sm_100a". */
DFK_API const char *dfk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DFK_H */
