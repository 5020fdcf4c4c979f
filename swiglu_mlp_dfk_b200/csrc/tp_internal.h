// tp_internal.h -- between the tensor-parallel entry points (tp.cu) and the
// tensor-core launcher (dfk_api.cu).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>

namespace dfk {

constexpr int TP_MAX_RANKS = 8;
constexpr int TP_MAX_BLOCKS = 256;  // row blocks a rank's flag array holds

// One group member's device buffer (identical layout on every rank):
//   recv   [2][world][bmax][d_model] fp32  partial sums, two alternating sets
//   flags  [TP_MAX_BLOCKS][world] u64      flag of (row block, source rank)
//   seq    u64                             calls this rank has completed
//   exit   u32                             CTAs of the current call done
struct TpLayout {
  size_t recv_bytes, flags_off, seq_off, exit_off, total;
};
TpLayout tp_layout(int world, int bmax, int d_model);

struct TpLaunch {
  int world;            // ranks in the group
  int rank0;            // first rank this launch computes
  int ranks_here;       // ranks this launch computes: 1, or world (emulated on one device)
  const void *h;        // [ranks_here][B][d_ff_shard] bf16
  const void *w;        // [ranks_here][d_model][d_ff_shard] bf16
  void *y;              // [ranks_here][B][d_model] bf16
  int B, d_model, d_ff_shard, bmax;
  void *buf[TP_MAX_RANKS];  // every rank's buffer (peer mappings for other ranks)
  void *ctl;                // the buffer whose seq / exit counters this launch uses
  bool cooperative;         // emulated group: one co-resident grid
};

int launch_tp_down(const TpLaunch &a, cudaStream_t s);

// Records `msg` as this thread's dfk_last_error text; returns `status`.
int report_error(int status, const char *msg);

}  // namespace dfk
