"""Tensor-parallel SwiGLU MLP: d_ff sharded over the ranks of a
torch.distributed group, one GPU per rank.

"Deep Kernel Fusion for Transformers" (abstract) keeps the fused kernel
adaptable to inference configurations.  Across GPUs the decode MLP splits
along d_ff with a single exchange:

* rank r owns rows [f0_r, f1_r) of W_gate and W_up -- whole gate/up pairs,
  so h_r = SiLU(x W_gate_r^T) * (x W_up_r^T) is the unchanged fused gate/up
  kernel on the shard (row-major, column-major or interleaved storage) and
  needs no communication;
* it owns columns [f0_r, f1_r) of W_down as its own contiguous matrix, so
  y = sum_r h_r W_down_r^T;
* the sum runs inside the down-projection kernel
  (``dfk_tp_down_proj_allreduce``): every CTA pushes its fp32 partial rows to
  all ranks over peer memory and adds the ranks' partials in rank order, so
  every rank holds the same bits of y.

This module holds only host logic -- shard boundaries, slicing the weights,
exchanging the peer-memory handles -- and calls the library for every step
of the computation.  torch.distributed is used for the one-time handle
exchange (any backend: the handles are a few bytes of host data).
"""
from typing import List, Optional, Tuple

import torch

import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

# shard sizes are multiples of this many d_ff rows: the down projection's
# reduction length must be a multiple of 8 (16-byte rows for the copy engine)
SHARD_GRANULE = 8


def shard_bounds(d_ff: int, world: int, granule: int = SHARD_GRANULE) -> List[Tuple[int, int]]:
    """Contiguous [f0, f1) ranges of d_ff, one per rank, in rank order: each a
    multiple of `granule`, sizes differing by at most one granule."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if d_ff % granule or d_ff < granule * world:
        raise ValueError("d_ff=%d must be a multiple of %d and hold %d shards"
                         % (d_ff, granule, world))
    units = d_ff // granule
    base, extra = divmod(units, world)
    out, f0 = [], 0
    for r in range(world):
        n = (base + (1 if r < extra else 0)) * granule
        out.append((f0, f0 + n))
        f0 += n
    return out


def shard_weights(w_gate: torch.Tensor, w_up: Optional[torch.Tensor], w_down: torch.Tensor,
                  layout: int, world: int, rank: int):
    """This rank's shard of one MLP layer.

    w_gate / w_up are in `layout` storage (row [F, D]; col [D, F];
    interleaved [F, 2, D] with w_up None), w_down is [D, F].  Returns
    (wg_r, wu_r, wd_r, (f0, f1)) with wg_r / wu_r in the same layout over
    rows f0 .. f1 - 1 and wd_r = w_down[:, f0:f1] as a contiguous [D, f1 - f0]
    matrix."""
    F = w_down.shape[1]
    f0, f1 = shard_bounds(F, world)[rank]
    if layout == I.LAYOUT_ROW:
        wg, wu = w_gate[f0:f1].contiguous(), w_up[f0:f1].contiguous()
    elif layout == I.LAYOUT_COL:
        wg, wu = w_gate[:, f0:f1].contiguous(), w_up[:, f0:f1].contiguous()
    elif layout == I.LAYOUT_INTERLEAVED:
        wg, wu = w_gate[f0:f1].contiguous(), None
    else:
        raise ValueError("unknown layout %r" % (layout,))
    return wg, wu, w_down[:, f0:f1].contiguous(), (f0, f1)


def exchange_handles(handle: bytes, group=None) -> List[bytes]:
    """Every rank's handle, in rank order (an all-gather of host bytes)."""
    import torch.distributed as dist
    out: List[Optional[bytes]] = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, handle, group=group)
    return [bytes(h) for h in out]


class TPGroup:
    """The library's peer-memory group for the fused down-projection
    all-reduce (``dfk_tp_group_*``), set up collectively on every rank."""

    def __init__(self, world: int, rank: int, max_B: int, d_model: int, exchange=None):
        self.world, self.rank, self.d_model = world, rank, d_model
        self.handle, mine = dfk.dfk_tp_group_create(world, rank, max_B, d_model)
        handles = (exchange or exchange_handles)(mine) if world > 1 else [mine]
        if len(handles) != world:
            raise ValueError("expected %d handles, got %d" % (world, len(handles)))
        dfk.dfk_tp_group_connect(self.handle, handles)

    def down_proj_allreduce(self, h, w_down_shard, y=None, stream=None):
        return dfk.dfk_tp_down_proj_allreduce(self.handle, h, w_down_shard, y=y, stream=stream)

    def close(self):
        if self.handle is not None:
            dfk.dfk_tp_group_destroy(self.handle)
            self.handle = None


class TensorParallelMLP:
    """One decode MLP layer (optional fused RMSNorm, gate/up, down) sharded
    over the ranks of the default torch.distributed group.  Every rank passes
    the full weights it was given (or its shard through ``shards``) and the
    same x; forward returns the full y on every rank."""

    def __init__(self, gamma, eps, w_gate, w_up, w_down, layout=I.LAYOUT_ROW, max_B=64,
                 world=None, rank=None, exchange=None, shards=None):
        if world is None or rank is None:
            import torch.distributed as dist
            world, rank = dist.get_world_size(), dist.get_rank()
        self.gamma, self.eps, self.layout = gamma, eps, layout
        if shards is None:
            shards = shard_weights(w_gate, w_up, w_down, layout, world, rank)
        self.wg, self.wu, self.wd, self.bounds = shards
        self.group = TPGroup(world, rank, max_B, self.wd.shape[0], exchange)

    def forward(self, x, y=None, stream=None):
        if self.gamma is not None:
            h = dfk.dfk_rmsnorm_swiglu_gate_up(x, self.gamma, self.eps, self.wg, self.wu,
                                               self.layout, stream=stream)
        else:
            h = dfk.dfk_swiglu_gate_up(x, self.wg, self.wu, self.layout, stream=stream)
        return self.group.down_proj_allreduce(h, self.wd, y=y, stream=stream)

    def close(self):
        self.group.close()


def emulated_forward(x, gamma, eps, w_gate, w_up, w_down, layout, world: int):
    """The tensor-parallel layer with `world` ranks emulated on the current
    device: each rank's gate/up on its shard (the ordinary fused kernel), then
    one grid running every rank's fused down projection and all-reduce
    (``dfk_tp_down_proj_allreduce_emulated``).  Shards must be equal.
    Returns (y_all [world][B][D], h_all [world][B][F / world])."""
    bounds = shard_bounds(w_down.shape[1], world)
    if len({f1 - f0 for f0, f1 in bounds}) != 1:
        raise ValueError("emulated groups need equal shards")
    hs, wds = [], []
    for r in range(world):
        wg, wu, wd, _ = shard_weights(w_gate, w_up, w_down, layout, world, r)
        if gamma is not None:
            hs.append(dfk.dfk_rmsnorm_swiglu_gate_up(x, gamma, eps, wg, wu, layout))
        else:
            hs.append(dfk.dfk_swiglu_gate_up(x, wg, wu, layout))
        wds.append(wd)
    h_all = torch.stack(hs).contiguous()
    w_all = torch.stack(wds).contiguous()
    return dfk.dfk_tp_down_proj_allreduce_emulated(h_all, w_all), h_all

