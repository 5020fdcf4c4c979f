"""Tensor-parallel MLP, host side, on CPU: shard boundaries, the weight
shards of every layout, the handle exchange over two gloo ranks, and the
sharded arithmetic itself -- each rank's partial down projection computed by
the fp64 oracle on its shard, gathered over gloo and added in rank order --
against the oracle's whole layer."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from swiglu_mlp_dfk_b200 import inputs as I  # noqa: E402
from swiglu_mlp_dfk_b200 import tp  # noqa: E402


@pytest.mark.parametrize("F,world", [(14336, 2), (14336, 8), (688, 3), (2056, 4), (8, 1),
                                     (64, 8)])
def test_shard_bounds_cover_d_ff(F, world):
    b = tp.shard_bounds(F, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == F
    sizes = [f1 - f0 for f0, f1 in b]
    assert all(s % 8 == 0 and s > 0 for s in sizes)
    assert max(sizes) - min(sizes) <= 8
    assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))


def test_shard_bounds_reject():
    with pytest.raises(ValueError):
        tp.shard_bounds(100, 2)          # not a multiple of 8
    with pytest.raises(ValueError):
        tp.shard_bounds(16, 4)           # fewer granules than ranks
    with pytest.raises(ValueError):
        tp.shard_bounds(64, 0)


@pytest.mark.parametrize("layout", [I.LAYOUT_ROW, I.LAYOUT_COL, I.LAYOUT_INTERLEAVED])
def test_shards_reassemble_the_layer(layout):
    inp = I.make_inputs(2, 64, 200, seed=3, device="cpu")
    wg, wu = I.to_layout(inp.w_gate, inp.w_up, layout)
    parts = [tp.shard_weights(wg, wu, inp.w_down, layout, 3, r) for r in range(3)]
    cat_d = torch.cat([p[2] for p in parts], dim=1)
    assert torch.equal(cat_d, inp.w_down)
    if layout == I.LAYOUT_COL:
        assert torch.equal(torch.cat([p[0] for p in parts], 1), wg)
        assert torch.equal(torch.cat([p[1] for p in parts], 1), wu)
    else:
        assert torch.equal(torch.cat([p[0] for p in parts], 0), wg)
        if layout == I.LAYOUT_ROW:
            assert torch.equal(torch.cat([p[1] for p in parts], 0), wu)
        else:
            assert all(p[1] is None for p in parts)
            # whole gate/up pairs: shard rows j are [gate_j, up_j]
            f0, f1 = parts[1][3]
            assert torch.equal(parts[1][0][:, 0], inp.w_gate[f0:f1])
            assert torch.equal(parts[1][0][:, 1], inp.w_up[f0:f1])


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle as O
    from swiglu_mlp_dfk_b200 import inputs as In
    from swiglu_mlp_dfk_b200 import tp as T
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # the handle exchange: every rank gets every rank's bytes in rank order
        hs = T.exchange_handles(bytes([rank] * 64))
        assert hs == [bytes([r] * 64) for r in range(world)]
        # the sharded layer: rank r's gate/up on its rows, its partial down
        # projection on its W_down columns (fp64 oracle), gathered and added
        # in rank order as the fused kernel does
        inp = In.make_inputs(3, 128, 400, seed=11, w_std=0.05, device="cpu")
        out = []
        for layout in (In.LAYOUT_ROW, In.LAYOUT_COL, In.LAYOUT_INTERLEAVED):
            wg, wu = In.to_layout(inp.w_gate, inp.w_up, layout)
            sg, su, sd, (f0, f1) = T.shard_weights(wg, wu, inp.w_down, layout, world, rank)
            h_r = O.gate_up(In.to_bits(inp.x), In.to_bits(sg),
                            In.to_bits(su) if su is not None else None, layout=layout,
                            gamma=In.to_bits(inp.gamma), eps=inp.eps)
            y_r = torch.from_numpy(O.down(h_r, In.to_bits(sd)))
            parts = [torch.zeros_like(y_r) for _ in range(world)]
            dist.all_gather(parts, y_r)
            acc = parts[0].clone()
            for p in parts[1:]:
                acc = acc + p
            out.append(acc.numpy())
        q.put((rank, out))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_sharded_layer_equals_whole_layer_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = I.make_inputs(3, 128, 400, seed=11, w_std=0.05, device="cpu")
    _, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                          I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
    for layout_i in range(3):
        a, b = res[0][layout_i], res[1][layout_i]
        assert np.array_equal(a, b)            # every rank holds the same bits
        # the split only reorders an fp64 sum
        assert np.allclose(a, y_ref, rtol=1e-12, atol=1e-12)
