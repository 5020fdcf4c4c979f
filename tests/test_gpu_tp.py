"""Tensor-parallel MLP on the GPU: the down projection with the all-reduce
fused into its epilogue.

One GPU is available, so the multi-rank kernel runs with its ranks emulated
in one cooperative grid (every CTA resident, so CTAs may wait on one
another): each emulated rank pushes its fp32 partial rows into every rank's
receive buffer, raises its flags, waits for the others and adds the
partials in rank order -- the code path of the multi-GPU call, on one
device.  A one-rank group exercises the multi-GPU entry point itself.
Checked against the fp64 oracle's whole layer, every rank's y bit-identical,
and repeated calls (both alternating buffer sets) bit-identical."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I
from swiglu_mlp_dfk_b200 import tp

pytestmark = pytest.mark.gpu

ATOL = 1e-2
RTOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from swiglu_mlp_dfk_b200 import build
    build.build()
    dfk.dfk_device_error()
    yield
    torch.cuda.synchronize()
    assert dfk.dfk_device_error() == 0


def assert_close(got, want, what):
    g = I.bf16_values(got)
    bad = np.abs(g - want) > ATOL + RTOL * np.abs(want)
    assert not bad.any(), "%s: %d/%d out of tolerance" % (what, bad.sum(), bad.size)


def bits_equal(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [1, 5, 16, 64])
def test_emulated_group_matches_oracle(world, B):
    D, F = 512, 2048
    inp = I.make_inputs(B, D, F, seed=700 + B, w_std=0.03, device="cuda")
    y_all, h_all = tp.emulated_forward(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up,
                                       inp.w_down, I.LAYOUT_ROW, world)
    torch.cuda.synchronize()
    for r in range(1, world):
        assert bits_equal(y_all[0], y_all[r]), "rank %d's y differs" % r
    # end to end: the oracle's whole layer
    _, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                          I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
    assert_close(y_all[0], y_ref, "world %d B %d end to end" % (world, B))
    # isolated: the sum of the oracle's partial down projections on the GPU's h
    bounds = tp.shard_bounds(F, world)
    iso = sum(oracle.down(I.to_bits(h_all[r]), I.to_bits(inp.w_down[:, f0:f1].contiguous()))
              for r, (f0, f1) in enumerate(bounds))
    assert_close(y_all[0], iso, "world %d B %d isolated" % (world, B))
    # repeated calls alternate the receive-buffer sets and give the same bits
    w_all = torch.stack([inp.w_down[:, f0:f1].contiguous() for f0, f1 in bounds])
    for _ in range(3):
        again = dfk.dfk_tp_down_proj_allreduce_emulated(h_all, w_all)
        torch.cuda.synchronize()
        assert bits_equal(again, y_all)


@pytest.mark.parametrize("layout", [I.LAYOUT_COL, I.LAYOUT_INTERLEAVED])
def test_emulated_group_every_layout(layout):
    B, D, F = 8, 1024, 4096
    inp = I.make_inputs(B, D, F, seed=710, w_std=0.02, device="cuda")
    wg, wu = I.to_layout(inp.w_gate, inp.w_up, layout)
    y_all, _ = tp.emulated_forward(inp.x, inp.gamma, inp.eps, wg, wu, inp.w_down, layout, 4)
    torch.cuda.synchronize()
    _, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                          I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
    assert_close(y_all[3], y_ref, "layout %d" % layout)


def test_emulated_group_llama3_8b_sampled():
    # the 8B layer split over two emulated ranks (7168 d_ff rows each)
    B = 4
    inp = I.make_workload("llama3_8b_sweep", B=B, device="cuda", with_down=True)
    y_all, h_all = tp.emulated_forward(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up,
                                       inp.w_down, I.LAYOUT_ROW, 2)
    torch.cuda.synchronize()
    assert bits_equal(y_all[0], y_all[1])
    rows = np.unique(np.concatenate([[0, 4095], np.random.default_rng(5).integers(0, 4096,
                                                                                   256)]))
    rows = rows.astype(np.int32)
    h_full = torch.cat([h_all[0], h_all[1]], dim=1)
    ref = oracle.down(I.to_bits(h_full), I.to_bits(inp.w_down), rows=rows)
    assert_close(y_all[0][:, rows], ref, "8B two ranks")


def test_one_rank_group_and_graph_replay():
    # the multi-GPU entry point with a group of one: create, connect, call;
    # then captured in a CUDA graph and replayed (the call counter lives on
    # the device, so each replay is a new call)
    B, D, F = 4, 512, 1024
    inp = I.make_inputs(B, D, F, seed=720, w_std=0.03, device="cuda")
    mlp = tp.TensorParallelMLP(inp.gamma, inp.eps, inp.w_gate, inp.w_up, inp.w_down,
                               I.LAYOUT_ROW, max_B=8, world=1, rank=0)
    try:
        _, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                              I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
        y = mlp.forward(inp.x)
        torch.cuda.synchronize()
        assert_close(y, y_ref, "one-rank group")
        y2 = torch.empty_like(y)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            mlp.forward(inp.x, y=y2)
        for _ in range(3):
            y2.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert bits_equal(y2, y)
        del g
        with pytest.raises(dfk.DfkError) as e:
            mlp.group.down_proj_allreduce(torch.empty(9, F // 1, dtype=torch.bfloat16,
                                                      device="cuda"), mlp.wd)
        assert e.value.status == dfk.DFK_ERR_UNSUPPORTED_SHAPE     # B above max_B
    finally:
        mlp.close()


def test_emulated_group_too_large_is_rejected():
    # every emulated rank's CTAs must be resident at once: 8 ranks of an
    # 8192-row down projection need more CTAs than the device holds
    h = torch.zeros(8, 1, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(8, 8192, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dfk.DfkError) as e:
        dfk.dfk_tp_down_proj_allreduce_emulated(h, w)
    assert e.value.status == dfk.DFK_ERR_UNSUPPORTED_SHAPE
