"""The allocation-free down projection, checked against the ordinary one and
against the fp64 oracle.

dfk_down_proj_static_scratch is for callers that cannot allocate device
memory while they run the MLP (a runtime that owns all device memory through
its own pool, or code running inside CUDA stream capture).  It keeps its
split-K partial sums in a scratch array that is part of the library image.
This file runs last (pytest collects files in name order), so that a
failure here does not hide the results of the other GPU tests; it also passes
when run on its own in a fresh process, where its first call is the one that
looks up the array's device address.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

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


def _check(got, ref, what):
    bad = np.abs(got - ref) > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), "%s: %d elements differ beyond tolerance" % (what, bad.sum())


def _sample_rows(D, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, 1, D // 2, D - 1], rng.integers(0, D, n)]))
    return rows.astype(np.int32)


@pytest.mark.parametrize("B,D,F", [(4, 4096, 14336), (16, 4096, 14336), (64, 1024, 2048),
                                   (3, 1000, 688)])
def test_static_scratch_matches_down_proj_twice(B, D, F):
    g = torch.Generator(device="cuda").manual_seed(B * 31 + D)
    h = (torch.randn(B, F, generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    wd = (torch.randn(D, F, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    ref = I.bf16_values(dfk.dfk_down_proj(h, wd))           # the existing entry point
    # the fp64 oracle on the same bytes (sampled output rows at the 8B shape)
    rows = _sample_rows(D, 256, B) if D * F > 1 << 24 else np.arange(D, dtype=np.int32)
    want = oracle.down(I.to_bits(h), I.to_bits(wd), rows=rows)
    for call in range(2):                                   # two calls in a row
        y = dfk.dfk_down_proj_static_scratch(h, wd)
        torch.cuda.synchronize()
        got = I.bf16_values(y)
        _check(got, ref, "call %d against dfk_down_proj" % call)
        _check(got[:, rows], want, "call %d against the oracle" % call)


def test_static_scratch_empty_batch_is_a_no_op():
    wd = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    assert dfk.lib().dfk_down_proj_static_scratch(None, wd.data_ptr(), None, 0, 64, 64,
                                                  None) == dfk.DFK_OK


def test_rejected_calls_enqueue_nothing():
    # a call that fails validation returns its status before any work reaches
    # the stream: captured into a graph, it leaves the graph without nodes
    h = torch.zeros(4, 512, dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    lib = dfk.lib()
    dfk.dfk_down_proj_static_scratch(h, wd)                # address looked up before capture
    torch.cuda.synchronize()
    cases = [
        ((None, wd.data_ptr(), y.data_ptr(), 4, 256, 512), dfk.DFK_ERR_INVALID_ARG),
        ((h.data_ptr(), wd.data_ptr(), y.data_ptr() + 2, 4, 256, 512), dfk.DFK_ERR_MISALIGNED),
        ((h.data_ptr(), wd.data_ptr(), y.data_ptr(), 65, 256, 512),
         dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    ]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    for args, status in cases:
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=s):
            rc = lib.dfk_down_proj_static_scratch(*args, ctypes.c_void_p(s.cuda_stream))
        assert rc == status, (args, rc)
        assert graph_node_count(g) == 0, "a rejected call enqueued work"
        del g


def graph_node_count(g):
    """Nodes in a captured (kept) torch CUDA graph, via the CUDA runtime that
    torch has loaded."""
    rt = ctypes.CDLL("libcudart.so.12")
    n = ctypes.c_size_t(0)
    rc = rt.cudaGraphGetNodes(ctypes.c_void_p(g.raw_cuda_graph()), None, ctypes.byref(n))
    assert rc == 0, rc
    return n.value
