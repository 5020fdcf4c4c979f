"""The allocation-free down projection, checked against the ordinary one.

dfk_down_proj_static_scratch is for callers that cannot allocate device
memory while they run the MLP (a runtime that owns all device memory through
its own pool, or code running inside CUDA stream capture).  It keeps its
split-K partial sums in a scratch array that is part of the library image.
This file runs last (pytest collects files in name order), so that a
failure here does not hide the results of the other GPU tests; it also passes
when run on its own in a fresh process, where its first call is the one that
looks up the array's device address.
"""
import numpy as np
import pytest
import torch

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


@pytest.mark.parametrize("B,D,F", [(4, 4096, 14336), (16, 4096, 14336), (64, 1024, 2048),
                                   (3, 1000, 688)])
def test_static_scratch_matches_down_proj_twice(B, D, F):
    g = torch.Generator(device="cuda").manual_seed(B * 31 + D)
    h = (torch.randn(B, F, generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    wd = (torch.randn(D, F, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    ref = I.bf16_values(dfk.dfk_down_proj(h, wd))           # the existing entry point
    for call in range(2):                                   # two calls in a row
        y = dfk.dfk_down_proj_static_scratch(h, wd)
        torch.cuda.synchronize()
        got = I.bf16_values(y)
        bad = np.abs(got - ref) > ATOL + RTOL * np.abs(ref)
        assert not bad.any(), "call %d: %d elements differ beyond tolerance" % (call, bad.sum())


def test_static_scratch_empty_batch_is_a_no_op():
    wd = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    assert dfk.lib().dfk_down_proj_static_scratch(None, wd.data_ptr(), None, 0, 64, 64,
                                                  None) == dfk.DFK_OK
