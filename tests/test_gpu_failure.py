"""Failure detection on the GPU without a fault: a bounded pipeline wait that
nothing completes gives up after the device's wait limit, the kernel
returns, the device error word reports the timeout, and the context keeps
running the MLP kernels (checked against the oracle afterwards)."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from swiglu_mlp_dfk_b200 import build
    build.build()
    dfk.dfk_device_error()
    yield
    dfk.dfk_set_wait_limit(0)
    torch.cuda.synchronize()
    assert dfk.dfk_device_error() == 0


@pytest.mark.parametrize("limit_us", [200, 2000])
def test_bounded_wait_gives_up_and_reports_timeout(limit_us):
    dfk.dfk_device_error()                          # clear
    dfk.dfk_set_wait_limit(limit_us * 1000)
    try:
        t = dfk.dfk_selftest_bounded_wait()
        st, code, text = dfk.dfk_device_status()    # synchronises
    finally:
        dfk.dfk_set_wait_limit(0)
    waited = int(t.item())
    assert st == dfk.DFK_ERR_TIMEOUT and code & 1, (st, code, text)
    # the wait lasted at least the limit and gave up well before the default 4 s
    assert limit_us * 1000 <= waited < 500_000_000, waited
    # the error word was cleared by the read
    assert dfk.dfk_device_error() == 0


def test_context_usable_after_a_timeout():
    dfk.dfk_set_wait_limit(100_000)
    try:
        dfk.dfk_selftest_bounded_wait()
        assert dfk.dfk_device_error() & 1
    finally:
        dfk.dfk_set_wait_limit(0)
    inp = I.make_inputs(4, 512, 1032, seed=90, w_std=0.05, device="cuda")
    h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up, "row")
    y = dfk.dfk_down_proj(h, inp.w_down)
    torch.cuda.synchronize()
    assert dfk.dfk_device_error() == 0
    h_ref, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                              I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
    for got, ref in ((h, h_ref), (y, y_ref)):
        g = I.bf16_values(got)
        assert np.all(np.abs(g - ref) <= 1e-2 + 1e-2 * np.abs(ref))


def test_default_limit_does_not_fire_in_healthy_calls():
    # with the default limit a full-size call never trips the wait
    inp = I.make_workload("llama3_8b", device="cuda", with_down=True)
    for _ in range(3):
        h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up,
                                           "row")
        dfk.dfk_down_proj(h, inp.w_down)
    assert dfk.dfk_device_error() == 0
