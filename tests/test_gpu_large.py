"""GPU parity at the largest shapes the library is meant for: a
Llama-3-405B-shaped MLP layer (d_model 16384, d_ff 53248: 3.5 GB of gate/up
weights and 1.7 GB of down weights in bf16, 1.74e9 bytes per matrix, close
to the 2^31 limit of 32-bit byte offsets) at the smallest and the largest
decode batch, through the C ABI, with the scheduler's own choice of variant.
Shapes only, seeded synthetic weights.

Outputs are compared on sampled columns against the fp64 oracle run on the
same sampled weight rows (tolerance 1e-2 + 1e-2 |oracle|); the down
projection is checked on the GPU's own bf16 h, its input in HBM."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

pytestmark = pytest.mark.gpu

D405, F405 = 16384, 53248
ATOL = RTOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from swiglu_mlp_dfk_b200 import build
    build.build()
    dfk.dfk_device_error()
    yield
    torch.cuda.synchronize()
    assert dfk.dfk_device_error() == 0, "a kernel pipeline wait timed out"


@pytest.fixture(scope="module")
def layer405():
    inp = I.make_inputs(64, D405, F405, seed=9, w_std=0.008, norm=True, with_down=True,
                        device="cuda")
    yield inp
    del inp
    torch.cuda.empty_cache()


def assert_close(got_bf16, want_f64, what):
    g = I.bf16_values(got_bf16)
    w = np.asarray(want_f64, dtype=np.float64)
    assert g.shape == w.shape, (g.shape, w.shape)
    err = np.abs(g - w)
    bad = err > ATOL + RTOL * np.abs(w)
    assert not bad.any(), "%s: %d/%d out of tolerance, max err %g" % (
        what, int(bad.sum()), bad.size, float(err.max()))


def sample(n, k, seed):
    rng = np.random.default_rng(seed)
    s = np.unique(np.concatenate([[0, 1, n - 2, n - 1], rng.choice(n, k, replace=False)]))
    return s.astype(np.int64)


@pytest.mark.parametrize("B", [1, 64])
def test_llama3_405b_shaped_layer(B, layer405):
    inp = layer405
    x = inp.x[:B].contiguous()
    h = dfk.dfk_rmsnorm_swiglu_gate_up(x, inp.gamma, 1e-5, inp.w_gate, inp.w_up, "row")
    y = dfk.dfk_down_proj(h, inp.w_down)
    torch.cuda.synchronize()
    hc = sample(F405, 160, 10 + B)
    hi = torch.from_numpy(hc).cuda()
    h_ref = oracle.gate_up(I.to_bits(x), I.to_bits(inp.w_gate[hi].contiguous()),
                           I.to_bits(inp.w_up[hi].contiguous()), gamma=I.to_bits(inp.gamma),
                           eps=1e-5)
    assert_close(h[:, hi].contiguous(), h_ref, "405B gate/up B=%d" % B)
    yc = sample(D405, 96, 20 + B)
    yi = torch.from_numpy(yc).cuda()
    y_ref = oracle.down(I.to_bits(h), I.to_bits(inp.w_down[yi].contiguous()))
    assert_close(y[:, yi].contiguous(), y_ref, "405B down B=%d" % B)


@pytest.mark.parametrize("B", [1, 16])
def test_llama3_405b_shaped_layer_fp8(B, layer405):
    inp = layer405
    x = inp.x[:B].contiguous()
    qg, sg = I.to_fp8_rows(inp.w_gate)
    qu, su = I.to_fp8_rows(inp.w_up)
    h = dfk.dfk_rmsnorm_swiglu_gate_up_fp8(x, inp.gamma, 1e-5, qg, sg, qu, su)
    del qu, su
    qd, sd = I.to_fp8_rows(inp.w_down)
    y = dfk.dfk_down_proj_fp8(h, qd, sd)
    torch.cuda.synchronize()
    hc = sample(F405, 160, 30 + B)
    hi = torch.from_numpy(hc).cuda()
    host = lambda t: t.detach().cpu().numpy()
    qu_s, su_s = I.to_fp8_rows(inp.w_up[hi].contiguous())
    h_ref = oracle.gate_up_fp8(I.to_bits(x), host(qg[hi]), host(sg[hi]), host(qu_s),
                               host(su_s), gamma=I.to_bits(inp.gamma), eps=1e-5)
    assert_close(h[:, hi].contiguous(), h_ref, "405B FP8 gate/up B=%d" % B)
    yc = sample(D405, 96, 40 + B)
    yi = torch.from_numpy(yc).cuda()
    y_ref = oracle.down_fp8(I.to_bits(h), host(qd[yi]), host(sd[yi]))
    assert_close(y[:, yi].contiguous(), y_ref, "405B FP8 down B=%d" % B)
