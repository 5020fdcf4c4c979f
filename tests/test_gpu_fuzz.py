"""Randomised GPU parity: seeded random shapes (ragged B, d_model and d_ff),
layouts and options for every entry point, each result against the fp64
oracle within 1e-2 + 1e-2 |oracle|, with the scheduler's own choice of
variant (timed on first use of each shape, as a user's first call would be).
The shapes are drawn once from a fixed seed, so a failure reproduces."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

pytestmark = pytest.mark.gpu

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


def assert_close(got_bf16, want_f64, what):
    g = I.bf16_values(got_bf16)
    w = np.asarray(want_f64, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    err = np.abs(g - w)
    bad = err > ATOL + RTOL * np.abs(w)
    assert not bad.any(), "%s: %d/%d out of tolerance, max err %g" % (
        what, int(bad.sum()), bad.size, float(err.max()))


def _shapes(n, seed, d_mult, f_mult, bmax=64):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        B = int(rng.choice([1, 2, 3, 4, 5, 7, 8, 12, 16, 17, 31, 32, 33, 48, 63, 64]))
        B = min(B, bmax)
        D = int(rng.integers(8, 1600 // d_mult)) * d_mult
        F = int(rng.integers(1, 2600 // f_mult)) * f_mult
        out.append((B, D, F, int(rng.integers(0, 1 << 30))))
    return out


# bf16 fused gate/up: any d_model % 8, any d_ff (column-major needs d_ff % 8)
@pytest.mark.parametrize("B,D,F,seed", _shapes(14, 11, 8, 1))
@pytest.mark.parametrize("layout", ["row", "col", "interleaved"])
def test_fuzz_gate_up(B, D, F, seed, layout):
    if layout == "col" and F % 8:
        F += 8 - F % 8
    norm = bool(seed & 1)
    inp = I.make_inputs(B, D, F, seed=seed, w_std=0.04, norm=norm, with_down=True, device="cuda")
    lay = {"row": I.LAYOUT_ROW, "col": I.LAYOUT_COL, "interleaved": I.LAYOUT_INTERLEAVED}[layout]
    wg, wu = I.to_layout(inp.w_gate, inp.w_up, lay)
    if norm:
        h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, layout)
    else:
        h = dfk.dfk_swiglu_gate_up(inp.x, wg, wu, layout)
    torch.cuda.synchronize()
    h_ref = oracle.gate_up(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                           gamma=I.to_bits(inp.gamma) if norm else None, eps=inp.eps)
    assert_close(h, h_ref, "gate/up %s B=%d D=%d F=%d norm=%d" % (layout, B, D, F, norm))
    if F % 8:  # the down projection reduces over d_ff: d_ff % 8 is required
        with pytest.raises(dfk.DfkError) as e:
            dfk.dfk_down_proj(h, inp.w_down)
        assert e.value.status == dfk.DFK_ERR_UNSUPPORTED_SHAPE
        return
    y = dfk.dfk_down_proj(h, inp.w_down)
    torch.cuda.synchronize()
    y_ref = oracle.down(I.to_bits(h), I.to_bits(inp.w_down))
    assert_close(y, y_ref, "down B=%d D=%d F=%d" % (B, D, F))


# FP8 weights: the reduction length a multiple of 16 (d_model for gate/up,
# d_ff for the down projection)
@pytest.mark.parametrize("B,D,F,seed", _shapes(10, 12, 16, 16))
def test_fuzz_fp8(B, D, F, seed):
    norm = bool(seed & 1)
    inp = I.make_inputs(B, D, F, seed=seed, w_std=0.04, norm=norm, with_down=True, device="cuda")
    qg, sg = I.to_fp8_rows(inp.w_gate)
    qu, su = I.to_fp8_rows(inp.w_up)
    qd, sd = I.to_fp8_rows(inp.w_down)
    if norm:
        h = dfk.dfk_rmsnorm_swiglu_gate_up_fp8(inp.x, inp.gamma, inp.eps, qg, sg, qu, su)
    else:
        h = dfk.dfk_swiglu_gate_up_fp8(inp.x, qg, sg, qu, su)
    y = dfk.dfk_down_proj_fp8(h, qd, sd)
    torch.cuda.synchronize()
    host = lambda t: t.detach().cpu().numpy()
    h_ref = oracle.gate_up_fp8(I.to_bits(inp.x), host(qg), host(sg), host(qu), host(su),
                               gamma=I.to_bits(inp.gamma) if norm else None, eps=inp.eps)
    assert_close(h, h_ref, "fp8 gate/up B=%d D=%d F=%d norm=%d" % (B, D, F, norm))
    y_ref = oracle.down_fp8(I.to_bits(h), host(qd), host(sd))
    assert_close(y, y_ref, "fp8 down B=%d D=%d F=%d" % (B, D, F))


# packed QKV: random part sizes (k and v may be empty)
@pytest.mark.parametrize("B,D,F,seed", _shapes(8, 13, 8, 8))
def test_fuzz_qkv(B, D, F, seed):
    rng = np.random.default_rng(seed)
    nq = F
    nk = int(rng.integers(0, 4)) * 8 * int(rng.integers(1, 33))
    nv = nk
    norm = bool(seed & 1)
    g = I.make_generator(seed, "cuda")
    x = torch.randn(B, D, generator=g, device="cuda").to(torch.bfloat16)
    gamma = (1.0 + 0.1 * torch.randn(D, generator=g, device="cuda")).to(torch.bfloat16)
    w = (0.04 * torch.randn(nq + nk + nv, D, generator=g, device="cuda")).to(torch.bfloat16)
    q, k, v = dfk.dfk_rmsnorm_qkv_proj(x, gamma if norm else None, 1e-5, w, nq, nk, nv)
    torch.cuda.synchronize()
    want = oracle.qkv(I.to_bits(x), I.to_bits(w), nq, nk, nv,
                      gamma=I.to_bits(gamma) if norm else None, eps=1e-5)
    for got, ref, name in zip((q, k, v), want, "qkv"):
        assert_close(got, ref, "qkv %s B=%d D=%d parts %d/%d/%d norm=%d"
                     % (name, B, D, nq, nk, nv, norm))
