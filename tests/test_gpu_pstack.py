"""The persistent decode step (one kernel per step for the whole layer
stack, ``dfk_mlp_stack_step``) against the separate kernels and the oracle.

The persistent kernel keeps the arithmetic of the separate launches with
the tensor-core gate/up (in-kernel RMSNorm) and the four-slice split-K
tensor-core down projection, so a step must give the same bits as those
launches; each layer is also checked teacher-forced against the fp64 oracle
(gate/up on the layer's input, down on the GPU's h, the rescale on the
last y)."""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I
from swiglu_mlp_dfk_b200.stack import DecodeStack, PersistentDecodeStack

pytestmark = pytest.mark.gpu


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


def close(got, want, rtol=1e-2, atol=1e-2):
    g = I.bf16_values(got)
    bad = np.abs(g - want) > atol + rtol * np.abs(want)
    return not bad.any(), int(bad.sum())


def bits_equal(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def matching_variants():
    """A tensor-core gate/up id and the four-slice split-K tensor-core GEMV id
    (the column-major gate/up kernel always takes 128 columns per CTA, like
    the one-launch step's column-major phases)."""
    gu = dn = None
    for i in range(1, dfk.dfk_variant_count() + 1):
        v = dfk.dfk_variant_info(i)
        if v["family"] != 1 or v["e4m3_mma"]:
            continue
        if v["op"] == dfk.DFK_OP_GATE_UP and gu is None and v["full_m_tiles"] == 0:
            gu = i
        if (v["op"] == dfk.DFK_OP_DOWN and dn is None and v["k_split"] == 4
                and v["full_m_tiles"] == 0):
            dn = i
    return gu, dn


def teacher_forced(ps, x_in, layers, rows=None, drows=None):
    """Check every listed layer of the step just run against the oracle."""
    gam, wg, wu, wd = (t for t in (ps.gammas, ps.wg, ps.wu, ps.wd))
    if ps.layout == "col":
        wg, wu = wg.transpose(1, 2).contiguous(), wu.transpose(1, 2).contiguous()
    for l in layers:
        xin = x_in if l == 0 else ps.y_all[l - 1]
        ref_h = oracle.gate_up(I.to_bits(xin), I.to_bits(wg[l]), I.to_bits(wu[l]),
                               gamma=I.to_bits(gam[l]), eps=ps.eps, rows=rows)
        got_h = ps.h_all[l] if rows is None else ps.h_all[l][:, rows]
        ok, n = close(got_h, ref_h)
        assert ok, "layer %d gate/up: %d outside" % (l, n)
        ref_y = oracle.down(I.to_bits(ps.h_all[l]), I.to_bits(wd[l]), rows=drows)
        got_y = ps.y_all[l] if drows is None else ps.y_all[l][:, drows]
        ok, n = close(got_y, ref_y)
        assert ok, "layer %d down: %d outside" % (l, n)


@pytest.mark.parametrize("B", [1, 4, 13, 16])
@pytest.mark.parametrize("layout", ["row", "col"])
def test_persistent_step_equals_separate_kernels_and_oracle(B, layout):
    L, D, F = 3, 512, 1024
    x0, params = I.make_stack(L, B, D, F, seed=40 + B, w_std=0.03, device="cuda")
    ps = PersistentDecodeStack(params, x0, layout=layout)
    ref = DecodeStack(params, x0, layout=layout)
    ref.gu_variant, ref.dn_variant = matching_variants()
    for step in range(3):
        x_in = ps.x.clone()
        ps.step_eager()
        ref.step_eager()
        torch.cuda.synchronize()
        # same bits as the separate launches (which keep the last two layers' y
        # and the last layer's h)
        assert bits_equal(ps.y_all[L - 2], ref.acts[(L - 2) % 2]), step
        assert bits_equal(ps.y_all[L - 1], ref.acts[(L - 1) % 2]), step
        assert bits_equal(ps.h_all[L - 1], ref.h), step
        assert bits_equal(ps.x, ref.x), "step %d: next input differs" % step
        teacher_forced(ps, x_in, range(L))
        ok, n = close(ps.x, oracle.rms_rescale(I.bf16_values(ps.y_all[L - 1]), 1e-5))
        assert ok, "rescale: %d outside" % n


def test_persistent_step_graph_replay():
    L, B, D, F = 4, 4, 1024, 2048
    x0, params = I.make_stack(L, B, D, F, seed=50, w_std=0.02, device="cuda")
    ps = PersistentDecodeStack(params, x0)
    eager = PersistentDecodeStack(params, x0)
    ps.step_eager()
    eager.step_eager()
    ps.capture()
    for _ in range(4):
        ps.step()
        eager.step_eager()
        torch.cuda.synchronize()
        assert bits_equal(ps.x, eager.x)
        assert bits_equal(ps.h_all, eager.h_all) and bits_equal(ps.y_all, eager.y_all)
    ps.release()


@pytest.mark.parametrize("layout", ["row", "col"])
def test_persistent_step_llama3_8b_stack(layout):
    # the 32-layer Llama-3-8B-shaped stack (B = 4): bit-identical to the
    # separate kernels over two steps, teacher-forced against the oracle on
    # layers 0, 15 and 31 (sampled output rows)
    L, B, D, F = 32, 4, 4096, 14336
    x0, params = I.make_stack(L, B, D, F, seed=4, w_std=0.02, device="cuda")
    stacked = tuple(torch.stack([p[i] for p in params]) for i in range(4))
    del params
    layers = [tuple(t[l] for t in stacked) for l in range(L)]
    ps = PersistentDecodeStack(x0=x0, stacked=stacked, layout=layout)
    ref = DecodeStack(layers, x0, layout=layout)
    ref.gu_variant, ref.dn_variant = matching_variants()
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([[0, F - 1], rng.integers(0, F, 192)])).astype(np.int32)
    drows = np.unique(np.concatenate([[0, D - 1], rng.integers(0, D, 128)])).astype(np.int32)
    for step in range(2):
        x_in = ps.x.clone()
        ps.step_eager()
        ref.step_eager()
        torch.cuda.synchronize()
        assert bits_equal(ps.x, ref.x), "step %d" % step
        assert bits_equal(ps.y_all[L - 1], ref.acts[(L - 1) % 2])
        teacher_forced(ps, x_in, (0, 15, 31), rows=rows, drows=drows)


def test_persistent_step_rejects_unsupported_shapes():
    L, B, D, F = 2, 17, 512, 1024
    x0, params = I.make_stack(L, 16, D, F, seed=1, device="cuda")
    with pytest.raises(dfk.DfkError):
        dfk.dfk_mlp_stack_workspace_bytes(L, B, D, F)      # B > 16
    with pytest.raises(dfk.DfkError):
        dfk.dfk_mlp_stack_workspace_bytes(L, 4, D, 128 * 200)   # d_ff > 128 rows per SM
