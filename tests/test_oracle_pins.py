"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each test fixes a value by closed form, invariant, a special case that
reduces to a textbook result or an independent library routine, or brute
force on tiny inputs, so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.

The method pinned is the SwiGLU gate/up fusion of "Deep Kernel Fusion for
Transformer Decoding" (episode description: gate projection, up
projection, SiLU, elementwise multiply; down projection separate) with the
RMSNorm prologue of GPULlama3.java PR #78 (the ``rms_ffn_gate_up`` task).
"""
import math

import numpy as np
import torch
import pytest

import oracle
from oracle import LAYOUT_COL, LAYOUT_INTERLEAVED, LAYOUT_ROW

E = math.e


def bits(vals):
    """Exact bf16 bit patterns of values that bf16 represents exactly."""
    a = np.asarray(vals, dtype=np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def layouts_of(wg, wu):
    """The three storage layouts of row-major [F, D] weights (bit patterns)."""
    F, D = wg.shape
    return {
        LAYOUT_ROW: (wg, wu),
        LAYOUT_COL: (np.ascontiguousarray(wg.T), np.ascontiguousarray(wu.T)),
        LAYOUT_INTERLEAVED: (np.ascontiguousarray(np.stack([wg, wu], axis=1)), None),
    }


# ---------------------------------------------------------------- bf16 codec

def test_bf16_decode_known_patterns(oracle_mod):
    assert oracle.bf16_to_f64(np.array([0x3F80], np.uint16))[0] == 1.0
    assert oracle.bf16_to_f64(np.array([0xC000], np.uint16))[0] == -2.0
    assert oracle.bf16_to_f64(np.array([0x3E80], np.uint16))[0] == 0.25
    assert math.isinf(oracle.bf16_to_f64(np.array([0x7F80], np.uint16))[0])
    assert oracle.bf16_to_f64(np.array([0x0001], np.uint16))[0] == 2.0 ** -133


def test_bf16_round_nearest_even(oracle_mod):
    ulp = 2.0 ** -7                                   # bf16 spacing in [1, 2)
    assert oracle.f64_to_bf16([1.0 + ulp / 2])[0] == 0x3F80          # tie -> even (down)
    assert oracle.f64_to_bf16([1.0 + 1.5 * ulp])[0] == 0x3F82        # tie -> even (up)
    assert oracle.f64_to_bf16([1.0 + ulp / 2 + 2.0 ** -30])[0] == 0x3F81
    assert oracle.f64_to_bf16([-3.0])[0] == 0xC040
    assert oracle.f64_to_bf16([0.0])[0] == 0x0000
    assert oracle.f64_to_bf16([-0.0])[0] == 0x8000
    assert oracle.f64_to_bf16([1e39])[0] == 0x7F80                   # overflow -> inf


def test_bf16_round_matches_torch_on_float32_values(oracle_mod):
    # For values already exact in float32, a single RNE rounding to bf16 is
    # what torch's float32 -> bf16 cast does: an independent library routine.
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(2000).astype(np.float32),
                        (rng.standard_normal(500) * 1e-38).astype(np.float32),
                        (rng.standard_normal(500) * 1e30).astype(np.float32)])
    ours = oracle.f64_to_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------- SiLU

def test_silu_closed_forms(oracle_mod):
    assert oracle.silu(0.0) == 0.0
    # sigmoid(ln a) = a / (1 + a)  =>  SiLU(ln a) = ln(a) * a / (1 + a)
    for a in (3.0, 0.5, 7.0, 1e-3, 250.0):
        want = math.log(a) * a / (1.0 + a)
        assert oracle.silu(math.log(a)) == pytest.approx(want, rel=1e-14, abs=1e-300)
    # SiLU(1) = e / (1 + e), SiLU(-1) = -1 / (1 + e)
    assert oracle.silu(1.0) == pytest.approx(E / (1 + E), rel=1e-15)
    assert oracle.silu(-1.0) == pytest.approx(-1.0 / (1 + E), rel=1e-15)


def test_silu_symmetry_and_limits(oracle_mod):
    # SiLU(x) - SiLU(-x) = x  (x*s(x) + x*s(-x)... since s(x) + s(-x) = 1)
    for x in (0.3, 1.7, 5.0, 13.0, 40.0):
        assert oracle.silu(x) - oracle.silu(-x) == pytest.approx(x, rel=1e-14)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)           # -> x
    assert abs(oracle.silu(-40.0)) < 1e-15                               # -> 0-
    assert oracle.silu(-40.0) < 0.0
    v = oracle.silu(-800.0)                                              # exp overflow
    assert v == 0.0 and math.copysign(1.0, v) == -1.0
    # SiLU(20) = 20 / (1 + e^-20) ~ 19.99999995877..
    assert oracle.silu(20.0) == pytest.approx(19.999999958776925, rel=1e-15)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector(oracle_mod):
    for c in (3.0, -0.5, 96.0):
        x = bits(np.full((1, 16), c))
        xn = oracle.rmsnorm(x, None, eps=0.0)
        assert np.allclose(xn, math.copysign(1.0, c), rtol=0, atol=1e-15)


def test_rmsnorm_mean_over_d_and_eps_inside_sqrt(oracle_mod):
    # x = [2, 0, 0, 0]: mean(x^2) over D=4 is 1 -> r = 1 (over D-1 it would be 4/3)
    xn = oracle.rmsnorm(bits([[2.0, 0.0, 0.0, 0.0]]), None, eps=0.0)
    assert np.array_equal(xn, [[2.0, 0.0, 0.0, 0.0]])
    # x = 1, eps = 3: r = 1/sqrt(1 + 3) = 1/2
    xn = oracle.rmsnorm(bits([[1.0] * 8]), None, eps=3.0)
    assert np.array_equal(xn, np.full((1, 8), 0.5))


def test_rmsnorm_gamma_is_per_column(oracle_mod):
    # x = [1, 1, 1, 1] -> r = 1; gamma scales column k only
    g = bits([2.0, 1.0, 0.5, -4.0])
    xn = oracle.rmsnorm(bits([[1.0, 1.0, 1.0, 1.0]]), g, eps=0.0)
    assert np.array_equal(xn, [[2.0, 1.0, 0.5, -4.0]])


def test_rmsnorm_scale_invariance(oracle_mod):
    rng = np.random.default_rng(3)
    x = oracle.f64_to_bf16(rng.standard_normal((3, 40)))
    x2 = oracle.f64_to_bf16(oracle.bf16_to_f64(x) * 4.0)      # exact scaling by 4
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(40))
    assert np.array_equal(oracle.rmsnorm(x, g, eps=0.0), oracle.rmsnorm(x2, g, eps=0.0))


# ---------------------------------------------------------------- gate/up

# own hand-worked example: D = 3, F = 2
X23 = [[1.0, 0.0, -1.0]]
WG23 = [[1.0, 0.0, 0.0], [0.0, 1.0, 1.0]]
WU23 = [[1.0, 1.0, 0.0], [2.0, 0.0, 0.0]]


@pytest.mark.parametrize("layout", [LAYOUT_ROW, LAYOUT_COL, LAYOUT_INTERLEAVED])
def test_gate_up_hand_example(oracle_mod, layout):
    # a = x Wg^T = [1, -1], u = x Wu^T = [1, 2]
    # h = [SiLU(1) * 1, SiLU(-1) * 2] = [e/(1+e), -2/(1+e)]
    wg, wu = layouts_of(bits(WG23), bits(WU23))[layout]
    h, a, u = oracle.gate_up(bits(X23), wg, wu, layout=layout, return_au=True)
    assert np.array_equal(a, [[1.0, -1.0]])
    assert np.array_equal(u, [[1.0, 2.0]])
    assert h[0, 0] == pytest.approx(E / (1 + E), rel=1e-15)
    assert h[0, 1] == pytest.approx(-2.0 / (1 + E), rel=1e-15)
    assert h[0, 0] == pytest.approx(0.7310585786300049, rel=1e-15)
    assert h[0, 1] == pytest.approx(-0.5378828427399902, rel=1e-15)


@pytest.mark.parametrize("layout", [LAYOUT_ROW, LAYOUT_COL, LAYOUT_INTERLEAVED])
def test_gate_up_hand_example_with_rmsnorm(oracle_mod, layout):
    # mean(x^2) = 2/3 -> r = sqrt(3/2) = s; gamma = [2, 1, 0.5]
    # xn = [2s, 0, -0.5s]; a = [2s, -0.5s]; u = [2s, 4s]
    s = math.sqrt(1.5)
    wg, wu = layouts_of(bits(WG23), bits(WU23))[layout]
    h, a, u = oracle.gate_up(bits(X23), wg, wu, layout=layout, gamma=bits([2.0, 1.0, 0.5]),
                             eps=0.0, return_au=True)
    assert a[0] == pytest.approx([2 * s, -0.5 * s], rel=1e-15)
    assert u[0] == pytest.approx([2 * s, 4 * s], rel=1e-15)
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    assert h[0, 0] == pytest.approx(2 * s * sig(2 * s) * 2 * s, rel=1e-14)
    assert h[0, 1] == pytest.approx(-0.5 * s * sig(-0.5 * s) * 4 * s, rel=1e-14)


def test_gate_up_equal_weights_invariant(oracle_mod):
    # W_gate = W_up  =>  u = a and h = SiLU(a) * a; a checked against numpy's matmul
    rng = np.random.default_rng(11)
    B, D, F = 3, 24, 10
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    w = oracle.f64_to_bf16(0.1 * rng.standard_normal((F, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    h, a, u = oracle.gate_up(x, w, w, gamma=g, eps=1e-5, return_au=True)
    assert np.array_equal(a, u)
    xn = oracle.rmsnorm(x, g, eps=1e-5)
    assert np.allclose(a, xn @ oracle.bf16_to_f64(w).T, rtol=1e-13, atol=1e-13)
    sig = 1.0 / (1.0 + np.exp(-a))
    assert np.allclose(h, a * sig * a, rtol=1e-13, atol=1e-15)


def test_gate_up_identity_and_permutation(oracle_mod):
    # F = D, W_up = I  =>  u = xn;  W_gate = permutation P  =>  a = xn[:, perm]
    rng = np.random.default_rng(5)
    B, D = 2, 16
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    perm = rng.permutation(D)
    eye = np.eye(D)
    P = eye[perm]                       # row j selects column perm[j]
    h, a, u = oracle.gate_up(x, bits(P), bits(eye), return_au=True)
    xv = oracle.bf16_to_f64(x)
    assert np.array_equal(u, xv)
    assert np.array_equal(a, xv[:, perm])


def test_gate_up_zero_input(oracle_mod):
    rng = np.random.default_rng(1)
    w = oracle.f64_to_bf16(rng.standard_normal((6, 8)))
    h = oracle.gate_up(bits(np.zeros((2, 8))), w, w)
    assert np.array_equal(h, np.zeros((2, 6)))


def test_layouts_agree_exactly(oracle_mod):
    rng = np.random.default_rng(9)
    B, D, F = 4, 40, 24
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    wg = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wu = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    outs = []
    for layout, (lg, lu) in layouts_of(wg, wu).items():
        outs.append(oracle.gate_up(x, lg, lu, layout=layout, gamma=g))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(2)
    B, D, F = 2, 32, 50
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    wg = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wu = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    full = oracle.gate_up(x, wg, wu)
    rows = [49, 0, 7, 7, 31]
    assert np.array_equal(oracle.gate_up(x, wg, wu, rows=rows), full[:, rows])


def test_brute_force_tiny_against_numpy(oracle_mod):
    # brute force on tiny random shapes (incl. odd, ragged sizes) with numpy fp64
    rng = np.random.default_rng(17)
    for _ in range(12):
        B, D, F = int(rng.integers(1, 6)), int(rng.integers(1, 65)), int(rng.integers(1, 65))
        x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
        wg = oracle.f64_to_bf16(0.3 * rng.standard_normal((F, D)))
        wu = oracle.f64_to_bf16(0.3 * rng.standard_normal((F, D)))
        g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
        xv, gv = oracle.bf16_to_f64(x), oracle.bf16_to_f64(g)
        xn = xv / np.sqrt(np.mean(xv * xv, axis=1, keepdims=True) + 1e-5) * gv
        a = xn @ oracle.bf16_to_f64(wg).T
        u = xn @ oracle.bf16_to_f64(wu).T
        want = a / (1.0 + np.exp(-a)) * u
        for layout, (lg, lu) in layouts_of(wg, wu).items():
            got = oracle.gate_up(x, lg, lu, layout=layout, gamma=g, eps=1e-5)
            assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def test_thread_count_does_not_change_result(oracle_mod):
    rng = np.random.default_rng(4)
    B, D, F = 3, 64, 96
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    wg = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wu = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    n0 = oracle.threads()
    try:
        oracle.set_threads(1)
        one = oracle.gate_up(x, wg, wu)
        oracle.set_threads(max(2, n0))
        many = oracle.gate_up(x, wg, wu)
    finally:
        oracle.set_threads(n0)
    assert np.array_equal(one, many)


def _torch_bf16(v):
    # torch's own cast (float64 -> bfloat16, round to nearest even) as the
    # independent rounding routine
    return torch.tensor(np.asarray(v, dtype=np.float64)).to(torch.bfloat16).to(
        torch.float64).numpy()


def test_mirror_mode_rounds_at_the_stated_points(oracle_mod):
    # mirror mode = the pure computation with a bf16 rounding (RNE) of xn, of
    # h and of y: each stage checked against torch's rounding of the pure
    # stage fed the previous stage's rounded values
    rng = np.random.default_rng(18)
    B, D, F = 3, 48, 40
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    wg = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wu = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wd = oracle.f64_to_bf16(0.2 * rng.standard_normal((D, F)))
    xn_m = oracle.rmsnorm(x, g, 1e-5, mirror=True)
    assert np.array_equal(xn_m, _torch_bf16(oracle.rmsnorm(x, g, 1e-5)))
    h_m = oracle.gate_up(x, wg, wu, gamma=g, eps=1e-5, mirror=True)
    h_from_rounded_xn = oracle.gate_up(oracle.f64_to_bf16(xn_m), wg, wu)
    assert np.array_equal(h_m, _torch_bf16(h_from_rounded_xn))
    y_m = oracle.down(h_m, wd, mirror=True)
    assert np.array_equal(y_m, _torch_bf16(oracle.down(h_m, wd)))
    # and mirror mode differs from the pure one (it does round)
    assert not np.array_equal(y_m, oracle.down(h_m, wd))


def test_mirror_mode_outputs_are_bf16(oracle_mod):
    rng = np.random.default_rng(8)
    x = oracle.f64_to_bf16(rng.standard_normal((2, 32)))
    w = oracle.f64_to_bf16(0.2 * rng.standard_normal((16, 32)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(32))
    h = oracle.gate_up(x, w, w, gamma=g, mirror=True)
    assert np.array_equal(oracle.bf16_to_f64(oracle.f64_to_bf16(h)), h)
    hp = oracle.gate_up(x, w, w, gamma=g)
    assert np.allclose(h, hp, rtol=2e-2, atol=1e-3)


# ---------------------------------------------------------------- down projection

def test_down_hand_example(oracle_mod):
    # h = [1, 2]; Wd (D=3, F=2) = [[1, 0], [0, 1], [3, -1]]  =>  y = [1, 2, 1]
    y = oracle.down(np.array([[1.0, 2.0]]), bits([[1.0, 0.0], [0.0, 1.0], [3.0, -1.0]]))
    assert np.array_equal(y, [[1.0, 2.0, 1.0]])


def test_down_identity_and_linearity(oracle_mod):
    rng = np.random.default_rng(6)
    F = 12
    h = rng.standard_normal((3, F))
    assert np.array_equal(oracle.down(h, bits(np.eye(F))), h)
    wd = oracle.f64_to_bf16(0.3 * rng.standard_normal((5, F)))
    y1, y2 = oracle.down(h, wd), oracle.down(2.0 * h, wd)
    assert np.array_equal(2.0 * y1, y2)              # scaling by 2 is exact
    assert np.allclose(y1, h @ oracle.bf16_to_f64(wd).T, rtol=1e-13, atol=1e-14)
    assert np.array_equal(oracle.down(h, wd, rows=[4, 1]), y1[:, [4, 1]])


def test_rms_rescale(oracle_mod):
    y = np.array([[3.0, -3.0, 3.0, 3.0], [0.5, 0.0, 0.0, 0.0]])
    out = oracle.rms_rescale(y, eps=0.0)
    assert np.allclose(out[0], [1.0, -1.0, 1.0, 1.0], rtol=0, atol=1e-15)
    assert np.allclose(out[1], [2.0, 0.0, 0.0, 0.0], rtol=0, atol=1e-15)


def test_full_mlp_composition(oracle_mod):
    # y of the whole MLP equals down(gate_up(...)) and is zero for zero input
    rng = np.random.default_rng(12)
    B, D, F = 2, 16, 24
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    wg = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wu = oracle.f64_to_bf16(0.2 * rng.standard_normal((F, D)))
    wd = oracle.f64_to_bf16(0.2 * rng.standard_normal((D, F)))
    h, y = oracle.mlp(x, wg, wu, wd)
    assert np.array_equal(y, oracle.down(oracle.gate_up(x, wg, wu), wd))
    _, y0 = oracle.mlp(bits(np.zeros((B, D))), wg, wu, wd)
    assert np.array_equal(y0, np.zeros((B, D)))


def test_bad_arguments_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle.gate_up(bits([[1.0, 2.0]]), bits([[1.0, 2.0, 3.0]]), bits([[1.0, 2.0, 3.0]]))
    with pytest.raises(ValueError):
        oracle.gate_up(bits([[1.0]]), bits([[1.0]]), bits([[1.0]]), rows=[1])


# ---------------------------------------------------------------- FP8 weights

def fp8(vals):
    """E4M3 codes of values that E4M3 represents exactly (torch cast)."""
    import torch
    t = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn)
    assert torch.equal(t.float(), torch.tensor(vals, dtype=torch.float32))
    return t.view(torch.uint8).numpy()


def test_e4m3_decoder_all_codes_match_torch(oracle_mod):
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2    # S.1111.111 only
    assert np.array_equal(ours[~nan], ref[~nan].astype(np.float64))
    signs = np.signbit(ours[~nan]) == np.signbit(ref[~nan])
    assert signs.all()


def test_e4m3_known_values(oracle_mod):
    v = lambda c: oracle.e4m3_to_f64(np.array([c], np.uint8))[0]
    assert v(0x38) == 1.0 and v(0x40) == 2.0 and v(0xB8) == -1.0
    assert v(0x7E) == 448.0                 # largest finite
    assert v(0x08) == 2.0 ** -6             # smallest normal
    assert v(0x01) == 2.0 ** -9             # smallest subnormal
    assert v(0x07) == 7 * 2.0 ** -9
    assert v(0x80) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))


def test_fp8_gate_up_hand_example(oracle_mod):
    # x = [1, 2]; Wg = 0.5 * [1, 2] -> a = 0.5 * (1 + 4) = 2.5
    #            Wu = 2 * [-1, 1]   -> u = 2 * (-1 + 2) = 2;  h = SiLU(2.5) * 2
    h, a, u = oracle.gate_up_fp8(bits([[1.0, 2.0]]), fp8([[1.0, 2.0]]), [0.5],
                                 fp8([[-1.0, 1.0]]), [2.0], return_au=True)
    assert a[0, 0] == 2.5 and u[0, 0] == 2.0
    assert h[0, 0] == pytest.approx(2.5 / (1 + math.exp(-2.5)) * 2.0, rel=1e-15)


def test_fp8_unit_scale_reduces_to_bf16_path(oracle_mod):
    # with s = 1 the dequantised weights are the E4M3 values, which bf16 holds
    # exactly: the FP8 oracle must equal the bf16 oracle on those weights
    rng = np.random.default_rng(21)
    B, D, F = 3, 40, 24
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    qg = rng.integers(0, 256, (F, D)).astype(np.uint8)
    qu = rng.integers(0, 256, (F, D)).astype(np.uint8)
    qg[(qg & 0x7F) == 0x7F] = 0x38           # no NaN codes
    qu[(qu & 0x7F) == 0x7F] = 0xB8
    ones = np.ones(F, np.float32)
    h8 = oracle.gate_up_fp8(x, qg, ones, qu, ones, gamma=g)
    wg = oracle.f64_to_bf16(oracle.e4m3_to_f64(qg))
    wu = oracle.f64_to_bf16(oracle.e4m3_to_f64(qu))
    assert np.array_equal(oracle.bf16_to_f64(wg), oracle.e4m3_to_f64(qg))   # exact in bf16
    assert np.array_equal(h8, oracle.gate_up(x, wg, wu, gamma=g))


def test_fp8_scales_are_per_row_and_linear(oracle_mod):
    rng = np.random.default_rng(22)
    B, D, F = 2, 32, 16
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    qg = fp8(np.round(rng.standard_normal((F, D)) * 4) / 4)
    qu = fp8(np.round(rng.standard_normal((F, D)) * 4) / 4)
    sg = (0.01 * (1 + np.arange(F))).astype(np.float32)
    su = np.full(F, 0.02, np.float32)
    _, a1, u1 = oracle.gate_up_fp8(x, qg, sg, qu, su, return_au=True)
    _, a2, u2 = oracle.gate_up_fp8(x, qg, 4 * sg, qu, su, return_au=True)
    assert np.array_equal(4 * a1, a2) and np.array_equal(u1, u2)   # gate scale only
    ref = oracle.bf16_to_f64(x) @ (oracle.e4m3_to_f64(qg) * sg.astype(np.float64)[:, None]).T
    assert np.allclose(a1, ref, rtol=1e-13, atol=1e-14)
    h = rng.standard_normal((B, F))
    qd = fp8(np.round(rng.standard_normal((D, F)) * 2) / 2)
    sd = (0.5 + np.arange(D)).astype(np.float32)
    y1 = oracle.down_fp8(h, qd, sd)
    assert np.array_equal(2 * y1, oracle.down_fp8(h, qd, 2 * sd))
    assert np.allclose(y1, h @ (oracle.e4m3_to_f64(qd) * sd.astype(np.float64)[:, None]).T,
                       rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- packed QKV

def test_qkv_hand_example(oracle_mod):
    # D = 2, nq = 2, nk = 1, nv = 1; x = [3, 4] -> mean(x^2) = 12.5, r = 1/sqrt(12.5)
    # gamma = [2, 1] -> xn = [6 r, 4 r]
    x = bits([[3.0, 4.0]])
    w = bits([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [1.0, -1.0]])
    q, k, v = oracle.qkv(x, w, 2, 1, 1, gamma=bits([2.0, 1.0]), eps=0.0)
    r = 1.0 / math.sqrt(12.5)
    assert q[0] == pytest.approx([6 * r, 4 * r], rel=1e-15)
    assert k[0, 0] == pytest.approx(10 * r, rel=1e-15)
    assert v[0, 0] == pytest.approx(2 * r, rel=1e-15)
    # without RMSNorm the product of the raw x
    q, k, v = oracle.qkv(x, w, 2, 1, 1)
    assert q[0].tolist() == [3.0, 4.0] and k[0, 0] == 7.0 and v[0, 0] == -1.0


def test_qkv_packed_equals_three_projections_and_numpy(oracle_mod):
    # the packed projection computes what three separate linear layers do
    # (the fusion changes no math), checked against numpy's matmul as an
    # independent routine
    rng = np.random.default_rng(41)
    B, D, nq, nk, nv = 3, 48, 32, 8, 8
    x = oracle.f64_to_bf16(rng.standard_normal((B, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    wq = oracle.f64_to_bf16(0.05 * rng.standard_normal((nq, D)))
    wk = oracle.f64_to_bf16(0.05 * rng.standard_normal((nk, D)))
    wv = oracle.f64_to_bf16(0.05 * rng.standard_normal((nv, D)))
    w = np.concatenate([wq, wk, wv])
    q, k, v = oracle.qkv(x, w, nq, nk, nv, gamma=g, eps=1e-5)
    xn = oracle.rmsnorm(x, g, eps=1e-5)
    for got, ws in ((q, wq), (k, wk), (v, wv)):
        assert np.array_equal(got, oracle.down(xn, ws))                  # separate layer
        assert np.allclose(got, xn @ oracle.bf16_to_f64(ws).T, rtol=1e-13, atol=1e-14)
    # packed rows subset
    rows = np.array([0, nq, nq + nk, nq + nk + nv - 1], np.int32)
    o = oracle.qkv(x, w, nq, nk, nv, gamma=g, eps=1e-5, rows=rows)
    assert np.array_equal(o, np.concatenate([q[:, :1], k[:, :1], v[:, :1], v[:, -1:]], axis=1))


def test_qkv_identity_weights_return_the_normalised_input(oracle_mod):
    rng = np.random.default_rng(42)
    D = 16
    x = oracle.f64_to_bf16(rng.standard_normal((2, D)))
    g = oracle.f64_to_bf16(1.0 + 0.1 * rng.standard_normal(D))
    eye = oracle.f64_to_bf16(np.eye(D))
    w = np.concatenate([eye, eye[:4], eye[4:8]])
    q, k, v = oracle.qkv(x, w, D, 4, 4, gamma=g, eps=1e-5)
    xn = oracle.rmsnorm(x, g, eps=1e-5)
    assert np.array_equal(q, xn) and np.array_equal(k, xn[:, :4]) and np.array_equal(v, xn[:, 4:8])
