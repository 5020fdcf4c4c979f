"""GPU parity for FP8 E4M3 weight streaming (fused dequantisation), through
the C ABI, against the fp64 oracle on the same codes and scales.

Tolerance: |gpu - oracle| <= 1e-2 + 1e-2 |oracle| elementwise (the same bound
as the bf16 path: the codes are exact in fp32, only the fp32 accumulation and
the one bf16 rounding of the output differ from the oracle).  Bitwise
invariants: every CUDA-core variant gives the same bits, row b of the output
does not depend on the batch size, and with unit scales the FP8 kernel equals
the bf16 kernel run on the decoded weights up to the summation order.
"""
import numpy as np
import pytest
import torch

import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I

pytestmark = pytest.mark.gpu

ATOL = 1e-2
RTOL = 1e-2


def assert_close(got_bf16, want_f64, what=""):
    g = I.bf16_values(got_bf16)
    w = np.asarray(want_f64, dtype=np.float64)
    assert g.shape == w.shape, (g.shape, w.shape)
    err = np.abs(g - w)
    bound = ATOL + RTOL * np.abs(w)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError("%s: %d/%d elements out of tolerance; worst at %s: gpu %r oracle %r"
                             % (what, bad.sum(), bad.size, i, g[i], w[i]))


def bits_equal(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


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


class Fp8Layer:
    """bf16 layer tensors and their FP8 E4M3 row-scaled encodings (on the GPU)."""

    def __init__(self, B, D, F, seed, norm=True, with_down=True, w_std=0.02):
        inp = I.make_inputs(B, D, F, seed=seed, w_std=w_std, norm=norm, with_down=with_down,
                            device="cuda")
        self.inp = inp
        self.qg, self.sg = I.to_fp8_rows(inp.w_gate)
        self.qu, self.su = I.to_fp8_rows(inp.w_up)
        if with_down:
            self.qd, self.sd = I.to_fp8_rows(inp.w_down)

    def host(self, t):
        return t.detach().cpu().numpy()

    def gate_up(self, norm, variant=0, x=None):
        x = self.inp.x if x is None else x
        if norm:
            return dfk.dfk_rmsnorm_swiglu_gate_up_fp8(x, self.inp.gamma, self.inp.eps, self.qg,
                                                      self.sg, self.qu, self.su,
                                                      variant=variant)
        return dfk.dfk_swiglu_gate_up_fp8(x, self.qg, self.sg, self.qu, self.su,
                                          variant=variant)

    def oracle_gate_up(self, norm, rows=None):
        return oracle.gate_up_fp8(I.to_bits(self.inp.x), self.host(self.qg), self.host(self.sg),
                                  self.host(self.qu), self.host(self.su),
                                  gamma=I.to_bits(self.inp.gamma) if norm else None,
                                  eps=self.inp.eps, rows=rows)

    def oracle_down(self, h_bf16, rows=None):
        return oracle.down_fp8(I.bf16_values(h_bf16), self.host(self.qd), self.host(self.sd),
                               rows=rows)


def cc_ids(op):
    """CUDA-core variant ids of op's class usable with FP8 weights (<= 2 tiles per stage)."""
    want = dfk.DFK_OP_DOWN if op == dfk.DFK_OP_DOWN_FP8 else dfk.DFK_OP_GATE_UP
    out = []
    for i in range(1, dfk.dfk_variant_count() + 1):
        v = dfk.dfk_variant_info(i)
        if v["op"] == want and v["family"] == 0 and v["k_tiles_per_stage"] <= 2:
            out.append(v)
    return out


def bt_for(B, jpt):
    return min(1 << max(B - 1, 0).bit_length(), 4 if jpt == 4 else 8)


def try_variant(fn, vid):
    """Run fn(vid); None if the variant does not fit the shape."""
    try:
        return fn(vid)
    except dfk.DfkError as e:
        if e.status == dfk.DFK_ERR_NO_VARIANT:
            return None
        raise


# (B, D, F): several 128-wide tiles, ragged F over the CTAs, D not a multiple of 128
SHAPES = [(1, 256, 688), (2, 144, 200), (3, 400, 1000), (4, 1024, 1496), (5, 272, 96),
          (8, 512, 520)]


@pytest.mark.parametrize("B,D,F", SHAPES)
@pytest.mark.parametrize("norm", [False, True])
def test_fp8_gate_up_small_shapes(B, D, F, norm):
    L = Fp8Layer(B, D, F, seed=100 + B, norm=norm, with_down=False)
    h = L.gate_up(norm)
    torch.cuda.synchronize()
    assert_close(h, L.oracle_gate_up(norm), "fp8 gate/up B=%d D=%d F=%d" % (B, D, F))


@pytest.mark.parametrize("B,D,F", [(1, 256, 688), (3, 520, 400), (4, 1024, 2048)])
def test_fp8_down_small_shapes(B, D, F):
    L = Fp8Layer(B, D, F, seed=200 + B, norm=False)
    h = (torch.randn(B, F, device="cuda") * 0.5).to(torch.bfloat16)
    y = dfk.dfk_down_proj_fp8(h, L.qd, L.sd)
    torch.cuda.synchronize()
    assert_close(y, L.oracle_down(h), "fp8 down B=%d D=%d F=%d" % (B, D, F))


@pytest.mark.parametrize("B", [1, 3, 8])
def test_every_fp8_gate_up_variant_is_bitwise_identical(B):
    # the CUDA-core family is bitwise invariant; the tensor-core kernel (which
    # the scheduler may pick) is held to the tolerance only
    L = Fp8Layer(B, 384, 1000, seed=300 + B, norm=True, with_down=False)
    ids = [v for v in cc_ids(dfk.DFK_OP_GATE_UP_FP8)
           if v["token_tile"] == bt_for(B, v["j_per_thread"])]
    ref = L.gate_up(True, variant=ids[0]["variant_id"])
    torch.cuda.synchronize()
    assert_close(ref, L.oracle_gate_up(True), "fp8 gate/up reference run")
    ran = 0
    for v in ids:
        if v["token_tile"] != bt_for(B, v["j_per_thread"]):
            continue
        h = try_variant(lambda vid: L.gate_up(True, variant=vid), v["variant_id"])
        if h is None:
            continue
        torch.cuda.synchronize()
        assert bits_equal(h, ref), "variant %d differs" % v["variant_id"]
        ran += 1
    assert ran >= 4


def test_every_fp8_down_variant_is_bitwise_identical():
    B, D, F = 2, 512, 2064
    L = Fp8Layer(B, D, F, seed=310, norm=False)
    h = (torch.randn(B, F, device="cuda")).to(torch.bfloat16)
    # the k split and (when it is above 1) the tiles per stage fix which tiles
    # each team sums, so bits agree within one such pair; across pairs the
    # results are held to the tolerance
    ids = [v for v in cc_ids(dfk.DFK_OP_DOWN_FP8)
           if v["token_tile"] == bt_for(B, v["j_per_thread"])]
    want = L.oracle_down(h)
    refs = {}
    ran = 0
    for v in ids:
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is None:
            continue
        torch.cuda.synchronize()
        assert_close(y, want, "fp8 down variant %d" % v["variant_id"])
        key = (v["k_split"], v["k_tiles_per_stage"] if v["k_split"] > 1 else 0)
        ref = refs.setdefault(key, y)
        assert bits_equal(y, ref), "variant %d differs" % v["variant_id"]
        ran += 1
    assert ran >= 8 and len(refs) >= 2


def test_fp8_rows_do_not_depend_on_batch():
    # CUDA-core family: row b is independent of B for any tile (one variant forced)
    L = Fp8Layer(8, 512, 688, seed=320, norm=True, with_down=False)
    vid = next(v["variant_id"] for v in cc_ids(dfk.DFK_OP_GATE_UP_FP8)
               if v["j_per_thread"] == 2 and v["token_tile"] == 8)
    full = L.gate_up(True, variant=vid)
    for b in (1, 2, 5):
        part = L.gate_up(True, variant=vid, x=L.inp.x[:b].contiguous())
        torch.cuda.synchronize()
        assert bits_equal(part, full[:b].contiguous()), b


def test_fp8_unit_scale_matches_bf16_kernel_on_decoded_weights():
    # with s = 1 the weights the FP8 kernel multiplies by are the decoded codes,
    # which bf16 holds exactly: the bf16 kernel on those weights computes the
    # same sums (in its own order), so the two agree within fp32 rounding
    B, D, F = 2, 512, 688
    L = Fp8Layer(B, D, F, seed=330, norm=False, with_down=False)
    ones = torch.ones(F, dtype=torch.float32, device="cuda")
    h8 = dfk.dfk_swiglu_gate_up_fp8(L.inp.x, L.qg, ones, L.qu, ones)
    wg = L.qg.view(torch.float8_e4m3fn).to(torch.bfloat16)
    wu = L.qu.view(torch.float8_e4m3fn).to(torch.bfloat16)
    h16 = dfk.dfk_swiglu_gate_up(L.inp.x, wg, wu, "row")
    torch.cuda.synchronize()
    a, b = I.bf16_values(h8), I.bf16_values(h16)
    assert np.all(np.abs(a - b) <= 1e-2 + 1e-2 * np.abs(b))
    assert np.mean(a == b) > 0.9


def test_fp8_zero_scale_gives_zero():
    L = Fp8Layer(3, 256, 264, seed=340, norm=True, with_down=False)
    z = torch.zeros_like(L.sg)
    h = dfk.dfk_swiglu_gate_up_fp8(L.inp.x, L.qg, z, L.qu, L.su)
    torch.cuda.synchronize()
    assert not torch.any(h.float() != 0)


def sample_rows(n_total, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, n_total - 1], rng.choice(n_total, n, replace=False)]))
    return rows.astype(np.int32)


@pytest.mark.parametrize("B", [1, 4])
def test_fp8_llama3_8b_full_size_sampled_rows(B):
    # the full Llama-3-8B-shaped layer (d_model 4096, d_ff 14336) in the launch
    # configuration the benchmark uses (scheduler's choice), checked on sampled
    # output rows that the oracle computes one by one
    w = I.WORKLOADS["llama3_8b"]
    L = Fp8Layer(B, w.d_model, w.d_ff, seed=w.seed, norm=True)
    h = L.gate_up(True)
    y = dfk.dfk_down_proj_fp8(h, L.qd, L.sd)
    torch.cuda.synchronize()
    rows = sample_rows(w.d_ff, 192, 7)
    idx = torch.from_numpy(rows).long().cuda()
    assert_close(h[:, idx].contiguous(), L.oracle_gate_up(True, rows=rows),
                 "fp8 8B gate/up rows")
    drows = sample_rows(w.d_model, 128, 8)
    didx = torch.from_numpy(drows).long().cuda()
    assert_close(y[:, didx].contiguous(), L.oracle_down(h, rows=drows), "fp8 8B down rows")


def test_fp8_scheduler_select_variant():
    B, D, F = 2, 1024, 2048
    L = Fp8Layer(B, D, F, seed=350, norm=True)
    h = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
    v = dfk.dfk_select_variant(dfk.DFK_OP_RMSNORM_GATE_UP_FP8, B, D, F, "row",
                               sample=[L.inp.x, L.inp.gamma, L.qg, L.sg, L.qu, L.su, h])
    assert v["family"] == 0 and v["k_tiles_per_stage"] <= 2
    assert dfk.dfk_cached_variant(dfk.DFK_OP_RMSNORM_GATE_UP_FP8, B, D, F)["variant_id"] == \
        v["variant_id"]
    vd = dfk.dfk_select_variant(dfk.DFK_OP_DOWN_FP8, B, D, F, "row")
    assert vd["family"] == 0
    h2 = L.gate_up(True)
    torch.cuda.synchronize()
    assert_close(h2, L.oracle_gate_up(True), "fp8 gate/up after tuning")


# ------------------------------------------------------------------ tensor-core FP8 kernel

def tc_fp8_ids(down):
    """Ids of the widening FP8 tensor-core kernel (one k tile per stage, rows spread)."""
    want = dfk.DFK_OP_DOWN if down else dfk.DFK_OP_GATE_UP
    return [v for v in (dfk.dfk_variant_info(i) for i in range(1, dfk.dfk_variant_count() + 1))
            if v["op"] == want and v["family"] == 1 and v["k_tiles_per_stage"] == 1
            and v["full_m_tiles"] == 0 and v["e4m3_mma"] == 0]


TC_SHAPES = [(1, 256, 688), (2, 144, 200), (5, 400, 1000), (16, 1024, 1496), (17, 272, 96),
             (33, 512, 520), (64, 256, 264)]


@pytest.mark.parametrize("B,D,F", TC_SHAPES)
@pytest.mark.parametrize("norm", [False, True])
def test_fp8_tensor_core_gate_up(B, D, F, norm):
    (v,) = tc_fp8_ids(False)
    L = Fp8Layer(B, D, F, seed=400 + B, norm=norm, with_down=False)
    h = L.gate_up(norm, variant=v["variant_id"])
    torch.cuda.synchronize()
    assert_close(h, L.oracle_gate_up(norm), "fp8 tc gate/up B=%d D=%d F=%d" % (B, D, F))


@pytest.mark.parametrize("B,D,F", [(1, 256, 688), (3, 520, 400), (16, 1024, 2048),
                                   (40, 272, 1024), (64, 384, 2064)])
def test_fp8_tensor_core_down_every_split(B, D, F):
    L = Fp8Layer(B, D, F, seed=410 + B, norm=False)
    h = (torch.randn(B, F, device="cuda") * 0.5).to(torch.bfloat16)
    want = L.oracle_down(h)
    ran = 0
    for v in tc_fp8_ids(True):
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is None:
            continue
        y2 = dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=v["variant_id"])  # counters reset
        torch.cuda.synchronize()
        assert_close(y, want, "fp8 tc down ks=%d B=%d" % (v["k_split"], B))
        assert bits_equal(y, y2), "split-K result not repeatable"
        ran += 1
    assert ran >= 2


def test_fp8_tensor_core_rows_do_not_depend_on_batch_within_a_tile():
    # tokens are columns of one MMA: row b of h does not change with B while
    # the token tile (16) stays the same
    (v,) = tc_fp8_ids(False)
    L = Fp8Layer(16, 512, 688, seed=420, norm=True, with_down=False)
    full = L.gate_up(True, variant=v["variant_id"])
    part = L.gate_up(True, variant=v["variant_id"], x=L.inp.x[:5].contiguous())
    torch.cuda.synchronize()
    assert bits_equal(part, full[:5].contiguous())


@pytest.mark.parametrize("B", [2, 16, 64])
def test_fp8_tensor_core_llama3_8b_sampled_rows(B):
    w = I.WORKLOADS["llama3_8b"]
    L = Fp8Layer(B, w.d_model, w.d_ff, seed=w.seed, norm=True)
    (vg,) = tc_fp8_ids(False)
    h = L.gate_up(True, variant=vg["variant_id"])
    ys = []
    for v in tc_fp8_ids(True):
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is not None:
            ys.append(y)
    torch.cuda.synchronize()
    rows = sample_rows(w.d_ff, 160, 11)
    idx = torch.from_numpy(rows).long().cuda()
    assert_close(h[:, idx].contiguous(), L.oracle_gate_up(True, rows=rows),
                 "fp8 tc 8B gate/up rows B=%d" % B)
    drows = sample_rows(w.d_model, 96, 12)
    didx = torch.from_numpy(drows).long().cuda()
    want = L.oracle_down(h, rows=drows)
    assert ys
    for y in ys:
        assert_close(y[:, didx].contiguous(), want, "fp8 tc 8B down rows B=%d" % B)


def test_fp8_tensor_core_is_exact_dequantisation():
    # unit scales, weights covering every finite E4M3 code: the widening FP8
    # tensor-core kernel must give the bits of the bf16 tensor-core kernel on
    # the decoded weights (same MMA k-slice sequence into one accumulator,
    # same epilogue), so a lost subnormal or a wrong exponent shows up bitwise
    # (no RMSNorm: the bf16 kernel takes r_b from its prep kernel)
    (v,) = tc_fp8_ids(False)
    B, D, F = 4, 512, 688
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    rng = np.random.default_rng(430)
    qg = torch.from_numpy(codes[rng.integers(0, codes.size, (F, D))]).cuda()
    qu = torch.from_numpy(codes[rng.integers(0, codes.size, (F, D))]).cuda()
    ones = torch.ones(F, dtype=torch.float32, device="cuda")
    inp = I.make_inputs(B, D, F, seed=431, norm=True, with_down=False, device="cuda")
    x = (inp.x.float() * 0.05).to(torch.bfloat16)       # keeps |a| moderate
    h8 = dfk.dfk_swiglu_gate_up_fp8(x, qg, ones, qu, ones, variant=v["variant_id"])
    wg = qg.view(torch.float8_e4m3fn).to(torch.bfloat16)
    wu = qu.view(torch.float8_e4m3fn).to(torch.bfloat16)
    h16 = dfk.dfk_swiglu_gate_up(x, wg, wu, "row", variant=v["variant_id"])
    torch.cuda.synchronize()
    assert bits_equal(h8, h16)


# ------------------------------------------------------------------ E4M3-MMA kernel

def e4m3_mma_ids(down, kinds=(1, 2)):
    # kind 1: activation terms from the prep kernel; kind 2: derived inside
    # the kernel (up to 16 tokens)
    want = dfk.DFK_OP_DOWN_FP8 if down else dfk.DFK_OP_GATE_UP_FP8
    return [v for v in (dfk.dfk_variant_info(i) for i in range(1, dfk.dfk_variant_count() + 1))
            if v["op"] == want and v["e4m3_mma"] in kinds]


def test_e4m3_mma_ids_are_fp8_only():
    gu, dn = e4m3_mma_ids(False), e4m3_mma_ids(True)
    assert len(gu) == 4 and len(dn) == 12      # one or two k tiles per stage, both kinds
    x = torch.zeros(2, 256, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(264, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dfk.DfkError) as e:
        dfk.dfk_swiglu_gate_up(x, w, w, "row", variant=gu[0]["variant_id"])
    assert e.value.status == dfk.DFK_ERR_INVALID_ARG


@pytest.mark.parametrize("B,D,F", TC_SHAPES)
@pytest.mark.parametrize("norm", [False, True])
def test_fp8_e4m3_mma_gate_up(B, D, F, norm):
    L = Fp8Layer(B, D, F, seed=500 + B, norm=norm, with_down=False)
    want = L.oracle_gate_up(norm)
    for v in e4m3_mma_ids(False):
        h = try_variant(lambda vid: L.gate_up(norm, variant=vid), v["variant_id"])
        if h is None:
            continue
        torch.cuda.synchronize()
        assert_close(h, want, "fp8 e4m3-mma gate/up nt=%d B=%d D=%d F=%d"
                     % (v["k_tiles_per_stage"], B, D, F))


@pytest.mark.parametrize("B,D,F", [(1, 256, 688), (3, 520, 400), (16, 1024, 2048),
                                   (40, 272, 1024), (64, 384, 2064)])
def test_fp8_e4m3_mma_down_every_split(B, D, F):
    L = Fp8Layer(B, D, F, seed=510 + B, norm=False)
    h = (torch.randn(B, F, device="cuda") * 0.5).to(torch.bfloat16)
    want = L.oracle_down(h)
    ran = 0
    for v in e4m3_mma_ids(True):
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is None:
            continue
        y2 = dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=v["variant_id"])
        torch.cuda.synchronize()
        assert_close(y, want, "fp8 e4m3-mma down ks=%d B=%d" % (v["k_split"], B))
        assert bits_equal(y, y2), "split-K result not repeatable"
        ran += 1
    assert ran >= 2


@pytest.mark.parametrize("norm", [False, True])
def test_fp8_e4m3_mma_encodes_activations_closely(norm):
    # the CUDA-core FP8 kernel multiplies by the exact activations; the E4M3
    # terms (2 for bf16 x, 4 for x * gamma) must leave only accumulation-order
    # and output-rounding differences: within two bf16 steps of each other
    B, D, F = 8, 1024, 1496
    L = Fp8Layer(B, D, F, seed=520 + norm, norm=norm, with_down=False)
    cc = next(w["variant_id"] for w in cc_ids(dfk.DFK_OP_GATE_UP_FP8)
              if w["j_per_thread"] == 2 and w["token_tile"] == 8)
    b = I.bf16_values(L.gate_up(norm, variant=cc))
    for kind in (1, 2):
        v = e4m3_mma_ids(False, kinds=(kind,))[0]
        a = I.bf16_values(L.gate_up(norm, variant=v["variant_id"]))
        torch.cuda.synchronize()
        assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.abs(b) + 1e-4), kind


@pytest.mark.parametrize("B,D,F", [(1, 256, 688), (5, 1024, 1496), (16, 4096, 2048)])
def test_fp8_in_kernel_terms_equal_prep_kernel_terms(B, D, F):
    # without RMSNorm and without a k split both kinds scale by the same
    # power of two (from max |x| over K) and write the same term codes: the
    # tensor cores see identical operands, so the results agree bit for bit
    L = Fp8Layer(B, D, F, seed=530 + B, norm=False, with_down=False)
    for nt in (1, 2):
        ids = [next(v["variant_id"] for v in e4m3_mma_ids(False, kinds=(k,))
                    if v["k_tiles_per_stage"] == nt) for k in (1, 2)]
        outs = [try_variant(lambda vid: L.gate_up(False, variant=vid), vid) for vid in ids]
        if outs[0] is None or outs[1] is None:
            continue
        torch.cuda.synchronize()
        assert bits_equal(outs[0], outs[1]), "nt=%d" % nt


@pytest.mark.parametrize("B,D,F", [(1, 256, 1024), (3, 512, 2208), (8, 384, 4096)])
def test_fp8_split_k_in_kernel_terms_equal_prep_kernel_terms(B, D, F):
    # with a k split both kinds take one power of two per token and slice
    # (from the largest |h| in the slice) and multiply each slice's partial
    # sums by it before the slices are added in order: the same y bit for bit
    L = Fp8Layer(B, D, F, seed=540 + B, norm=False)
    g = torch.Generator(device="cuda").manual_seed(541 + B)
    h = (0.5 * torch.randn(B, F, device="cuda", generator=g)).to(torch.bfloat16)
    h[:, : F // 3] *= 64            # slices of different magnitude
    compared = 0
    for ks in (2, 4):
        for nt in (1, 2):
            pair = {}
            for v in e4m3_mma_ids(True):
                if v["k_split"] == ks and v["k_tiles_per_stage"] == nt:
                    pair[v["e4m3_mma"]] = v["variant_id"]
            run = lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid)
            outs = [try_variant(run, pair[k]) if k in pair else None for k in (1, 2)]
            if outs[0] is None or outs[1] is None:
                continue
            torch.cuda.synchronize()
            assert bits_equal(outs[0], outs[1]), "k split %d, nt %d" % (ks, nt)
            compared += 1
    assert compared >= 2


@pytest.mark.parametrize("B", [1, 16, 64])
def test_fp8_e4m3_mma_llama3_8b_sampled_rows(B):
    w = I.WORKLOADS["llama3_8b"]
    L = Fp8Layer(B, w.d_model, w.d_ff, seed=w.seed, norm=True)
    h = None
    for vg in reversed(e4m3_mma_ids(False)):           # two tiles per stage where it fits
        h = try_variant(lambda vid: L.gate_up(True, variant=vid), vg["variant_id"])
        if h is not None:
            break
    ys = []
    for v in e4m3_mma_ids(True):
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, L.qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is not None:
            ys.append(y)
    torch.cuda.synchronize()
    rows = sample_rows(w.d_ff, 160, 13)
    idx = torch.from_numpy(rows).long().cuda()
    assert_close(h[:, idx].contiguous(), L.oracle_gate_up(True, rows=rows),
                 "fp8 e4m3-mma 8B gate/up rows B=%d" % B)
    drows = sample_rows(w.d_model, 96, 14)
    didx = torch.from_numpy(drows).long().cuda()
    want = L.oracle_down(h, rows=drows)
    assert ys
    for y in ys:
        assert_close(y[:, didx].contiguous(), want, "fp8 e4m3-mma 8B down rows B=%d" % B)


@pytest.mark.parametrize("B", [1, 3, 8])
def test_fp8_in_kernel_terms_capture_on_a_fresh_stream(B):
    # the in-kernel-term variants need no per-stream buffer: captured into a
    # CUDA graph on a stream that never ran them, the replay gives the eager
    # result bit for bit (gate/up with RMSNorm, then the split-K down)
    L = Fp8Layer(B, 1024, 2048, seed=540 + B, norm=True)
    gu = next(v["variant_id"] for v in e4m3_mma_ids(False, kinds=(2,)) if v["k_tiles_per_stage"] == 1)
    dn = next(v["variant_id"] for v in e4m3_mma_ids(True, kinds=(2,)) if v["k_split"] == 4)
    h_ref = L.gate_up(True, variant=gu)
    y_ref = dfk.dfk_down_proj_fp8(h_ref, L.qd, L.sd, variant=dn)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    h = torch.empty_like(h_ref)
    y = torch.empty_like(y_ref)
    # the split-K workspace is per stream: one eager call on the new stream first
    with torch.cuda.stream(s):
        dfk.dfk_down_proj_fp8(h_ref, L.qd, L.sd, y=y, variant=dn)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dfk.dfk_rmsnorm_swiglu_gate_up_fp8(L.inp.x, L.inp.gamma, L.inp.eps, L.qg, L.sg, L.qu,
                                           L.su, h=h, variant=gu, stream=s)
        dfk.dfk_down_proj_fp8(h, L.qd, L.sd, y=y, variant=dn, stream=s)
    h.zero_()
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert bits_equal(h, h_ref)
    assert bits_equal(y, y_ref)
    del g


# ------------------------------------------------------------------ E4M3 terms: wide dynamic range

def _wide_range_tokens(B, D, seed, spread_log2):
    """Activations whose tokens span a wide dynamic range: token 0 has two
    elements at 2^10 and -2^9 and the rest near 2^(10 - spread); token 1 lies
    entirely near 2^-30; token 2 mixes 2^8-sized and 2^(8 - spread)-sized
    halves; the others are N(0, 1)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, D, generator=g)
    sign = torch.where(torch.rand(B, D, generator=g) < 0.5, -1.0, 1.0)
    mag = 1.0 + torch.rand(B, D, generator=g)
    x[0] = sign[0] * mag[0] * 2.0 ** (10 - spread_log2)
    x[0, 17] = 1024.0
    x[0, D // 2] = -512.0
    x[1] = sign[1] * mag[1] * 2.0 ** -30
    x[2, : D // 2] = sign[2, : D // 2] * mag[2, : D // 2] * 2.0 ** 8
    x[2, D // 2:] = sign[2, D // 2:] * mag[2, D // 2:] * 2.0 ** (8 - spread_log2)
    return x.to(torch.bfloat16).cuda()


def _fp8_exact_ids():
    """FP8 gate/up variants that multiply by the exact activations: a
    CUDA-core one and the widening tensor-core one."""
    cc = next(w["variant_id"] for w in cc_ids(dfk.DFK_OP_GATE_UP_FP8)
              if w["j_per_thread"] == 4 and w["token_tile"] == 4)
    return [cc] + [v["variant_id"] for v in tc_fp8_ids(False)][:1]


@pytest.mark.parametrize("norm", [False, True])
def test_e4m3_mma_wide_range_within_the_exact_domain(norm):
    # Tokens spanning 2^13 (inside the 2^14 the two / four E4M3 terms carry
    # exactly), with gamma near the small end of bf16's normal range on a
    # quarter of the channels (x * gamma there is an fp32 subnormal whose
    # contribution is far below any rounding): every E4M3-MMA variant
    # (prep-kernel and in-kernel terms) and the exact-activation kernels
    # match the oracle within the contract tolerance.
    B, D, F = 4, 1024, 1496
    L = Fp8Layer(B, D, F, seed=530 + norm, norm=True, with_down=False)
    L.inp.x.copy_(_wide_range_tokens(B, D, 531, 13))
    gam = L.inp.gamma.clone()
    gam[: D // 4] = (torch.rand(D // 4, device="cuda") + 1.0).to(torch.bfloat16) * 2.0 ** -125
    L.inp.gamma.copy_(gam)
    want = L.oracle_gate_up(norm)
    ran = 0
    for vid in [v["variant_id"] for v in e4m3_mma_ids(False)] + _fp8_exact_ids():
        h = try_variant(lambda v: L.gate_up(norm, variant=v), vid)
        if h is None:
            continue
        torch.cuda.synchronize()
        assert_close(h, want, "wide-range fp8 gate/up variant %d norm=%d" % (vid, norm))
        ran += 1
    assert ran >= 5


@pytest.mark.parametrize("norm", [False, True])
def test_fp8_exact_activation_kernels_beyond_the_e4m3_domain(norm):
    # Tokens spanning 2^22: the kernels that multiply by the exact
    # activations (CUDA-core, widening tensor-core) still meet the contract
    # tolerance.  (The E4M3-MMA variants carry elements more than 2^14 below
    # their token's largest only to about 2^-21 of it; the down-projection
    # test below checks that bound.)
    B, D, F = 4, 1024, 1496
    L = Fp8Layer(B, D, F, seed=532 + norm, norm=True, with_down=False)
    L.inp.x.copy_(_wide_range_tokens(B, D, 533, 22))
    want = L.oracle_gate_up(norm)
    for vid in _fp8_exact_ids():
        h = L.gate_up(norm, variant=vid)
        torch.cuda.synchronize()
        assert_close(h, want, "wide-range fp8 gate/up variant %d norm=%d" % (vid, norm))


def test_e4m3_mma_wide_dynamic_range_down_error_bound():
    # The activation terms carry each element exactly when it lies within
    # 2^14 of its token's largest |value| (two terms for bf16 h: 8 significant
    # bits, the second term's last bit at 2^-13 after the scale that puts the
    # largest in [128, 256)); a smaller element is carried to within 2^-21 of
    # the largest.  Rows whose code at the large elements is zero see only the
    # small elements, so their error shows that bound directly:
    #   |y - oracle| <= 2^-8 |oracle| + 2^-21 max_k|h_k| sum_k |W_jk|
    #                   + 2^-12 sum_k |W_jk h_k|
    # (output rounding, the term representation, and a generous allowance for
    # the MMA's fp32 accumulation over K).
    B, D, F = 4, 512, 2048
    L = Fp8Layer(B, D, F, seed=540, norm=False)
    h = _wide_range_tokens(B, F, 541, 22)
    qd = L.qd.clone()
    qd[0::2, 17] = 0            # even rows: blind to the two large elements of token 0
    qd[0::2, F // 2] = 0
    want = oracle.down_fp8(I.bf16_values(h), L.host(qd), L.host(L.sd))
    hv = np.abs(I.bf16_values(h))
    qv = np.abs(I.fp8_values(qd)) * L.host(L.sd)[:, None]          # |W| per element
    hmax = hv.max(axis=1, keepdims=True)
    bound = (2.0 ** -8 * np.abs(want) + (2.0 ** -21 * hmax) * qv.sum(1)[None, :]
             + 2.0 ** -12 * (hv @ qv.T) + 1e-30)
    ran = 0
    for v in e4m3_mma_ids(True):
        y = try_variant(lambda vid: dfk.dfk_down_proj_fp8(h, qd, L.sd, variant=vid),
                        v["variant_id"])
        if y is None:
            continue
        torch.cuda.synchronize()
        got = I.bf16_values(y)
        assert_close(y, want, "wide-range fp8 down variant %d" % v["variant_id"])
        excess = np.abs(got - want) - bound
        assert (excess <= 0).all(), ("variant %d: error beyond the term bound at %s"
                                     % (v["variant_id"], np.unravel_index(np.argmax(excess),
                                                                         excess.shape)))
        ran += 1
    assert ran >= 4
