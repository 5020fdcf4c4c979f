"""GPU parity for the RMSNorm + packed QKV projection, through the C ABI,
against the fp64 oracle (tolerance |gpu - oracle| <= 1e-2 + 1e-2 |oracle|).

The packed projection is one GEMV over W_qkv = [W_q; W_k; W_v] whose output
rows are routed to q, k and v ("Optimizing QKV Projection with Operator
Fusion", section "Implementing Fusion: Packed Projections")."""
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
    bad = err > ATOL + RTOL * np.abs(w)
    if bad.any():
        i = np.unravel_index(np.argmax(err - (ATOL + RTOL * np.abs(w))), err.shape)
        raise AssertionError("%s: %d/%d out of tolerance; worst at %s: gpu %r oracle %r"
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


def layer(B, D, nq, nk, nv, seed, w_std=0.05):
    g = I.make_generator(seed, "cuda")
    x = (torch.randn(B, D, generator=g, device="cuda")).to(torch.bfloat16)
    gamma = (1.0 + 0.1 * torch.randn(D, generator=g, device="cuda")).to(torch.bfloat16)
    w = (w_std * torch.randn(nq + nk + nv, D, generator=g, device="cuda")).to(torch.bfloat16)
    return x, gamma, w


def oracle_qkv(x, gamma, w, nq, nk, nv, norm, rows=None):
    return oracle.qkv(I.to_bits(x), I.to_bits(w), nq, nk, nv,
                      gamma=I.to_bits(gamma) if norm else None, eps=1e-5, rows=rows)


def gemv_ids():
    return [dfk.dfk_variant_info(i) for i in range(1, dfk.dfk_variant_count() + 1)
            if dfk.dfk_variant_info(i)["op"] == dfk.DFK_OP_DOWN]


def bt_for(B, jpt):
    return min(1 << max(B - 1, 0).bit_length(), 4 if jpt == 4 else 8)


SHAPES = [(1, 256, 256, 64, 64), (3, 320, 200, 40, 40), (8, 512, 512, 128, 128),
          (17, 128, 96, 32, 32), (40, 256, 256, 64, 64), (64, 384, 384, 96, 96)]


@pytest.mark.parametrize("B,D,nq,nk,nv", SHAPES)
@pytest.mark.parametrize("norm", [False, True])
def test_qkv_every_variant_matches_oracle(B, D, nq, nk, nv, norm):
    x, gamma, w = layer(B, D, nq, nk, nv, seed=600 + B + D)
    want = oracle_qkv(x, gamma, w, nq, nk, nv, norm)
    ran, refs = 0, {}
    for v in [None] + gemv_ids():
        if v is not None and v["family"] == 0 and v["token_tile"] != bt_for(B, v["j_per_thread"]):
            continue
        vid = 0 if v is None else v["variant_id"]
        try:
            outs = dfk.dfk_rmsnorm_qkv_proj(x, gamma if norm else None, 1e-5, w, nq, nk, nv,
                                            variant=vid)
        except dfk.DfkError as e:
            assert e.status == dfk.DFK_ERR_NO_VARIANT
            continue
        torch.cuda.synchronize()
        for got, ref, name in zip(outs, want, "qkv"):
            assert_close(got, ref, "%s variant %d norm %d B=%d" % (name, vid, norm, B))
        if v is not None and v["family"] == 0:
            # CUDA-core: bits fixed by (k split, tiles per stage when split)
            key = (v["k_split"], v["k_tiles_per_stage"] if v["k_split"] > 1 else 0)
            packed = torch.cat(outs, dim=1)
            ref = refs.setdefault(key, packed)
            assert bits_equal(packed, ref), "variant %d" % vid
        ran += 1
    assert ran >= 4


def test_qkv_empty_part_and_empty_batch():
    B, D, nq, nk, nv = 2, 256, 128, 0, 64
    x, gamma, w = layer(B, D, nq, nk, nv, seed=610)
    q, k, v = dfk.dfk_rmsnorm_qkv_proj(x, gamma, 1e-5, w, nq, nk, nv)
    torch.cuda.synchronize()
    wq, _, wv = oracle_qkv(x, gamma, w, nq, nk, nv, True)
    assert k.shape == (B, 0)
    assert_close(q, wq, "q")
    assert_close(v, wv, "v")
    x0 = torch.empty(0, D, dtype=torch.bfloat16, device="cuda")
    outs = dfk.dfk_rmsnorm_qkv_proj(x0, gamma, 1e-5, w, nq, nk, nv)
    assert outs[0].shape == (0, nq)


def test_qkv_rows_do_not_depend_on_batch():
    x, gamma, w = layer(8, 512, 256, 64, 64, seed=620)
    vid = next(v["variant_id"] for v in gemv_ids()
               if v["family"] == 0 and v["j_per_thread"] == 2 and v["token_tile"] == 8
               and v["k_split"] == 1)
    full = torch.cat(dfk.dfk_rmsnorm_qkv_proj(x, gamma, 1e-5, w, 256, 64, 64, variant=vid), 1)
    for b in (1, 3):
        part = torch.cat(dfk.dfk_rmsnorm_qkv_proj(x[:b].contiguous(), gamma, 1e-5, w, 256, 64, 64,
                                                  variant=vid), 1)
        torch.cuda.synchronize()
        assert bits_equal(part, full[:b].contiguous())


def sample_rows(n_total, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, n_total - 1],
                                     rng.choice(n_total, n, replace=False)])).astype(np.int32)


@pytest.mark.parametrize("B", [1, 16, 64])
def test_qkv_llama3_8b_sampled_rows(B):
    # Llama-3-8B attention input projection: d_model 4096, 32 query heads and
    # 8 key/value heads of 128 -> n_q 4096, n_k = n_v = 1024 (shapes only)
    D, nq, nk, nv = 4096, 4096, 1024, 1024
    x, gamma, w = layer(B, D, nq, nk, nv, seed=630 + B, w_std=0.02)
    outs = dfk.dfk_rmsnorm_qkv_proj(x, gamma, 1e-5, w, nq, nk, nv)
    torch.cuda.synchronize()
    packed = torch.cat(outs, dim=1)
    rows = sample_rows(nq + nk + nv, 192, B)
    idx = torch.from_numpy(rows).long().cuda()
    assert_close(packed[:, idx].contiguous(), oracle_qkv(x, gamma, w, nq, nk, nv, True, rows=rows),
                 "8B qkv rows B=%d" % B)
