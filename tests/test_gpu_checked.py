"""The bounds-checked build (-DDFK_CHECKED, libdfk_checked.so): every kernel
family runs with its result stores and activation loads tested against the
tensors' extents.  Run in a child process with DFK_CHECKED=1 (the binding
then loads the checked library): the results still match the fp64 oracle
and no check fails (the device status word stays clear)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
sys.path.insert(0, os.environ["DFK_ROOT"])
import numpy as np, torch
import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I, tp
from swiglu_mlp_dfk_b200.stack import PersistentDecodeStack
assert dfk.LIB_PATH.endswith("libdfk_checked.so"), dfk.LIB_PATH

def close(got, want, rtol=1e-2):
    g = I.bf16_values(got)
    assert np.all(np.abs(g - want) <= 1e-2 + rtol * np.abs(want)), float(np.max(np.abs(g - want)))

def ids(op, family):
    return [i for i in range(1, dfk.dfk_variant_count() + 1)
            if dfk.dfk_variant_info(i)["op"] == op and dfk.dfk_variant_info(i)["family"] == family
            and not dfk.dfk_variant_info(i)["e4m3_mma"]]

dfk.dfk_device_error()
for B, D, F in [(1, 256, 688), (5, 320, 1000), (16, 512, 776), (40, 256, 264)]:
    inp = I.make_inputs(B, D, F, seed=B, w_std=0.05, device="cuda")
    ref = oracle.gate_up(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                         gamma=I.to_bits(inp.gamma), eps=inp.eps)
    for layout in (I.LAYOUT_ROW, I.LAYOUT_COL, I.LAYOUT_INTERLEAVED):
        wg, wu = I.to_layout(inp.w_gate, inp.w_up, layout)
        for vid in [0] + ids(dfk.DFK_OP_GATE_UP, 0)[:3] + ids(dfk.DFK_OP_GATE_UP, 1):
            try:
                h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, layout,
                                                   variant=vid)
            except dfk.DfkError as e:
                assert e.status == dfk.DFK_ERR_NO_VARIANT
                continue
            torch.cuda.synchronize()
            close(h, ref)
    h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up, "row")
    yref = oracle.down(I.to_bits(h), I.to_bits(inp.w_down))
    for vid in [0] + ids(dfk.DFK_OP_DOWN, 1):
        try:
            y = dfk.dfk_down_proj(h, inp.w_down, variant=vid)
        except dfk.DfkError as e:
            assert e.status == dfk.DFK_ERR_NO_VARIANT
            continue
        torch.cuda.synchronize()
        close(y, yref)
    # FP8 weights, every family through the scheduler and forced E4M3-MMA ids
    qg, sg = I.to_fp8_rows(inp.w_gate); qu, su = I.to_fp8_rows(inp.w_up)
    if D % 16 == 0:
        ref8 = oracle.gate_up_fp8(I.to_bits(inp.x), qg.cpu().numpy(), sg.cpu().numpy(),
                                  qu.cpu().numpy(), su.cpu().numpy(), gamma=I.to_bits(inp.gamma),
                                  eps=inp.eps)
        for i in range(1, dfk.dfk_variant_count() + 1):
            v = dfk.dfk_variant_info(i)
            if v["op"] != dfk.DFK_OP_GATE_UP_FP8 or not v["e4m3_mma"]:
                continue
            try:
                h8 = dfk.dfk_rmsnorm_swiglu_gate_up_fp8(inp.x, inp.gamma, inp.eps, qg, sg, qu, su,
                                                        variant=i)
            except dfk.DfkError as e:
                assert e.status == dfk.DFK_ERR_NO_VARIANT
                continue
            torch.cuda.synchronize()
            close(h8, ref8)
    # packed QKV with RMSNorm (the prep kernel's stores)
    w = (torch.randn(96, D, device="cuda") * 0.05).to(torch.bfloat16)
    q, k, v = dfk.dfk_rmsnorm_qkv_proj(inp.x, inp.gamma, inp.eps, w, 64, 16, 16)
    o = oracle.qkv(I.to_bits(inp.x), I.to_bits(w), 64, 16, 16, gamma=I.to_bits(inp.gamma),
                   eps=inp.eps)
    torch.cuda.synchronize()
    close(q, o[0]); close(k, o[1]); close(v, o[2])
# tensor-parallel emulated group and the one-launch decode step
inp = I.make_inputs(4, 512, 2048, seed=9, w_std=0.03, device="cuda")
y_all, _ = tp.emulated_forward(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up, inp.w_down,
                               I.LAYOUT_ROW, 4)
_, y_ref = oracle.mlp(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                      I.to_bits(inp.w_down), gamma=I.to_bits(inp.gamma), eps=inp.eps)
torch.cuda.synchronize()
close(y_all[2], y_ref)
x0, params = I.make_stack(2, 4, 512, 1024, seed=3, w_std=0.03, device="cuda")
ps = PersistentDecodeStack(params, x0)
ps.step_eager()
torch.cuda.synchronize()
g0, wg0, wu0, wd0 = params[0]
close(ps.h_all[0], oracle.gate_up(I.to_bits(x0), I.to_bits(wg0), I.to_bits(wu0),
                                  gamma=I.to_bits(g0), eps=1e-5))
st, code, text = dfk.dfk_device_status()
assert st == dfk.DFK_OK and code == 0, (st, code, text)
print("CHECKED_OK")
'''


def test_checked_build_runs_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from swiglu_mlp_dfk_b200 import build
    build.build()
    env = dict(os.environ, DFK_CHECKED="1", DFK_ROOT=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "CHECKED_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
