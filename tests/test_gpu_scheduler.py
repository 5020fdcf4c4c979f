"""Scheduler on the GPU: the persistent tune cache round-trips, survives a
corrupted file, and a failure of the timing step (host-side fault injection,
DFK_FAULT=tune) falls back to the heuristic choice with correct results.
Each case runs in a fresh process, because the cache is read once per
process and device."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, json
sys.path.insert(0, %r)
import numpy as np, torch
import oracle
import swiglu_mlp_dfk_b200 as dfk
from swiglu_mlp_dfk_b200 import inputs as I
inp = I.make_inputs(2, 512, 1024, seed=3, with_down=True, device="cuda")
h = dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, inp.w_gate, inp.w_up, "row")
y = dfk.dfk_down_proj(h, inp.w_down)
torch.cuda.synchronize()
ref = oracle.gate_up(I.to_bits(inp.x), I.to_bits(inp.w_gate), I.to_bits(inp.w_up),
                     gamma=I.to_bits(inp.gamma), eps=inp.eps)
err = np.abs(I.bf16_values(h) - ref) - (1e-2 + 1e-2 * np.abs(ref))
v = dfk.dfk_cached_variant(1, 2, 512, 1024, "row")
print(json.dumps({"ok": bool((err <= 0).all()), "variant": v["variant_id"],
                  "us": v["measured_us"], "dev_err": dfk.dfk_device_error()}))
""" % ROOT


def run_child(env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    import json
    return json.loads(r.stdout.strip().splitlines()[-1]), r.stderr


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_tune_cache_round_trip(tmp_path):
    cache = str(tmp_path / "tune.txt")
    first, _ = run_child({"DFK_TUNE_CACHE": cache})
    assert first["ok"] and first["dev_err"] == 0 and first["us"] > 0
    lines = open(cache).read().splitlines()
    assert len(lines) == 2 and all(l.startswith("dfk-tune 1 ") for l in lines)
    second, _ = run_child({"DFK_TUNE_CACHE": cache})
    assert second["ok"] and second["variant"] == first["variant"]
    assert abs(second["us"] - first["us"]) < 1e-2          # read back, not re-timed
    assert len(open(cache).read().splitlines()) == 2       # nothing new appended


def test_corrupted_tune_cache_is_ignored(tmp_path):
    cache = str(tmp_path / "tune.txt")
    with open(cache, "w") as f:
        f.write("not a tune line\n")
        f.write("dfk-tune 1 NVIDIA_B200 148 1 1 2 512 1024 0 99999 1.0\n")   # bad id/driver
        f.write("dfk-tune 7 x\n")
    res, err = run_child({"DFK_TUNE_CACHE": cache, "DFK_LOG": "1"})
    assert res["ok"] and res["dev_err"] == 0
    assert "malformed" in err


def test_fault_injection_falls_back_to_heuristic(tmp_path):
    # a cache of its own: a cache file named by the environment may already
    # hold a timed decision for this shape
    res, _ = run_child({"DFK_FAULT": "tune", "DFK_TUNE_CACHE": str(tmp_path / "tune.txt")})
    assert res["ok"] and res["dev_err"] == 0
    assert res["us"] < 0            # chosen without timing
