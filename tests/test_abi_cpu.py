"""Host-side checks of the C ABI that need no GPU.

The library must load and export every function ``include/dfk.h`` declares;
argument validation must reject bad calls with the documented status codes
before touching the device; without a device every compute call fails
loudly (there is no CPU fallback).
"""
import ctypes
import os
import re

import pytest
import torch

import swiglu_mlp_dfk_b200 as dfk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from swiglu_mlp_dfk_b200 import build
    build.build()
    return dfk.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "dfk.h")).read()
    return sorted(set(re.findall(r"DFK_API\s+[\w\s\*]*?\b(dfk_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions()
    for n in ("dfk_swiglu_gate_up", "dfk_rmsnorm_swiglu_gate_up", "dfk_down_proj",
              "dfk_select_variant"):
        assert n in names
    assert set(names) == set(dfk.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for n in header_functions():
        assert hasattr(L, n), n
    assert dfk.dfk_version().startswith("dfk ")


def test_checked_library_exports_every_declared_symbol(L):
    # the bounds-checked build of the same sources (-DDFK_CHECKED)
    from swiglu_mlp_dfk_b200 import build
    C = ctypes.CDLL(build.LIB_CHECKED)
    for n in header_functions():
        assert hasattr(C, n), n


def test_status_strings(L):
    for s in range(10):
        assert L.dfk_status_string(s).decode()
    assert L.dfk_status_string(99).decode() == "unknown status"


def test_variant_table(L):
    n = dfk.dfk_variant_count()
    assert n >= 8
    ids = set()
    families = set()
    for i in range(1, n + 1):
        v = dfk.dfk_variant_info(i)
        assert v["variant_id"] == i
        families.add(v["family"])
        if v["family"] == 0:      # CUDA-core
            assert v["j_per_thread"] in (2, 4)
            assert v["token_tile"] in (1, 2, 4, 8)
        else:                     # tensor core: token tile 16/32/64 chosen from B
            assert v["family"] == 1 and v["token_tile"] == 64
        assert v["k_tiles_per_stage"] in (1, 2, 4, 8)
        ids.add(i)
    assert families == {0, 1}
    with pytest.raises(dfk.DfkError) as e:
        dfk.dfk_variant_info(n + 1)
    assert e.value.status == dfk.DFK_ERR_INVALID_ARG


# Fake, 16-byte aligned "device" addresses: validation rejects the calls below
# before any CUDA call, so the pointers are never dereferenced.
P = ctypes.c_void_p(0x10000)
P2 = ctypes.c_void_p(0x20000)
P3 = ctypes.c_void_p(0x30000)
MIS = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("call,status", [
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 7, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_LAYOUT),
    (lambda L: L.dfk_swiglu_gate_up(None, P2, P3, 0, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, None, 0, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 2, P, 1, 64, 64, 0, None),   # interleaved + w_up
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 0, P, 65, 64, 64, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 0, P, 1, 60, 64, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 1, P, 1, 64, 60, 0, None),   # col needs F%8
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_swiglu_gate_up(MIS, P2, P3, 0, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 0, P, -1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_swiglu_gate_up(P, P2, P3, 0, P, 1, 64, 64, 9999, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_swiglu_gate_up(P, None, 1e-5, P2, P3, 0, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_swiglu_gate_up(P, P, -1.0, P2, P3, 0, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_down_proj(P, P2, P3, 1, 64, 60, 0, None), dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_down_proj(P, None, P3, 1, 64, 64, 0, None), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_down_proj(P, P2, MIS, 1, 64, 64, 0, None), dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_down_proj(P, P2, P3, 1, 64, 64, 1, None),   # id 1 is a gate/up variant
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_silu(P, P2, -5, None), dfk.DFK_ERR_INVALID_ARG),
    # tensor-parallel group and the emulated call
    (lambda L: L.dfk_tp_group_create(0, 0, 4, 64, ctypes.byref(ctypes.c_void_p()),
                                     ctypes.create_string_buffer(64)), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_tp_group_create(2, 2, 4, 64, ctypes.byref(ctypes.c_void_p()),
                                     ctypes.create_string_buffer(64)), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_tp_group_create(2, 0, 65, 64, ctypes.byref(ctypes.c_void_p()),
                                     ctypes.create_string_buffer(64)),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_tp_down_proj_allreduce(None, P, P2, P3, 1, 64, 64, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_tp_down_proj_allreduce_emulated(9, P, P2, P3, 1, 64, 64, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_tp_down_proj_allreduce_emulated(2, P, P2, P3, 65, 64, 64, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    # one-launch decode step
    (lambda L: L.dfk_mlp_stack_step(P, 1e-5, P2, P3, 0, P2, P, P, P, None, 1 << 20, 2, 4, 64,
                                    64, None), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_mlp_stack_step(P, 1e-5, P2, P3, 0, P2, MIS, P, P, P, 1 << 20, 2, 4, 64,
                                    64, None), dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_mlp_stack_step(P, -1.0, P2, P3, 0, P2, P, P, P, P, 1 << 20, 2, 4, 64, 64,
                                    None), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_mlp_stack_step(P, 1e-5, P2, P3, 0, P2, P, P, P, P, -1, 2, 4, 64, 64, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_mlp_stack_step(P, 1e-5, P2, P3, 2, P2, P, P, P, P, 1 << 20, 2, 4, 64, 64,
                                    None), dfk.DFK_ERR_UNSUPPORTED_LAYOUT),
    # the bounded-wait self-test
    (lambda L: L.dfk_selftest_bounded_wait(None, None), dfk.DFK_ERR_INVALID_ARG),
    # FP8 weights: reduction length % 16, null scales, misaligned scales, tensor-core ids
    (lambda L: L.dfk_swiglu_gate_up_fp8(P, P2, P3, P2, P3, P, 1, 72, 64, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_swiglu_gate_up_fp8(P, P2, None, P2, P3, P, 1, 64, 64, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_swiglu_gate_up_fp8(P, P2, P3, P2, ctypes.c_void_p(0x30002), P, 1, 64, 64,
                                        0, None), dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_swiglu_gate_up_fp8(P, P2, P3, P2, P3, P, 65, 64, 64, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_rmsnorm_swiglu_gate_up_fp8(P, None, 1e-5, P2, P3, P2, P3, P, 1, 64, 64, 0,
                                                None), dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_swiglu_gate_up_fp8(P, P, 1e-5, P2, P3, P2, P3, P, 1, 64, 64,
                                                dfk.dfk_variant_count(), None),
     dfk.DFK_ERR_INVALID_ARG),                              # last id: a tensor-core GEMV
    (lambda L: L.dfk_down_proj_fp8(P, P2, P3, P, 1, 64, 72, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_down_proj_fp8(P, MIS, P3, P, 1, 64, 64, 0, None), dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_down_proj_fp8(P, P2, P3, P, 1, 64, 64, 1, None),   # gate/up id
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_select_variant(dfk.DFK_OP_DOWN_FP8, 1, 64, 64, 1, None, None,
                                    ctypes.byref(dfk.dfk_variant())),
     dfk.DFK_ERR_UNSUPPORTED_LAYOUT),
    # packed QKV: part sizes, null parts, misaligned parts, eps, bf16-only ids
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, P3, P3, 1, 64, -1, 8, 8, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, P3, P3, 1, 64, 0, 0, 0, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, None, P3, 1, 64, 8, 8, 8, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, MIS, P3, 1, 64, 8, 8, 8, 0, None),
     dfk.DFK_ERR_MISALIGNED),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, -1.0, P2, P3, P3, P3, 1, 64, 8, 8, 8, 0, None),
     dfk.DFK_ERR_INVALID_ARG),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, P3, P3, 1, 60, 8, 8, 8, 0, None),
     dfk.DFK_ERR_UNSUPPORTED_SHAPE),
    (lambda L: L.dfk_rmsnorm_qkv_proj(P, P, 1e-5, P2, P3, P3, P3, 1, 64, 8, 8, 8, 1, None),
     dfk.DFK_ERR_INVALID_ARG),                                   # id 1: a gate/up variant
    (lambda L: L.dfk_select_variant(9, 1, 64, 64, 0, None, None, None), dfk.DFK_ERR_INVALID_ARG),
])
def test_validation_rejects_without_launch(L, call, status):
    assert call(L) == status
    assert L.dfk_last_error().decode() != ""


def test_empty_batch_is_a_no_op(L):
    assert L.dfk_swiglu_gate_up(None, P2, P3, 0, None, 0, 64, 64, 0, None) == dfk.DFK_OK
    assert L.dfk_down_proj(None, P2, None, 0, 64, 64, 0, None) == dfk.DFK_OK
    assert L.dfk_silu(None, None, 0, None) == dfk.DFK_OK
    assert L.dfk_swiglu_gate_up_fp8(None, P2, P3, P2, P3, None, 0, 64, 64, 0, None) == dfk.DFK_OK
    assert L.dfk_down_proj_fp8(None, P2, P3, None, 0, 64, 64, 0, None) == dfk.DFK_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device behaviour")
def test_no_device_means_no_compute(L):
    # valid-looking arguments, but no CUDA device: the library refuses (no CPU fallback)
    assert L.dfk_swiglu_gate_up(P, P2, P3, 0, P, 1, 64, 64, 0, None) == dfk.DFK_ERR_ARCH
    assert L.dfk_down_proj(P, P2, P3, 1, 64, 64, 0, None) == dfk.DFK_ERR_ARCH
    code = ctypes.c_int(0)
    assert L.dfk_device_error(ctypes.byref(code)) == dfk.DFK_ERR_ARCH
    with pytest.raises(dfk.DfkError):
        dfk.dfk_device_error()


def test_python_binding_rejects_host_tensors():
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    with pytest.raises(dfk.DfkError):
        dfk.dfk_swiglu_gate_up(x, torch.zeros(64, 64, dtype=torch.bfloat16),
                               torch.zeros(64, 64, dtype=torch.bfloat16))


def test_stack_tuning_candidates(L):
    # the in-context tuner's candidate lists (host logic only): the library's
    # own choice first, then the tensor-core variants of the call's class;
    # E4M3-MMA variants only for the FP8 stack
    import types
    from swiglu_mlp_dfk_b200.stack import DecodeStack
    for fp8 in (False, True):
        fake = types.SimpleNamespace(fp8=fp8)
        for gate_up in (True, False):
            c = DecodeStack._candidates(fake, gate_up)
            assert c[0] == 0 and len(c) == len(set(c)) > 1
            for i in c[1:]:
                v = dfk.dfk_variant_info(i)
                assert v["family"] == 1
                assert (v["op"] in (dfk.DFK_OP_GATE_UP, dfk.DFK_OP_GATE_UP_FP8)) == gate_up
                assert fp8 or v["e4m3_mma"] == 0
            has_e4m3 = any(dfk.dfk_variant_info(i)["e4m3_mma"] for i in c[1:])
            assert has_e4m3 == fp8


def test_header_is_plain_c_and_links(L, tmp_path):
    # a C program (no C++, no torch) includes dfk.h, links against libdfk.so and
    # the CUDA runtime, and runs: without a device the entry points return a
    # status (here: invalid argument for the null buffers), never crash
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if gcc is None or not os.path.exists(os.path.join(cuda, "include", "cuda_runtime.h")):
        pytest.skip("needs gcc and the CUDA headers")
    src = tmp_path / "app.c"
    src.write_text(r'''
#include <stdio.h>
#include "dfk.h"
int main(void) {
  int st = dfk_rmsnorm_swiglu_gate_up(0, 0, 1e-5f, 0, 0, DFK_W_ROW_MAJOR, 0, 1, 4096, 14336,
                                      0, 0);
  printf("%d %s\n", st, dfk_status_string(st));
  return st == DFK_ERR_INVALID_ARG ? 0 : 1;
}
''')
    exe = tmp_path / "app"
    pkg = os.path.dirname(dfk.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", pkg, "-ldfk", "-Wl,-rpath," + pkg, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.split()[0] == str(dfk.DFK_ERR_INVALID_ARG)
