#!/usr/bin/env python
"""Benchmark: decode-stage SwiGLU MLP layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dfk|reference] [--quick]

One step = one pass of the hot path over one decode batch of a
Llama-3-8B-shaped MLP layer (B = 1, d_model 4096, d_ff 14336, bf16 weights
~N(0, 0.02), x ~N(0, 1), gamma = 1 + N(0, 0.1), seed 1, row-major weights):
the fused RMSNorm + gate/up + SiLU * up kernel followed by the separate
down-projection kernel.  Inputs are synthetic and resident in HBM; two
weight copies are used in rotation (705 MB, more than 5x the 126 MB L2) so
no step reads weights the previous step left in L2.

Printed (rank 0, one JSON line): whole-job achieved HBM GB/s over the
algorithmic bytes of the step (the metric is "fused gate/up us/call &
achieved HBM GB/s (% of B200 roofline) at batch 1-64"), the gate/up
kernel's us/call and roofline fraction, the end-to-end figure through the
host-memory C entry point, the batch sweep B = 1..64 (row- vs column-major,
scheduler's choice), the fused-vs-unfused speedup and the CPU oracle
baseline.  ``--impl reference`` times the fp64 CPU oracle on the same
workload instead.  Under torchrun every rank runs an independent replica on
its own GPU (the decode MLP does not shard across data-parallel replicas):
value = bytes of all ranks / max-over-ranks time.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused gate/up µs/call & achieved HBM GB/s (% of B200 roofline) at batch 1–64"
UNIT = "GB/s"
# The B200's HBM3e specification figure; fractions against it are reported
# beside the ones against the measured copy bandwidth.
NOMINAL_HBM_GBS = 8000.0
B1, D, F = 1, 4096, 14336
SEED = 1
FALLBACK_HBM_GBS = 6650.0


def gate_up_bytes(B, D, F):
    """Algorithmic bytes of the fused gate/up call: both weight matrices once,
    x, gamma, and h written once (bf16)."""
    return 2 * F * D * 2 + B * D * 2 + D * 2 + B * F * 2


def down_bytes(B, D, F):
    return D * F * 2 + B * F * 2 + B * D * 2


def step_bytes(B, D, F):
    return gate_up_bytes(B, D, F) + down_bytes(B, D, F)


def config_dict(parallelism):
    return {"workload": "llama3_8b_mlp_layer_decode", "B": B1, "d_model": D, "d_ff": F,
            "layout": "row", "rmsnorm": True, "seed": SEED,
            "step": "fused RMSNorm+gate/up+SiLU*up kernel, then down-projection kernel",
            "global_batch": B1, "seq_len": 1, "parallelism": parallelism,
            "l2": "inputs larger than L2: 2 rotating weight copies (705 MB vs 126 MB L2)"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def engine_source_hash():
    h = hashlib.sha256()
    for rel in ("swiglu_mlp_dfk_b200/csrc/cc_engine.cuh", "swiglu_mlp_dfk_b200/csrc/ptx.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per gate/up launch from the committed ncu summary, if it was
    taken on the kernel source as it is now; else None."""
    p = os.path.join(ROOT, "profiles", "gate_up_llama3_8b_b1.md")
    try:
        text = open(p).read()
    except OSError:
        return None
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    m_h = re.search(r"engine_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != engine_source_hash():
        return None
    return int(m_b.group(1))


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_dev):
        self.samples = []
        self.phase = "idle"
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[torch_dev]) if vis and vis.split(",")[0].isdigit() \
                    else torch_dev
                self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)

    def _reasons(self):
        nv = self.nv
        for name in ("nvmlDeviceGetCurrentClocksEventReasons",
                     "nvmlDeviceGetCurrentClocksThrottleReasons"):
            fn = getattr(nv, name, None)
            if fn:
                return fn(self.h)
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                self.samples.append((self.phase, mhz, self._reasons()))
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, phase="timed"):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        sel = [s for s in self.samples if s[0] == phase]
        note = "sampled during the timed region"
        if len(sel) < 3:
            sel = [s for s in self.samples if s[0] in ("warmup", "timed", "extra")]
            note = "timed region shorter than the sampling period: warm-up, timed and " \
                   "follow-on measurements pooled"
        mhz = [s[1] for s in sel]
        bits = 0
        for s in sel:
            bits |= s[2]
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel), "note": note}


# ---------------------------------------------------------------- replicas

def max_over_ranks(value, dist=None, device=None):
    """Largest `value` over all ranks of the default process group (a
    device-side time: the job ends when the slowest replica ends)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(bytes_per_step, steps, world, t_max_ms):
    """Whole-job GB/s of `world` independent replicas that each ran `steps`
    steps of `bytes_per_step` algorithmic bytes, the slowest taking t_max_ms."""
    return bytes_per_step * steps * world / (t_max_ms / 1e3) / 1e9


# ---------------------------------------------------------------- GPU arm

def gpu_arm(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()

    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import build as kbuild
    from swiglu_mlp_dfk_b200 import inputs as I

    if rank == 0 or not os.path.exists(kbuild.LIB):
        kbuild.build()
    if world > 1:
        dist.barrier()
    dfk.lib()
    dfk.dfk_device_error()

    inp = I.make_inputs(B1, D, F, seed=SEED, w_std=0.02, norm=True, with_down=True,
                        device="cuda")
    copies = [(inp.w_gate, inp.w_up, inp.w_down),
              (inp.w_gate.clone(), inp.w_up.clone(), inp.w_down.clone())]
    h = torch.empty(B1, F, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(B1, D, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        wg, wu, wd = copies[i % len(copies)]
        dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, "row", h=h)
        dfk.dfk_down_proj(h, wd, y=y)

    clocks = ClockSampler(dev)
    clocks.start()
    clocks.phase = "warmup"
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- timed region: K back-to-back steps (events only at its ends, so the
    # kernels' programmatic dependent launch overlaps each prologue with the
    # previous kernel's tail, as in a decode loop)
    K = args.steps
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.phase = "timed"
    ev0.record(stream)
    for i in range(K):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks.phase = "extra"
    if world > 1:
        dist.barrier()
    total_ms = ev0.elapsed_time(ev1)
    t_max = max_over_ranks(total_ms, dist, "cuda")
    value = replica_throughput(step_bytes(B1, D, F), K, world, t_max)

    # ---- the dominant kernel alone: K back-to-back fused gate/up launches
    # (average launch duration = elapsed / K), and the down projection alone
    def kernel_avg_us(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1000.0 / n

    def gate_up_call(i):
        wg, wu, _ = copies[i % len(copies)]
        dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, "row", h=h)

    # the down projection alone rotates 8 copies of W_down (940 MB): with two
    # (235 MB) the L2 still held part of the copy read two calls earlier
    down_ws = [c[2] for c in copies] + [copies[0][2].clone() for _ in range(6)]

    def down_call(i):
        dfk.dfk_down_proj(h, down_ws[i % len(down_ws)], y=y)

    clocks.phase = "timed"
    gu_avg = kernel_avg_us(gate_up_call, K)
    dn_avg = kernel_avg_us(down_call, K)
    clocks.phase = "extra"
    # single launches bracketed by events (no overlap with a neighbour)
    single = []
    for i in range(20):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gate_up_call(i)
        b.record(stream)
        single.append((a, b))
    torch.cuda.synchronize()
    gu_single = statistics.median(a.elapsed_time(b) * 1000.0 for a, b in single)
    peak, peak_src = measured_peaks()
    achieved = gate_up_bytes(B1, D, F) / (gu_avg * 1e-6) / 1e9

    # ---- end to end through the host-memory C entry point
    x_host = inp.x.cpu().pin_memory()
    y_host = torch.empty(B1, D, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(inp.x)
    Ke = max(1, min(K, 500))
    for i in range(3):
        wg, wu, wd = copies[i % 2]
        dfk.dfk_mlp_forward_host(x_host, inp.gamma, inp.eps, wg, wu, "row", wd, y_host, x_dev,
                                 h, y)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    t0 = time.perf_counter()
    for i in range(Ke):
        wg, wu, wd = copies[i % 2]
        dfk.dfk_mlp_forward_host(x_host, inp.gamma, inp.eps, wg, wu, "row", wd, y_host, x_dev,
                                 h, y)
    e1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    e2e_ms = max_over_ranks(max(e0.elapsed_time(e1), wall * 1e3), dist, "cuda")
    e2e_value = replica_throughput(step_bytes(B1, D, F), Ke, world, e2e_ms)

    extra = {}
    if world == 1 and not args.quick:
        # single-GPU characterisation (sweeps, 70B layer, decode stack); with
        # several replicas only the headline line is printed
        extra = extra_measurements(args, inp, copies, h, y, down_ws)
    clocks.stop()
    err = dfk.dfk_device_error()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t_max / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict("replicas%d" % world if world > 1 else "single-gpu"),
        "gate_up_us_per_call": round(gu_avg, 2), "gate_up_us_single_launch": round(gu_single, 2),
        "gate_up_GBps": round(achieved, 1), "down_us_per_call": round(dn_avg, 2),
        "down_GBps": round(down_bytes(B1, D, F) / (dn_avg * 1e-6) / 1e9, 1),
        "step_alg_bytes": step_bytes(B1, D, F),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_nominal_8tbps": round(achieved / NOMINAL_HBM_GBS, 4),
                     "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s",
                     "traffic": profiled_traffic(),
                     "kernel": "fused RMSNorm+gate/up (CUDA-core, TMA ring)",
                     "alg_bytes_per_launch": gate_up_bytes(B1, D, F),
                     "duration": "average of %d back-to-back launches (CUDA events)" % K},
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": B1 * D * 2, "d2h_bytes_per_step": B1 * D * 2,
                "ms_per_step": round(e2e_ms / Ke, 5), "steps": Ke,
                "path": "dfk_mlp_forward_host: pinned x -> device, gate/up, down, y -> host"},
        "gpu_launches": 2 * K,
        "gpu_launches_note": "timed step loop only; the kernel-alone loops add 2K more",
        "clocks": clocks.summary("timed"),
        "device_error_word": err,
    }
    line.update(extra)
    if world == 1:
        line["cpu_baseline"] = cpu_baseline()
    if "batch_sweep" in line:
        # last key, so that a reader keeping only the end of the line still
        # has the B = 1..64 gate/up figures (fraction of the measured peak)
        sw = line["batch_sweep"]
        compact = {
            "B": [r["B"] for r in sw],
            "row_us": [r["row"]["us"] for r in sw], "col_us": [r["col"]["us"] for r in sw],
            "row_frac": [r["row"]["frac"] for r in sw], "col_frac": [r["col"]["frac"] for r in sw],
            "family": ["%s/%s" % (r["row"]["family"], r["col"]["family"]) for r in sw]}
        # the other operations' sweeps, fractions of the measured peak
        if "down_sweep" in line:
            compact["down_frac"] = [r["frac"] for r in line["down_sweep"]]
        if "qkv_projection" in line:
            q = line["qkv_projection"]["sweep"]
            compact["qkv_B"] = [r["B"] for r in q]
            compact["qkv_frac"] = [r["fused_frac"] for r in q]
        if "fp8_weights" in line:
            f8 = line["fp8_weights"]["sweep"]
            compact["fp8_B"] = [r["B"] for r in f8]
            compact["fp8_gate_up_frac"] = [r["gate_up_frac"] for r in f8]
            compact["fp8_down_frac"] = [r["down_frac"] for r in f8]
        line["batch_sweep_compact"] = compact
    return line


def timed_us(fn, reps, flush=None, warm=3):
    """Mean duration of `reps` back-to-back calls, in us.  `warm` untimed calls
    run first (after the optional L2 flush, whose dirty lines they write back),
    so the timed calls see the steady state; every caller rotates weight copies
    whose total exceeds L2, so no timed call finds its weights cached."""
    import torch
    if flush is not None:
        flush.add_(1)
    for i in range(warm):
        fn(reps + i)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        fn(i)
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1000.0 / reps


def extra_measurements(args, inp, copies, h, y, down_ws):
    """Interleaved layout, fused vs unfused, and the B = 1..64 sweep (row vs col).

    Every figure is the mean of back-to-back calls over rotated weight copies
    (two of the 470 MB gate/up pair, eight of the 117 MB W_down), after an L2
    flush."""
    import torch
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    peak, _ = measured_peaks()
    reps = 100
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")  # 256 MB > L2
    out = {}
    # interleaved layout of the same weights (two copies, rotated)
    il = [I.to_layout(wg, wu, I.LAYOUT_INTERLEAVED)[0] for wg, wu, _ in copies]
    dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, il[0], None, "interleaved", h=h)
    t_il = timed_us(lambda i: dfk.dfk_rmsnorm_swiglu_gate_up(
        inp.x, inp.gamma, inp.eps, il[i % 2], None, "interleaved", h=h), reps, flush)
    del il
    # fused vs unfused (separate RMSNorm, 2 GEMVs, SiLU, multiply; bf16 in HBM)
    xn = torch.empty_like(inp.x)
    a = torch.empty_like(h)
    u = torch.empty_like(h)
    s = torch.empty_like(h)

    def unfused(i):
        wg, wu, _ = copies[i % 2]
        dfk.dfk_rmsnorm(inp.x, inp.gamma, inp.eps, out=xn)
        dfk.dfk_gemv(xn, wg, out=a)
        dfk.dfk_gemv(xn, wu, out=u)
        dfk.dfk_silu(a, out=s)
        dfk.dfk_mul(s, u, out=h)

    def fused(i):
        wg, wu, _ = copies[i % 2]
        dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, "row", h=h)

    unfused(0)
    t_unf = timed_us(unfused, reps, flush)
    t_fus = timed_us(fused, reps, flush)
    t_down = timed_us(lambda i: dfk.dfk_down_proj(h, down_ws[i % len(down_ws)], y=y), reps, flush)
    out["interleaved_gate_up_us"] = round(t_il, 2)
    out["fused_vs_unfused"] = {"fused_us": round(t_fus, 2), "unfused_us": round(t_unf, 2),
                               "speedup": round(t_unf / t_fus, 3),
                               "unfused": "rmsnorm + gemv(Wg) + gemv(Wu) + silu + mul"}
    out["down_proj_us"] = round(t_down, 2)
    out["down_proj_GBps"] = round(down_bytes(B1, D, F) / (t_down * 1e-6) / 1e9, 1)

    # batch sweep B = 1..64, row vs column-major, scheduler's choice
    sweep = []
    x64 = I.make_inputs(64, D, F, seed=2, with_down=False, device="cuda").x
    col = [I.to_layout(wg, wu, I.LAYOUT_COL) for wg, wu, _ in copies]
    row_w = [(wg, wu) for wg, wu, _ in copies]
    for B in (1, 2, 4, 8, 16, 32, 64):
        xb = x64[:B].contiguous()
        hb = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
        row = {"B": B}
        for name, ws in (("row", row_w), ("col", col)):
            dfk.dfk_rmsnorm_swiglu_gate_up(xb, inp.gamma, inp.eps, ws[0][0], ws[0][1], name,
                                           h=hb)  # first call: the scheduler times its variants
            t = timed_us(lambda i: dfk.dfk_rmsnorm_swiglu_gate_up(
                xb, inp.gamma, inp.eps, ws[i % 2][0], ws[i % 2][1], name, h=hb), reps, flush)
            gbs = gate_up_bytes(B, D, F) / (t * 1e-6) / 1e9
            v = dfk.dfk_cached_variant(dfk.DFK_OP_RMSNORM_GATE_UP, B, D, F, name) or {}
            row[name] = {"us": round(t, 2), "GBps": round(gbs, 1), "frac": round(gbs / peak, 4),
                         "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                         "tokens_per_s": round(B / (t * 1e-6), 1),
                         "variant": v.get("variant_id"),
                         "family": {0: "cuda_core", 1: "tensor_core"}.get(v.get("family"))}
        row["scheduler_pick"] = "row" if row["row"]["us"] <= row["col"]["us"] else "col"
        sweep.append(row)
    out["batch_sweep"] = sweep
    # down projection B = 1..64 (the scheduler's choice; eight W_down copies)
    dsweep = []
    for B in (1, 2, 4, 8, 16, 32, 64):
        hb = (0.5 * torch.randn(B, F, device="cuda")).to(torch.bfloat16)
        yb = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
        dfk.dfk_down_proj(hb, down_ws[0], y=yb)  # first call: the scheduler times its variants
        t = timed_us(lambda i: dfk.dfk_down_proj(hb, down_ws[i % len(down_ws)], y=yb), reps,
                     flush)
        gbs = down_bytes(B, D, F) / (t * 1e-6) / 1e9
        v = dfk.dfk_cached_variant(dfk.DFK_OP_DOWN, B, D, F) or {}
        dsweep.append({"B": B, "us": round(t, 2), "frac": round(gbs / peak, 4),
                       "family": {0: "cuda_core", 1: "tensor_core"}.get(v.get("family"))})
    out["down_sweep"] = dsweep
    del x64, col, row_w, flush
    torch.cuda.empty_cache()
    out["llama3_70b"] = llama70b_measure()
    torch.cuda.empty_cache()
    out["fp8_weights"] = fp8_measure()
    out["fp8_weights"]["bf16_b1_fused_us"] = round(t_fus, 2)
    torch.cuda.empty_cache()
    out["qkv_projection"] = qkv_measure()
    out["torch_eager_mlp"] = torch_eager_measure()
    out["decode_stack"] = decode_stack_measure(args.stack_steps)
    return out


def llama70b_measure(reps=30):
    """Llama-3-70B-shaped layer (d_model 8192, d_ff 28672, W ~ N(0, 0.015),
    no RMSNorm, seed 3): gate/up and down at B = 1 and 8, back-to-back calls
    over two rotated weight copies (1.9 GB each, far beyond L2)."""
    import torch
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    peak, _ = measured_peaks()
    D7, F7 = 8192, 28672
    res = []
    base = I.make_inputs(8, D7, F7, seed=3, w_std=0.015, norm=False, with_down=True,
                         device="cuda")
    cps = [(base.w_gate, base.w_up, base.w_down),
           (base.w_gate.clone(), base.w_up.clone(), base.w_down.clone())]
    for B in (1, 8):
        x = base.x[:B].contiguous()
        h = torch.empty(B, F7, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(B, D7, dtype=torch.bfloat16, device="cuda")
        dfk.dfk_swiglu_gate_up(x, cps[0][0], cps[0][1], "row", h=h)   # scheduler decides
        dfk.dfk_down_proj(h, cps[0][2], y=y)
        tg = timed_us(lambda i: dfk.dfk_swiglu_gate_up(x, cps[i % 2][0], cps[i % 2][1], "row",
                                                        h=h), reps)
        td = timed_us(lambda i: dfk.dfk_down_proj(h, cps[i % 2][2], y=y), reps)
        gg = gate_up_bytes(B, D7, F7) / (tg * 1e-6) / 1e9
        gd = down_bytes(B, D7, F7) / (td * 1e-6) / 1e9
        vg = dfk.dfk_cached_variant(dfk.DFK_OP_GATE_UP, B, D7, F7, "row") or {}
        vd = dfk.dfk_cached_variant(dfk.DFK_OP_DOWN, B, D7, F7, "row") or {}
        res.append({"B": B, "gate_up_us": round(tg, 2), "gate_up_frac": round(gg / peak, 4),
                    "gate_up_frac_nominal": round(gg / NOMINAL_HBM_GBS, 4),
                    "gate_up_family": {0: "cuda_core", 1: "tensor_core"}.get(vg.get("family")),
                    "down_us": round(td, 2), "down_frac": round(gd / peak, 4),
                    "down_frac_nominal": round(gd / NOMINAL_HBM_GBS, 4),
                    "down_family": {0: "cuda_core", 1: "tensor_core"}.get(vd.get("family")),
                    "mlp_us": round(tg + td, 2)})
    del base, cps
    return res


def fp8_gate_up_bytes(B, D, F):
    """FP8 E4M3 codes of both matrices, their fp32 row scales, x, gamma, h."""
    return 2 * F * D + 2 * F * 4 + B * D * 2 + D * 2 + B * F * 2


def fp8_down_bytes(B, D, F):
    return D * F + D * 4 + B * F * 2 + B * D * 2


def fp8_measure(reps=100, ncopies=4):
    """FP8 E4M3 weight streaming (row scales, fused dequantisation) on the
    Llama-3-8B-shaped layer: the bench's seeded bf16 weights encoded per row,
    fused RMSNorm + gate/up and the down projection at B = 1..16, back-to-back
    calls over `ncopies` weight copies (176 MB each; together beyond L2)."""
    import torch
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    peak, _ = measured_peaks()
    base = I.make_inputs(16, D, F, seed=2, norm=True, with_down=True, device="cuda")
    qg, sg = I.to_fp8_rows(base.w_gate)
    qu, su = I.to_fp8_rows(base.w_up)
    qd, sd = I.to_fp8_rows(base.w_down)
    del base.w_gate, base.w_up, base.w_down
    cps = [(qg, qu, qd)] + [(qg.clone(), qu.clone(), qd.clone()) for _ in range(ncopies - 1)]
    res = []
    for B in (1, 2, 4, 8, 16):
        x = base.x[:B].contiguous()
        h = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
        dfk.dfk_rmsnorm_swiglu_gate_up_fp8(x, base.gamma, base.eps, qg, sg, qu, su, h=h)
        dfk.dfk_down_proj_fp8(h, qd, sd, y=y)        # first calls: the scheduler decides
        tg = timed_us(lambda i: dfk.dfk_rmsnorm_swiglu_gate_up_fp8(
            x, base.gamma, base.eps, cps[i % ncopies][0], sg, cps[i % ncopies][1], su, h=h), reps)
        td = timed_us(lambda i: dfk.dfk_down_proj_fp8(h, cps[i % ncopies][2], sd, y=y), reps)
        gg = fp8_gate_up_bytes(B, D, F) / (tg * 1e-6) / 1e9
        gd = fp8_down_bytes(B, D, F) / (td * 1e-6) / 1e9
        vg = dfk.dfk_cached_variant(dfk.DFK_OP_RMSNORM_GATE_UP_FP8, B, D, F, "row") or {}
        vd = dfk.dfk_cached_variant(dfk.DFK_OP_DOWN_FP8, B, D, F, "row") or {}
        res.append({"B": B, "gate_up_us": round(tg, 2), "gate_up_GBps": round(gg, 1),
                    "gate_up_frac": round(gg / peak, 4), "gate_up_variant": vg.get("variant_id"),
                    "down_us": round(td, 2), "down_GBps": round(gd, 1),
                    "down_frac": round(gd / peak, 4), "down_variant": vd.get("variant_id"),
                    "mlp_us": round(tg + td, 2)})
    del cps, qg, qu, qd, base
    torch.cuda.empty_cache()
    return {"workload": "llama3_8b_fp8_e4m3_row_scales", "weights": "E4M3 codes + fp32 row "
            "scales from the seeded bf16 weights (absmax / 448 per row)", "sweep": res}


def qkv_bytes(B, D, N):
    """Packed QKV projection: the weights once, x, gamma, the outputs."""
    return N * D * 2 + B * D * 2 + D * 2 + B * N * 2


def qkv_measure(reps=100, ncopies=4):
    """RMSNorm + packed QKV projection on the Llama-3-8B attention input shape
    (d_model 4096, n_q 4096, n_k = n_v = 1024; seeded weights ~ N(0, 0.02)):
    fused (one kernel, one weight stream) against the pages' unfused form
    (an RMSNorm kernel, then three separate projections), B = 1..64,
    back-to-back calls over `ncopies` weight copies (50 MB each)."""
    import torch
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    peak, _ = measured_peaks()
    Dq, nq, nk, nv = 4096, 4096, 1024, 1024
    N = nq + nk + nv
    g = I.make_generator(7, "cuda")
    x64 = torch.randn(64, Dq, generator=g, device="cuda").to(torch.bfloat16)
    gamma = (1.0 + 0.1 * torch.randn(Dq, generator=g, device="cuda")).to(torch.bfloat16)
    ws = [(0.02 * torch.randn(N, Dq, generator=g, device="cuda")).to(torch.bfloat16)
          for _ in range(ncopies)]
    res = []
    for B in (1, 4, 16, 64):
        x = x64[:B].contiguous()
        q = torch.empty(B, nq, dtype=torch.bfloat16, device="cuda")
        k = torch.empty(B, nk, dtype=torch.bfloat16, device="cuda")
        v = torch.empty(B, nv, dtype=torch.bfloat16, device="cuda")
        xn = torch.empty_like(x)
        dfk.dfk_rmsnorm_qkv_proj(x, gamma, 1e-5, ws[0], nq, nk, nv, q=q, k=k, v=v)

        def unfused(i):
            w = ws[i % ncopies]
            dfk.dfk_rmsnorm(x, gamma, 1e-5, out=xn)
            dfk.dfk_gemv(xn, w[:nq], out=q)
            dfk.dfk_gemv(xn, w[nq:nq + nk], out=k)
            dfk.dfk_gemv(xn, w[nq + nk:], out=v)

        unfused(0)                                    # scheduler decisions first
        tf = timed_us(lambda i: dfk.dfk_rmsnorm_qkv_proj(x, gamma, 1e-5, ws[i % ncopies], nq, nk,
                                                         nv, q=q, k=k, v=v), reps)
        tu = timed_us(unfused, reps)
        gbs = qkv_bytes(B, Dq, N) / (tf * 1e-6) / 1e9
        vq = dfk.dfk_cached_variant(dfk.DFK_OP_RMSNORM_QKV, B, Dq, N) or {}
        res.append({"B": B, "fused_us": round(tf, 2), "fused_GBps": round(gbs, 1),
                    "fused_frac": round(gbs / peak, 4), "unfused_us": round(tu, 2),
                    "speedup": round(tu / tf, 3), "variant": vq.get("variant_id"),
                    "family": {0: "cuda_core", 1: "tensor_core"}.get(vq.get("family"))})
    del ws, x64
    torch.cuda.empty_cache()
    return {"workload": "llama3_8b_qkv (d_model 4096, n_q 4096, n_k 1024, n_v 1024)",
            "unfused": "rmsnorm + gemv(W_q) + gemv(W_k) + gemv(W_v)", "sweep": res}


def torch_eager_measure(reps=50):
    """Informational: the same Llama-3-8B-shaped MLP layer in torch eager ops
    (RMSNorm, two cuBLAS linears, SiLU, multiply, cuBLAS down projection),
    two rotated weight copies, back-to-back calls.  Library kernels, not this
    repository's; reported for context only."""
    import torch
    import torch.nn.functional as Fn
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    base = I.make_inputs(64, D, F, seed=2, norm=True, with_down=True, device="cuda")
    cps = [(base.w_gate, base.w_up, base.w_down),
           (base.w_gate.clone(), base.w_up.clone(), base.w_down.clone())]
    res = []
    for B in (1, 16, 64):
        x = base.x[:B].contiguous()

        def step(i):
            wg, wu, wd = cps[i % 2]
            xn = Fn.rms_norm(x, (D,), base.gamma, base.eps)
            return Fn.linear(Fn.silu(Fn.linear(xn, wg)) * Fn.linear(xn, wu), wd)

        t = timed_us(step, reps)
        h = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")

        def ours(i):
            wg, wu, wd = cps[i % 2]
            dfk.dfk_rmsnorm_swiglu_gate_up(x, base.gamma, base.eps, wg, wu, "row", h=h)
            dfk.dfk_down_proj(h, wd, y=y)

        ours(0)
        t2 = timed_us(ours, reps)
        res.append({"B": B, "torch_mlp_us": round(t, 2),
                    "torch_GBps": round(step_bytes(B, D, F) / (t * 1e-6) / 1e9, 1),
                    "dfk_mlp_us": round(t2, 2),
                    "dfk_GBps": round(step_bytes(B, D, F) / (t2 * 1e-6) / 1e9, 1),
                    "dfk_speedup": round(t / t2, 3)})
    del cps, base
    torch.cuda.empty_cache()
    return {"what": "torch eager: rms_norm + linear(Wg), linear(Wu) + silu * mul + linear(Wd) "
            "(cuBLAS), against this library's fused RMSNorm+gate/up + down on the same "
            "weights; informational", "sweep": res}


def decode_stack_measure(steps, layers=32, B=4):
    """Long-generation decode: a 32-layer stack of Llama-3-8B-shaped MLPs
    (11.3 GB of distinct weights, seed 4), B = 4, one step per CUDA-graph
    replay: fused vs unfused kernels, the fused stack with W_gate / W_up in
    the layout the scheduler picks for the shape (layout "auto"), and the
    fused stack with the weights encoded as FP8 E4M3 + row scales (5.6 GB
    per step)."""
    import torch
    from swiglu_mlp_dfk_b200 import inputs as I
    from swiglu_mlp_dfk_b200.stack import DecodeStack

    peak, _ = measured_peaks()
    x0, params = I.make_stack(layers, B, D, F, seed=4, w_std=0.02, device="cuda")
    res = {"layers": layers, "B": B, "steps": steps,
           "weights_GB": round(sum(t.numel() * 2 for p in params for t in p) / 1e9, 2)}
    for fused, fp8, layout in ((True, False, "row"), (False, False, "row"),
                               (True, False, "auto"), (True, True, "row")):
        st = DecodeStack(params, x0, fused=fused, fp8=fp8, layout=layout)
        st.step_eager()                      # scheduler decisions outside capture
        torch.cuda.synchronize()
        st.capture()
        for _ in range(3):
            st.step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            st.step()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        key = "fp8" if fp8 else ("fused_auto" if layout == "auto" else
                                 ("fused" if fused else "unfused"))
        res[key + "_ms_per_step"] = round(ms, 4)
        if layout == "auto" or fp8:
            # in-context tuning: the step timed with forced variants of each
            # call, then the same timed loop again with the winners
            st.release()
            tuned = st.tune_variants()
            st.step_eager()
            torch.cuda.synchronize()
            st.capture()
            for _ in range(3):
                st.step()
            a.record()
            for _ in range(steps):
                st.step()
            b.record()
            torch.cuda.synchronize()
            tms = a.elapsed_time(b) / steps
            res[key + "_tuned_ms_per_step"] = round(tms, 4)
            res[key + "_tuned_variants"] = {"gate_up": tuned["gate_up"], "down": tuned["down"]}
            res[key + "_tuned_frac_of_peak"] = round(
                st.bytes_per_step() / (tms * 1e-3) / 1e9 / peak, 4)
        if layout == "auto":
            gbs = st.bytes_per_step() / (ms * 1e-3) / 1e9
            res["fused_auto_layout"] = st.layout
            res["fused_auto_GBps"] = round(gbs, 1)
            res["fused_auto_frac_of_peak"] = round(gbs / peak, 4)
            st.release()
            del st
            continue
        if fp8:  # the E4M3-MMA calls launch two kernels each (prep + main)
            res["fp8_calls_per_step"] = st.kernels_per_step()
        else:
            res[key + "_kernels_per_step"] = st.kernels_per_step()
        if fp8:
            gbs = st.bytes_per_step() / (ms * 1e-3) / 1e9
            res["fp8_GBps"] = round(gbs, 1)
            res["fp8_frac_of_peak"] = round(gbs / peak, 4)
            res["fp8_weights_GB"] = round(st.bytes_per_step() / 1e9, 2)
        elif fused:
            gbs = st.bytes_per_step() / (ms * 1e-3) / 1e9
            res["fused_GBps"] = round(gbs, 1)
            res["fused_frac_of_peak"] = round(gbs / peak, 4)
            res["roofline_ms_per_step"] = round(st.bytes_per_step() / (peak * 1e9) * 1e3, 4)
        st.release()
        del st
    # one persistent kernel per step (dfk_mlp_stack_step): the same layers,
    # stacked into [L][...] tensors, with row- and column-major gate/up weights
    from swiglu_mlp_dfk_b200.stack import PersistentDecodeStack
    stacked = tuple(torch.stack([p[i] for p in params]) for i in range(4))
    for lay in ("row", "col"):
        ps = PersistentDecodeStack(x0=x0, stacked=stacked, layout=lay)
        ps.step_eager()
        torch.cuda.synchronize()
        ps.capture()
        for _ in range(3):
            ps.step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            ps.step()
        b.record()
        torch.cuda.synchronize()
        pms = a.elapsed_time(b) / steps
        key = "persistent" if lay == "row" else "persistent_col"
        res[key + "_ms_per_step"] = round(pms, 4)
        res[key + "_frac_of_peak"] = round(ps.bytes_per_step() / (pms * 1e-3) / 1e9 / peak, 4)
        res[key + "_speedup_over_fused"] = round(res["fused_ms_per_step"] / pms, 3)
        res["persistent_kernels_per_step"] = ps.kernels_per_step()
        ps.release()
        del ps
        torch.cuda.empty_cache()
    del stacked
    res["fused_speedup"] = round(res["unfused_ms_per_step"] / res["fused_ms_per_step"], 3)
    res["fused_auto_speedup_over_row"] = round(res["fused_ms_per_step"] /
                                               res["fused_auto_ms_per_step"], 3)
    res["fp8_speedup_over_bf16_fused"] = round(res["fused_ms_per_step"] / res["fp8_ms_per_step"], 3)
    del params, x0
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- CPU oracle

def _oracle_layer_inputs():
    from swiglu_mlp_dfk_b200 import inputs as I
    inp = I.make_inputs(B1, D, F, seed=SEED, w_std=0.02, norm=True, with_down=True,
                        device="cpu")
    return [I.to_bits(t) for t in (inp.x, inp.gamma, inp.w_gate, inp.w_up, inp.w_down)]


def cpu_baseline(min_s=10.0, max_reps=400):
    """The fp64 CPU oracle, as it stands, on the full B = 1 layer, repeated ~10 s."""
    import oracle
    x, g, wg, wu, wd = _oracle_layer_inputs()
    reps = 0
    t0 = time.perf_counter()
    while True:
        hh = oracle.gate_up(x, wg, wu, gamma=g, eps=1e-5)
        oracle.down(hh, wd)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s or reps >= max_reps:
            break
    return {"value": round(step_bytes(B1, D, F) * reps / el / 1e9, 3), "unit": UNIT,
            "cores": oracle.threads(), "kind": "oracle",
            "sample": "full Llama-3-8B-shaped layer at B=1 (14336 gate/up columns + 4096 "
                      "down rows), repeated %d times in %.1f s" % (reps, el)}


def reference_arm(args):
    """--impl reference: the fp64 CPU oracle timed on this arm's workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import numpy as np
    import oracle
    x, g, wg, wu, wd = _oracle_layer_inputs()
    # one step = a bounded sample of the layer: 1/8 of the gate/up columns and
    # 1/8 of the down rows (the metric counts the sample's algorithmic bytes)
    rows = np.arange(0, F, 8, dtype=np.int32)
    drows = np.arange(0, D, 8, dtype=np.int32)
    sample_bytes = (2 * rows.size * D * 2 + B1 * D * 2 + D * 2 + B1 * rows.size * 2
                    + drows.size * F * 2 + B1 * F * 2 + B1 * drows.size * 2)
    hfull = oracle.gate_up(x, wg, wu, gamma=g, eps=1e-5)

    def one():
        oracle.gate_up(x, wg, wu, gamma=g, eps=1e-5, rows=rows)
        oracle.down(hfull, wd, rows=drows)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = sample_bytes * args.steps / el / 1e9
    sample = ("1/8 of the Llama-3-8B-shaped layer per step (1792 gate/up columns + 512 "
              "down rows, B=1)")
    # n_gpus: the N this arm was launched with (the oracle itself runs on rank
    # 0's host cores only)
    return {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3 / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_dict("cpu"),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def profile_arm(args):
    """--profile KERNEL: run one kernel of the workload inside an NVTX range
    named dfk_profile (for ncu --nvtx-include dfk_profile/), nothing else."""
    import torch
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import inputs as I

    torch.cuda.set_device(0)
    B = args.batch
    if args.profile == "pstack":
        # the one-launch decode step on a 2-layer Llama-3-8B-shaped stack
        # (0.7 GB of weights: small enough for a full ncu capture)
        from swiglu_mlp_dfk_b200.stack import PersistentDecodeStack
        x0, params = I.make_stack(2, B, D, F, seed=4, w_std=0.02, device="cuda")
        ps = PersistentDecodeStack(params, x0)
        fn = ps.step_eager
    else:
        inp = I.make_inputs(B, D, F, seed=SEED, w_std=0.02, norm=True,
                            with_down=args.profile.startswith("down"), device="cuda")
        return _profile_one(args, dfk, I, inp, B)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("dfk_profile")
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    print(json.dumps({"profile": args.profile, "B": B, "layers": 2, "calls": args.steps,
                      "device_error_word": dfk.dfk_device_error()}))
    return None


def _profile_one(args, dfk, I, inp, B):
    import torch
    h = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
    lay = {"row": I.LAYOUT_ROW, "col": I.LAYOUT_COL, "interleaved": I.LAYOUT_INTERLEAVED}
    wg, wu = I.to_layout(inp.w_gate, inp.w_up, lay[args.layout])
    if args.profile == "gate_up":
        fn = lambda: dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu,
                                                    args.layout, h=h, variant=args.variant)
    elif args.profile == "gate_up_fp8":
        qg, sg = I.to_fp8_rows(inp.w_gate)
        qu, su = I.to_fp8_rows(inp.w_up)
        fn = lambda: dfk.dfk_rmsnorm_swiglu_gate_up_fp8(inp.x, inp.gamma, inp.eps, qg, sg, qu,
                                                        su, h=h, variant=args.variant)
    elif args.profile == "qkv":
        nq, nk, nv = 4096, 1024, 1024
        w_qkv = torch.cat([inp.w_gate[:nq], inp.w_up[:nk + nv]]).contiguous()  # seeded weights
        fn = lambda: dfk.dfk_rmsnorm_qkv_proj(inp.x, inp.gamma, inp.eps, w_qkv, nq, nk, nv,
                                              variant=args.variant)
    elif args.profile == "down_fp8":
        qd, sd = I.to_fp8_rows(inp.w_down)
        fn = lambda: dfk.dfk_down_proj_fp8(h, qd, sd, y=y, variant=args.variant)
    else:
        fn = lambda: dfk.dfk_down_proj(h, inp.w_down, y=y, variant=args.variant)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("dfk_profile")
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    print(json.dumps({"profile": args.profile, "B": B, "layout": args.layout,
                      "calls": args.steps, "device_error_word": dfk.dfk_device_error()}))
    return None


def tp_arm(args):
    """Tensor-parallel layer: the same 8B-shaped layer with d_ff sharded over
    the torchrun ranks (one GPU each), the all-reduce fused into the down
    projection.  Strong scaling: the layer is fixed, every rank streams its
    1/N of the weights; value = the layer's algorithmic bytes per step /
    max-over-ranks step time."""
    import datetime
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import swiglu_mlp_dfk_b200 as dfk
    from swiglu_mlp_dfk_b200 import build as kbuild
    from swiglu_mlp_dfk_b200 import inputs as I
    from swiglu_mlp_dfk_b200 import tp

    if rank == 0 or not os.path.exists(kbuild.LIB):
        kbuild.build()
    if world > 1:
        dist.barrier()
    dfk.dfk_device_error()
    inp = I.make_inputs(B1, D, F, seed=SEED, w_std=0.02, norm=True, with_down=True,
                        device="cuda")
    # two shard copies in rotation (inputs larger than L2)
    shards = [tp.shard_weights(inp.w_gate, inp.w_up, inp.w_down, I.LAYOUT_ROW, world, rank)]
    shards.append(tuple(t.clone() if torch.is_tensor(t) else t for t in shards[0]))
    group = tp.TPGroup(world, rank, 64, D)
    h = torch.empty(B1, shards[0][2].shape[1], dtype=torch.bfloat16, device="cuda")
    y = torch.empty(B1, D, dtype=torch.bfloat16, device="cuda")

    def step(i):
        wg, wu, wd, _ = shards[i % 2]
        dfk.dfk_rmsnorm_swiglu_gate_up(inp.x, inp.gamma, inp.eps, wg, wu, "row", h=h)
        group.down_proj_allreduce(h, wd, y=y)

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks.phase = "timed"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    clocks.phase = "extra"
    clocks.stop()
    t_max = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, "cuda")
    err = dfk.dfk_device_error()
    group.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    value = step_bytes(B1, D, F) * args.steps / (t_max / 1e3) / 1e9
    return {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_max / args.steps, 5), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(config_dict("tp%d" % world),
                           step="per rank: fused RMSNorm+gate/up on its d_ff shard, then the "
                                "down projection with the all-reduce fused in"),
            "gpu_launches": 2 * args.steps, "clocks": clocks.summary("timed"),
            "device_error_word": err}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["dfk", "reference"], default="dfk")
    ap.add_argument("--quick", action="store_true",
                    help="skip the sweep / unfused / interleaved / decode-stack measurements")
    ap.add_argument("--stack-steps", type=int, default=512,
                    help="decode steps of the 32-layer stack measurement")
    ap.add_argument("--profile",
                    choices=["gate_up", "down", "gate_up_fp8", "down_fp8", "qkv", "pstack"],
                    default=None,
                    help="run only this kernel (inside an NVTX range) for ncu")
    ap.add_argument("--batch", type=int, default=1, help="batch for --profile")
    ap.add_argument("--layout", default="row", help="weight layout for --profile")
    ap.add_argument("--variant", type=int, default=0,
                    help="variant id for --profile (0 = the scheduler's choice)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel layer over the torchrun ranks (d_ff sharded, the "
                         "all-reduce fused into the down projection) instead of replicas")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile:
        return profile_arm(args)
    if args.tp and args.impl != "reference":
        line = tp_arm(args)
    else:
        line = reference_arm(args) if args.impl == "reference" else gpu_arm(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
