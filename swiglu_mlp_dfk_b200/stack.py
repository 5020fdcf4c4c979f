"""Multi-layer decode loop over the library's kernels, captured in a CUDA graph.

Each decode step runs, for every layer l, the fused RMSNorm + gate/up +
SiLU * up kernel and then the separate down projection, feeding layer l's
output y to layer l + 1 (no residual: each layer's RMSNorm prologue keeps the
activations in range); after the last layer the step's output is rescaled
per row, x_{t+1} = y_t / sqrt(mean(y_t^2) + eps), and fed back.  This is the
long-generation setting of "Deep Kernel Fusion for Transformers" (abstract:
consistent speed-ups over generation lengths), as a stack of SwiGLU MLP
layers only.

The fused bf16 stack can hold W_gate / W_up in any of the library's gate/up
layouts: row-major [d_ff][d_model] as given, column-major [d_model][d_ff],
or gate/up rows interleaved [d_ff][2][d_model].  With layout="auto" the
library's scheduler times the fused RMSNorm + gate/up op for the stack's
shape over every layout (dfk_select_variant with DFK_W_ANY) and the weights
are stored once in the winner's layout: the profiler-driven choice between
row- and column-major kernels of "Deep Kernel Fusion for Transformer
Decoding" (episode description), made per model at load time.

The unfused variant runs the same step with separate kernels (RMSNorm, two
GEMVs, SiLU, multiply, down projection) and bf16 intermediates in HBM.  The
FP8 variant encodes every layer's weights once as E4M3 codes with one fp32
scale per output row (the library's FP8 entry points: half the weight bytes
per step, dequantised inside the kernels).

In-context tuning (``tune_variants``): the library's scheduler times each
operation on its own, in bursts of back-to-back launches of that one
operation.  Inside the stack every gate/up call follows a down projection and
every down projection follows a gate/up call, and a variant that wins in a
burst can lose there.  With FP8 weights the in-kernel-term E4M3 variants
win the bursts at B = 4 but lose inside the stack: every CTA converts the
whole activation into E4M3 terms before its first MMA, and in the stack, where
the two kernels alternate on every SM, that code runs from a cold
instruction cache at half the speed it has in a burst, so the variants with
a prep kernel (which converts once per token) win there.  The tuner
times the captured step itself with each candidate variant of one
operation while the other keeps its current choice, first for the gate/up
call, then for the down projection, and keeps the fastest.

Everything launched here is a libdfk kernel; torch provides the buffers, the
stream and the CUDA graph.
"""
import torch

import swiglu_mlp_dfk_b200 as dfk


class DecodeStack:
    """A stack of SwiGLU MLP layers driven one decode step at a time.

    layers: list of (gamma [D], W_gate [F, D], W_up [F, D], W_down [D, F]) bf16
    x0:     [B, D] bf16 first-step input
    layout: "row", "col", "interleaved" or "auto" -- how the fused bf16
            stack stores W_gate / W_up (converted copies; "auto" asks the
            scheduler); the unfused and FP8 stacks are row-major only
    """

    def __init__(self, layers, x0, eps=1e-5, fused=True, fp8=False, layout="row"):
        if fp8 and not fused:
            raise ValueError("the FP8 stack runs the fused kernels")
        if layout not in ("row", "col", "interleaved", "auto"):
            raise ValueError("layout must be row, col, interleaved or auto")
        if layout != "row" and (fp8 or not fused):
            raise ValueError("only the fused bf16 stack takes another weight layout")
        self.eps = float(eps)
        self.fused = fused
        self.fp8 = fp8
        if fp8:
            from . import inputs as I
            enc = []
            for gamma, wg, wu, wd in layers:
                enc.append((gamma,) + I.to_fp8_rows(wg) + I.to_fp8_rows(wu) + I.to_fp8_rows(wd))
            layers = enc
        self.B, self.D = x0.shape
        self.F = layers[0][1].shape[0]     # W_gate rows (bf16 or FP8 codes)
        dev = x0.device
        # the stream exists before the layout choice so the scheduler's
        # timing and every later launch share it
        self.stream = torch.cuda.Stream(device=dev)
        if layout == "auto":
            with torch.cuda.stream(self.stream):
                rec = dfk.dfk_select_variant(dfk.DFK_OP_RMSNORM_GATE_UP, self.B, self.D, self.F,
                                             layout=dfk.DFK_W_ANY, stream=self.stream)
            self.stream.synchronize()
            layout = {dfk.DFK_W_ROW_MAJOR: "row", dfk.DFK_W_COL_MAJOR: "col",
                      dfk.DFK_W_GU_INTERLEAVED: "interleaved"}[rec["layout"]]
        self.layout = layout
        if layout == "col":
            layers = [(g, wg.t().contiguous(), wu.t().contiguous(), wd)
                      for g, wg, wu, wd in layers]
        elif layout == "interleaved":
            layers = [(g, torch.stack([wg, wu], 1).contiguous(), None, wd)
                      for g, wg, wu, wd in layers]
        self.layers = layers
        self.x = x0.clone()                       # step input (graph-static buffer)
        self.acts = [torch.empty(self.B, self.D, dtype=torch.bfloat16, device=dev)
                     for _ in range(2)]          # ping-pong layer outputs
        self.h = torch.empty(self.B, self.F, dtype=torch.bfloat16, device=dev)
        if not fused:
            self.xn = torch.empty(self.B, self.D, dtype=torch.bfloat16, device=dev)
            self.a = torch.empty_like(self.h)
            self.u = torch.empty_like(self.h)
            self.s = torch.empty_like(self.h)
        self.graph = None
        # forced variants of the two per-layer calls (0 = the library's choice)
        self.gu_variant = 0
        self.dn_variant = 0
        # every launch of the stack (eager warm-up, capture, replay) goes to
        # self.stream, so the capture finds the scheduler's decisions and the
        # split-K workspace that the warm-up made on that stream

    def layer_input(self, l):
        return self.x if l == 0 else self.acts[(l - 1) % 2]

    def _layer(self, l):
        xin = self.layer_input(l)
        y = self.acts[l % 2]
        if self.fp8:
            gamma, qg, sg, qu, su, qd, sd = self.layers[l]
            dfk.dfk_rmsnorm_swiglu_gate_up_fp8(xin, gamma, self.eps, qg, sg, qu, su, h=self.h,
                                               variant=self.gu_variant)
            dfk.dfk_down_proj_fp8(self.h, qd, sd, y=y, variant=self.dn_variant)
            return
        gamma, wg, wu, wd = self.layers[l]
        if self.fused:
            dfk.dfk_rmsnorm_swiglu_gate_up(xin, gamma, self.eps, wg, wu, self.layout, h=self.h,
                                           variant=self.gu_variant)
        else:
            dfk.dfk_rmsnorm(xin, gamma, self.eps, out=self.xn)
            dfk.dfk_gemv(self.xn, wg, out=self.a)
            dfk.dfk_gemv(self.xn, wu, out=self.u)
            dfk.dfk_silu(self.a, out=self.s)
            dfk.dfk_mul(self.s, self.u, out=self.h)
        dfk.dfk_down_proj(self.h, wd, y=y, variant=self.dn_variant)

    def _launch_step(self):
        for l in range(len(self.layers)):
            self._layer(l)
        dfk.dfk_rms_rescale(self.acts[(len(self.layers) - 1) % 2], self.eps, out=self.x)

    def step_eager(self):
        """One decode step, launched kernel by kernel on the stack's stream
        (ordered after the caller's current stream and back)."""
        cur = torch.cuda.current_stream(self.stream.device)
        self.stream.wait_stream(cur)
        with torch.cuda.stream(self.stream):
            self._launch_step()
        cur.wait_stream(self.stream)

    def capture(self):
        """Capture one step in a CUDA graph on the stack's stream (call after a
        warm-up step, so the scheduler's decisions are cached and nothing is
        timed during capture)."""
        torch.cuda.synchronize(self.stream.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self._launch_step()
        self.graph = g
        return g

    def step(self):
        if self.graph is not None:
            cur = torch.cuda.current_stream(self.stream.device)
            self.stream.wait_stream(cur)
            with torch.cuda.stream(self.stream):
                self.graph.replay()
            cur.wait_stream(self.stream)
        else:
            self.step_eager()

    def release(self):
        self.graph = None

    def _candidates(self, gate_up):
        """Variant ids worth timing in context for one of the two calls: the
        library's own choice (0) and every tensor-core variant of the call's
        class (the CUDA-core variants are many; the library's choice stands
        for that family)."""
        out = [0]
        for i in range(1, dfk.dfk_variant_count() + 1):
            v = dfk.dfk_variant_info(i)
            if v["family"] != 1:
                continue
            is_gu = v["op"] in (dfk.DFK_OP_GATE_UP, dfk.DFK_OP_GATE_UP_FP8)
            if is_gu != gate_up:
                continue
            if v["e4m3_mma"] and not self.fp8:
                continue
            out.append(i)
        return out

    def _time_step(self, steps):
        """Mean device time of one captured step (ms), or None when a forced
        variant does not fit the shape."""
        self.release()
        try:
            self.step_eager()
        except dfk.DfkError:
            torch.cuda.synchronize(self.stream.device)
            return None
        torch.cuda.synchronize(self.stream.device)
        self.capture()
        for _ in range(2):
            self.step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream(self.stream.device)
        a.record(cur)
        for _ in range(steps):
            self.step()
        b.record(cur)
        b.synchronize()
        self.release()
        return a.elapsed_time(b) / steps

    def tune_variants(self, steps=10):
        """Pick the gate/up and down-projection variants by timing the whole
        captured step: each candidate of the gate/up call with the down
        projection at its current choice, then each candidate of the down
        projection.  Changes the stack's state (x advances by the timed steps);
        returns {"gate_up": id, "down": id, "ms_per_step": best, "library_ms":
        time with the library's own choices}.  Forced ids count as 0 = the
        library's choice."""
        if not self.fused:
            raise ValueError("in-context tuning covers the fused stacks")
        self.gu_variant = self.dn_variant = 0
        base = self._time_step(steps)
        best = base
        for attr, gate_up in (("gu_variant", True), ("dn_variant", False)):
            keep = getattr(self, attr)
            for vid in self._candidates(gate_up):
                if vid == keep:
                    continue
                setattr(self, attr, vid)
                t = self._time_step(steps)
                if t is not None and t < best:
                    best, keep = t, vid
            setattr(self, attr, keep)
        return {"gate_up": self.gu_variant, "down": self.dn_variant, "ms_per_step": best,
                "library_ms": base}

    def kernels_per_step(self):
        """Library calls per step (one kernel each, except the FP8 tensor-core
        calls that launch a prep kernel first)."""
        return len(self.layers) * (2 if self.fused else 6) + 1

    def bytes_per_step(self):
        """Algorithmic bytes of one step: every weight once, activations in/out."""
        B, D, F = self.B, self.D, self.F
        if self.fp8:  # codes (1 byte) + fp32 row scales
            per_layer = (2 * F * D + 2 * F * 4 + B * D * 2 + D * 2 + B * F * 2
                         + D * F + D * 4 + B * F * 2 + B * D * 2)
            return len(self.layers) * per_layer + 2 * B * D * 2
        per_layer = (2 * F * D * 2 + B * D * 2 + D * 2 + B * F * 2      # fused gate/up
                     + D * F * 2 + B * F * 2 + B * D * 2)               # down projection
        return len(self.layers) * per_layer + 2 * B * D * 2             # + rescale


class PersistentDecodeStack:
    """The fused bf16 decode step of ``DecodeStack`` (row-major weights) as
    ONE kernel launch per step (``dfk_mlp_stack_step``): a persistent kernel
    whose per-SM producers stream the weights of every layer's gate/up and
    down projection back to back, with grid-wide counters between the
    phases instead of kernel boundaries.

    layers: list of (gamma [D], W_gate [F, D], W_up [F, D], W_down [D, F]) bf16,
            or ``stacked=(gammas [L, D], W_gate [L, F, D], W_up [L, F, D],
            W_down [L, D, F])`` to use existing stacked tensors without a copy
    x0:     [B, D] bf16 first-step input
    layout: "row" or "col" -- how the step reads W_gate / W_up ("col" stores
            a transposed copy [L, D, F] once)

    After a step, ``h_all[l]`` and ``y_all[l]`` hold every layer's h and y and
    ``x`` the next step's input.
    """

    def __init__(self, layers=None, x0=None, eps=1e-5, stacked=None, layout="row"):
        if layout not in ("row", "col"):
            raise ValueError("layout must be row or col")
        if stacked is None:
            stacked = tuple(torch.stack([lay[i] for lay in layers]).contiguous()
                            for i in range(4))
        self.gammas, self.wg, self.wu, self.wd = stacked
        self.L, self.D, self.F = self.wd.shape
        self.layout = layout
        if layout == "col" and self.wg.shape[1] != self.D:
            # stored once as [L][D][F] (the column-major gate/up phases)
            self.wg = self.wg.transpose(1, 2).contiguous()
            self.wu = self.wu.transpose(1, 2).contiguous()
        self.B = x0.shape[0]
        self.eps = float(eps)
        dev = x0.device
        self.stream = torch.cuda.Stream(device=dev)
        self.x = x0.clone()
        self.h_all = torch.empty(self.L, self.B, self.F, dtype=torch.bfloat16, device=dev)
        self.y_all = torch.empty(self.L, self.B, self.D, dtype=torch.bfloat16, device=dev)
        n = dfk.dfk_mlp_stack_workspace_bytes(self.L, self.B, self.D, self.F)
        self.workspace = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.graph = None

    def _launch_step(self):
        dfk.dfk_mlp_stack_step(self.gammas, self.eps, self.wg, self.wu, self.wd, self.x,
                               self.h_all, self.y_all, self.workspace, layout=self.layout)

    def step_eager(self):
        cur = torch.cuda.current_stream(self.stream.device)
        self.stream.wait_stream(cur)
        with torch.cuda.stream(self.stream):
            self._launch_step()
        cur.wait_stream(self.stream)

    def capture(self):
        torch.cuda.synchronize(self.stream.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self._launch_step()
        self.graph = g
        return g

    def step(self):
        if self.graph is not None:
            cur = torch.cuda.current_stream(self.stream.device)
            self.stream.wait_stream(cur)
            with torch.cuda.stream(self.stream):
                self.graph.replay()
            cur.wait_stream(self.stream)
        else:
            self.step_eager()

    def release(self):
        self.graph = None

    def kernels_per_step(self):
        return 1

    def bytes_per_step(self):
        B, D, F = self.B, self.D, self.F
        per_layer = (2 * F * D * 2 + B * D * 2 + D * 2 + B * F * 2
                     + D * F * 2 + B * F * 2 + B * D * 2)
        return self.L * per_layer + 2 * B * D * 2
