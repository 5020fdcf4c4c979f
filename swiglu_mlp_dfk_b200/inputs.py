"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module draws random numbers and rearranges memory; it holds none of the
MLP's arithmetic.  Every tensor is drawn as float32 normal noise from a
``torch.Generator`` seeded per workload, scaled, and cast to bf16 (round to
nearest even).  Draw order is fixed: x, gamma, W_gate, W_up, W_down.  The
same (seed, device) always yields the same bytes; the CPU and CUDA generators
yield different streams, so a check must hand the oracle the very bytes the
kernel read (``to_bits``).

The workloads are Llama-3-shaped decode MLP layers (shapes only -- no trained
weights exist here): d_model 4096 / d_ff 14336 (8B) and 8192 / 28672 (70B),
plus a tiny 256 / 688 layer.  Weights ~ N(0, 0.02) (0.015 for 70B),
x ~ N(0, 1), gamma = 1 + N(0, 0.1), eps = 1e-5.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch

LAYOUT_ROW = 0
LAYOUT_COL = 1
LAYOUT_INTERLEAVED = 2
LAYOUT_NAMES = {LAYOUT_ROW: "row", LAYOUT_COL: "col", LAYOUT_INTERLEAVED: "interleaved"}


@dataclass(frozen=True)
class Workload:
    name: str
    d_model: int
    d_ff: int
    batches: Tuple[int, ...]
    w_std: float
    seed: int
    norm: bool = True
    eps: float = 1e-5
    x_std: float = 1.0
    gamma_std: float = 0.1
    layers: int = 1
    note: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", 256, 688, (1,), 0.02, 0, norm=True,
                     note="tiny SwiGLU MLP, row-major, oracle finishes in well under a second"),
    "llama3_8b": Workload("llama3_8b", 4096, 14336, (1,), 0.02, 1, norm=True,
                          note="Llama-3-8B-shaped layer, fused RMSNorm, row-major and interleaved"),
    "llama3_8b_sweep": Workload("llama3_8b_sweep", 4096, 14336, (1, 2, 4, 8, 16, 32, 64), 0.02, 2,
                                norm=True, note="decode batch sweep, row- vs column-major"),
    "llama3_70b": Workload("llama3_70b", 8192, 28672, (1, 8), 0.015, 3, norm=False,
                           note="Llama-3-70B-shaped layer, full MLP incl. down projection"),
    "stack32": Workload("stack32", 4096, 14336, (4,), 0.02, 4, norm=True, layers=32,
                        note="32-layer decode stack, 512 steps, CUDA graph"),
}


@dataclass
class MLPInputs:
    x: torch.Tensor                       # [B, D] bf16
    gamma: Optional[torch.Tensor]         # [D] bf16
    w_gate: torch.Tensor                  # [F, D] bf16 (row-major)
    w_up: torch.Tensor                    # [F, D] bf16
    w_down: Optional[torch.Tensor]        # [D, F] bf16
    eps: float = 1e-5
    extra: dict = field(default_factory=dict)


def _normal_bf16(gen, shape, std, mean, device, chunk=1 << 26):
    """float32 N(mean, std) cast to bf16, drawn in chunks to bound the fp32 scratch."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        t = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        if mean != 0.0:
            t.add_(mean)
        flat[s:e].copy_(t)
    return out


def make_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_inputs(B: int, D: int, F: int, *, seed: int, w_std: float = 0.02, norm: bool = True,
                with_down: bool = True, device="cpu", x_std: float = 1.0,
                gamma_std: float = 0.1, eps: float = 1e-5, gen=None) -> MLPInputs:
    """One MLP layer's tensors in the fixed draw order x, gamma, Wg, Wu, Wd."""
    gen = gen if gen is not None else make_generator(seed, device)
    x = _normal_bf16(gen, (B, D), x_std, 0.0, device)
    gamma = _normal_bf16(gen, (D,), gamma_std, 1.0, device) if norm else None
    wg = _normal_bf16(gen, (F, D), w_std, 0.0, device)
    wu = _normal_bf16(gen, (F, D), w_std, 0.0, device)
    wd = _normal_bf16(gen, (D, F), w_std, 0.0, device) if with_down else None
    return MLPInputs(x, gamma, wg, wu, wd, eps)


def make_workload(name: str, B: Optional[int] = None, device="cpu", with_down=True) -> MLPInputs:
    w = WORKLOADS[name]
    b = w.batches[0] if B is None else B
    return make_inputs(b, w.d_model, w.d_ff, seed=w.seed, w_std=w.w_std, norm=w.norm,
                       with_down=with_down, device=device, x_std=w.x_std,
                       gamma_std=w.gamma_std, eps=w.eps)


def make_stack(layers: int, B: int, D: int, F: int, *, seed: int, w_std: float = 0.02,
               device="cuda"):
    """Decode-stack tensors: x0, then (gamma_l, Wg_l, Wu_l, Wd_l) for l = 0..layers-1."""
    gen = make_generator(seed, device)
    x0 = _normal_bf16(gen, (B, D), 1.0, 0.0, device)
    layer_params = []
    for _ in range(layers):
        gamma = _normal_bf16(gen, (D,), 0.1, 1.0, device)
        wg = _normal_bf16(gen, (F, D), w_std, 0.0, device)
        wu = _normal_bf16(gen, (F, D), w_std, 0.0, device)
        wd = _normal_bf16(gen, (D, F), w_std, 0.0, device)
        layer_params.append((gamma, wg, wu, wd))
    return x0, layer_params


def to_layout(w_gate: torch.Tensor, w_up: torch.Tensor, layout: int):
    """Rearrange row-major [F, D] weights into the requested storage layout.

    row: ([F, D], [F, D]); col: ([D, F], [D, F]) = transposes;
    interleaved: ([F, 2, D], None) with [j, 0] = gate row j, [j, 1] = up row j.
    """
    if layout == LAYOUT_ROW:
        return w_gate.contiguous(), w_up.contiguous()
    if layout == LAYOUT_COL:
        return w_gate.t().contiguous(), w_up.t().contiguous()
    if layout == LAYOUT_INTERLEAVED:
        return torch.stack([w_gate, w_up], dim=1).contiguous(), None
    raise ValueError("unknown layout %r" % (layout,))


def to_bits(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """bf16 tensor -> numpy uint16 bit patterns on the host (exact)."""
    if t is None:
        return None
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bf16")
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(bits: np.ndarray, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor (exact)."""
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a bf16 tensor (bit-level conversion, no arithmetic)."""
    bits = to_bits(t)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_fp8_rows(w: torch.Tensor):
    """FP8 E4M3 weights with one fp32 scale per row, from bf16 weights [N, K]:
    s = max|w| / 448 per row (1 for an all-zero row), Q = E4M3(w / s) by torch's
    round-to-nearest cast.  Returns (Q as uint8 [N, K], s float32 [N])."""
    wf = w.float()
    amax = wf.abs().amax(dim=1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (wf / s[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return q, s.contiguous()


def fp8_values(q: torch.Tensor) -> np.ndarray:
    """Exact float64 values of E4M3 codes (bit-level conversion through torch)."""
    return q.detach().contiguous().view(torch.float8_e4m3fn).float().cpu().numpy().astype(
        np.float64)
