"""fp64 CPU oracle for the decode-stage SwiGLU MLP -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package.  It wraps ``dfk_oracle.c`` (plain
C, IEEE double) through ctypes and shares nothing with the CUDA library.

What it computes follows "Deep Kernel Fusion for Transformer Decoding"
(episode description: gate projection, up projection, SiLU and the
elementwise multiply fused in one decode kernel; down projection separate)
and the RMSNorm fused in front of the gate/up projection in GPULlama3.java
PR #78 (description of the ``rms_ffn_gate_up`` task):

    xn = x * rsqrt(mean(x^2) + eps) * gamma        (optional)
    h  = SiLU(xn @ Wg^T) * (xn @ Wu^T),  SiLU(a) = a / (1 + exp(-a))
    y  = h @ Wd^T

and, for the packed QKV projection ("Optimizing QKV Projection with Operator
Fusion", section "Implementing Fusion: Packed Projections": one wider linear
layer replaces the three, its output split into Q, K and V; the RMSNorm in
front as in the PR's ``fusedRmsNormQKVMatmul``):

    o = xn @ Wqkv^T,  Wqkv = [Wq; Wk; Wv],  q, k, v = o[:, :nq], o[:, nq:nq+nk], o[:, nq+nk:]

Inputs are bf16 bit patterns (numpy uint16); outputs are float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

LAYOUT_ROW = 0
LAYOUT_COL = 1
LAYOUT_INTERLEAVED = 2

_lib = None


def _bind(lib):
    """Declare the C signatures on a loaded oracle library; returns it."""
    if True:
        u16p = ctypes.POINTER(ctypes.c_uint16)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lib.dfk_oracle_bf16_to_double.restype = ctypes.c_double
        lib.dfk_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.dfk_oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.dfk_oracle_double_to_bf16.argtypes = [ctypes.c_double]
        lib.dfk_oracle_silu.restype = ctypes.c_double
        lib.dfk_oracle_silu.argtypes = [ctypes.c_double]
        lib.dfk_oracle_threads.restype = ctypes.c_int
        lib.dfk_oracle_set_threads.restype = None
        lib.dfk_oracle_set_threads.argtypes = [ctypes.c_int]
        lib.dfk_oracle_rmsnorm.restype = ctypes.c_int
        lib.dfk_oracle_rmsnorm.argtypes = [u16p, u16p, ctypes.c_double, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, dp]
        lib.dfk_oracle_gate_up.restype = ctypes.c_int
        lib.dfk_oracle_gate_up.argtypes = [u16p, u16p, ctypes.c_double, u16p, u16p,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ip, ctypes.c_int, ctypes.c_int,
                                           dp, dp, dp]
        lib.dfk_oracle_down.restype = ctypes.c_int
        lib.dfk_oracle_down.argtypes = [dp, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ip, ctypes.c_int, ctypes.c_int, dp]
        u8p = ctypes.POINTER(ctypes.c_uint8)
        fp = ctypes.POINTER(ctypes.c_float)
        lib.dfk_oracle_e4m3_to_double.restype = ctypes.c_double
        lib.dfk_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.dfk_oracle_gate_up_fp8.restype = ctypes.c_int
        lib.dfk_oracle_gate_up_fp8.argtypes = [u16p, u16p, ctypes.c_double, u8p, fp, u8p, fp,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ip,
                                               ctypes.c_int, dp, dp, dp]
        lib.dfk_oracle_down_fp8.restype = ctypes.c_int
        lib.dfk_oracle_down_fp8.argtypes = [dp, u8p, fp, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ip, ctypes.c_int, dp]
        lib.dfk_oracle_rms_rescale.restype = ctypes.c_int
        lib.dfk_oracle_rms_rescale.argtypes = [dp, ctypes.c_double, ctypes.c_int,
                                               ctypes.c_int, dp]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


class _swapped:
    """Context manager: run the oracle functions on another build of the C
    source (used by the mutation test, which plants mistakes in a copy)."""

    def __init__(self, path):
        self.lib = _bind(ctypes.CDLL(path))

    def __enter__(self):
        global _lib
        self.prev, _lib = _load(), self.lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.prev
        return False


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy uint16), got %s" % a.dtype)
    return a


def _p(a, ctype):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return _load().dfk_oracle_threads()


def set_threads(n: int) -> None:
    """Use n OpenMP threads in later calls (results do not depend on n)."""
    _load().dfk_oracle_set_threads(int(n))


def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns (upper half of a binary32)."""
    b = _u16(bits)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    """Round doubles to bf16 bit patterns, nearest-even, in one step."""
    lib = _load()
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    flat_in, flat_out = v.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = lib.dfk_oracle_double_to_bf16(float(flat_in[i]))
    return out


def silu(a: float) -> float:
    """SiLU(a) = a / (1 + exp(-a)) in double."""
    return _load().dfk_oracle_silu(float(a))


def rmsnorm(x, gamma=None, eps=1e-5, mirror=False) -> np.ndarray:
    """RMSNorm rows of x [B, D] (bf16 bits) -> float64 [B, D]."""
    lib = _load()
    x = _u16(x)
    B, D = x.shape
    g = None if gamma is None else _u16(gamma)
    out = np.empty((B, D), dtype=np.float64)
    rc = lib.dfk_oracle_rmsnorm(_p(x, ctypes.c_uint16), _p(g, ctypes.c_uint16), float(eps),
                                B, D, int(mirror), _p(out, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_rmsnorm rejected its arguments")
    return out


def gate_up(x, wg, wu=None, layout=LAYOUT_ROW, gamma=None, eps=1e-5, rows=None,
            mirror=False, return_au=False):
    """h = SiLU(xn Wg^T) * (xn Wu^T) for the columns ``rows`` (all F if None).

    x [B, D] bf16 bits; gamma [D] bf16 bits or None (no RMSNorm);
    weights per ``layout``: row [F, D] each, col [D, F] each,
    interleaved wg [F, 2, D] (or [2F, D]) with wu None.
    Returns h [B, len(rows)] (and a, u when return_au) as float64.
    """
    lib = _load()
    x = _u16(x)
    B, D = x.shape
    wg = _u16(wg)
    if layout == LAYOUT_ROW:
        F = wg.shape[0]
        if wg.size != F * D:
            raise ValueError("row-major W_gate must be [F, D]")
    elif layout == LAYOUT_COL:
        F = wg.size // D
        if wg.size != F * D:
            raise ValueError("column-major W_gate must be [D, F]")
    elif layout == LAYOUT_INTERLEAVED:
        F = wg.size // (2 * D)
        if wg.size != 2 * F * D:
            raise ValueError("interleaved W must be [F, 2, D]")
    else:
        raise ValueError("unknown layout %r" % (layout,))
    if layout != LAYOUT_INTERLEAVED:
        wu = _u16(wu)
        if wu.size != wg.size:
            raise ValueError("W_up must match W_gate")
    else:
        wu = None
    g = None if gamma is None else _u16(gamma)
    if rows is None:
        r = None
        n = F
    else:
        r = np.ascontiguousarray(rows, dtype=np.int32)
        n = r.size
    h = np.empty((B, n), dtype=np.float64)
    a = np.empty((B, n), dtype=np.float64) if return_au else None
    u = np.empty((B, n), dtype=np.float64) if return_au else None
    rc = lib.dfk_oracle_gate_up(_p(x, ctypes.c_uint16), _p(g, ctypes.c_uint16), float(eps),
                                _p(wg, ctypes.c_uint16), _p(wu, ctypes.c_uint16), int(layout),
                                B, D, F, _p(r, ctypes.c_int), n, int(mirror),
                                _p(h, ctypes.c_double), _p(a, ctypes.c_double),
                                _p(u, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_gate_up rejected its arguments")
    return (h, a, u) if return_au else h


def down(h, wd, rows=None, mirror=False) -> np.ndarray:
    """y = h Wd^T for the rows ``rows`` of Wd (all D if None).

    h [B, F] float64 (or bf16 bits, converted exactly); wd [D, F] bf16 bits.
    """
    lib = _load()
    if np.asarray(h).dtype == np.uint16:
        h = bf16_to_f64(h)
    h = np.ascontiguousarray(h, dtype=np.float64)
    wd = _u16(wd)
    B, F = h.shape
    D = wd.shape[0]
    if wd.size != D * F:
        raise ValueError("W_down must be [D, F]")
    if rows is None:
        r, n = None, D
    else:
        r = np.ascontiguousarray(rows, dtype=np.int32)
        n = r.size
    y = np.empty((B, n), dtype=np.float64)
    rc = lib.dfk_oracle_down(_p(h, ctypes.c_double), _p(wd, ctypes.c_uint16), B, D, F,
                             _p(r, ctypes.c_int), n, int(mirror), _p(y, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_down rejected its arguments")
    return y


def mlp(x, wg, wu, wd, layout=LAYOUT_ROW, gamma=None, eps=1e-5, mirror=False):
    """Whole MLP: optional RMSNorm -> gate/up -> SwiGLU -> down.  Returns (h, y)."""
    h = gate_up(x, wg, wu, layout=layout, gamma=gamma, eps=eps, mirror=mirror)
    return h, down(h, wd, mirror=mirror)


def rms_rescale(y, eps=1e-5) -> np.ndarray:
    """Per-row y / sqrt(mean(y^2) + eps), in double (decode-stack step input)."""
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    B, D = y.shape
    out = np.empty_like(y)
    rc = lib.dfk_oracle_rms_rescale(_p(y, ctypes.c_double), float(eps), B, D,
                                    _p(out, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_rms_rescale rejected its arguments")
    return out


# ---------------------------------------------------------------- FP8 weights

def e4m3_to_f64(codes) -> np.ndarray:
    """Exact value of FP8 E4M3 codes (numpy uint8)."""
    lib = _load()
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    fo, fi = out.reshape(-1), c.reshape(-1)
    for i in range(fi.size):
        fo[i] = lib.dfk_oracle_e4m3_to_double(int(fi[i]))
    return out


def _u8(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint8:
        raise TypeError("FP8 codes must be numpy uint8, got %s" % a.dtype)
    return a


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def gate_up_fp8(x, qg, sg, qu, su, gamma=None, eps=1e-5, rows=None, return_au=False):
    """h = SiLU(xn Wg^T) * (xn Wu^T) with Wg = diag(sg) qg, Wu = diag(su) qu.

    x [B, D] bf16 bits; qg, qu [F, D] E4M3 codes (uint8); sg, su [F] float32.
    """
    lib = _load()
    x, qg, qu = _u16(x), _u8(qg), _u8(qu)
    sg, su = _f32(sg), _f32(su)
    B, D = x.shape
    F = qg.shape[0]
    if qg.shape != (F, D) or qu.shape != (F, D) or sg.size != F or su.size != F:
        raise ValueError("FP8 weights must be [F, D] with [F] scales")
    g = None if gamma is None else _u16(gamma)
    if rows is None:
        r, n = None, F
    else:
        r = np.ascontiguousarray(rows, dtype=np.int32)
        n = r.size
    h = np.empty((B, n), dtype=np.float64)
    a = np.empty((B, n), dtype=np.float64) if return_au else None
    u = np.empty((B, n), dtype=np.float64) if return_au else None
    rc = lib.dfk_oracle_gate_up_fp8(_p(x, ctypes.c_uint16), _p(g, ctypes.c_uint16), float(eps),
                                    _p(qg, ctypes.c_uint8), _p(sg, ctypes.c_float),
                                    _p(qu, ctypes.c_uint8), _p(su, ctypes.c_float), B, D, F,
                                    _p(r, ctypes.c_int), n, _p(h, ctypes.c_double),
                                    _p(a, ctypes.c_double), _p(u, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_gate_up_fp8 rejected its arguments")
    return (h, a, u) if return_au else h


def down_fp8(h, qd, sd, rows=None) -> np.ndarray:
    """y = h Wd^T with Wd = diag(sd) qd; qd [D, F] E4M3 codes, sd [D] float32."""
    lib = _load()
    if np.asarray(h).dtype == np.uint16:
        h = bf16_to_f64(h)
    h = np.ascontiguousarray(h, dtype=np.float64)
    qd, sd = _u8(qd), _f32(sd)
    B, F = h.shape
    D = qd.shape[0]
    if qd.shape != (D, F) or sd.size != D:
        raise ValueError("FP8 W_down must be [D, F] with [D] scales")
    if rows is None:
        r, n = None, D
    else:
        r = np.ascontiguousarray(rows, dtype=np.int32)
        n = r.size
    y = np.empty((B, n), dtype=np.float64)
    rc = lib.dfk_oracle_down_fp8(_p(h, ctypes.c_double), _p(qd, ctypes.c_uint8),
                                 _p(sd, ctypes.c_float), B, D, F, _p(r, ctypes.c_int), n,
                                 _p(y, ctypes.c_double))
    if rc != 0:
        raise ValueError("dfk_oracle_down_fp8 rejected its arguments")
    return y


def qkv(x, w_qkv, nq, nk, nv, gamma=None, eps=1e-5, rows=None):
    """RMSNorm (optional) + packed QKV projection; returns (q, k, v) float64.

    x [B, D] bf16 bits; w_qkv [nq + nk + nv, D] bf16 bits (rows of W_q, then
    W_k, then W_v).  With ``rows`` (indices into the packed output), returns
    the packed output o[:, rows] instead.  Composition of the RMSNorm and
    matrix-product oracles: xn stays float64, the product is the same
    definition as the down projection (sum_k xn[b][k] W[j][k])."""
    w = np.asarray(w_qkv)
    if w.shape[0] != nq + nk + nv:
        raise ValueError("w_qkv must have nq + nk + nv rows")
    xn = rmsnorm(x, gamma, eps) if gamma is not None else bf16_to_f64(np.asarray(x))
    o = down(xn, w, rows=rows)
    if rows is not None:
        return o
    return o[:, :nq], o[:, nq:nq + nk], o[:, nq + nk:]
