"""swiglu_mlp_dfk_b200 -- B200 (sm_100a) decode-stage SwiGLU MLP.

Thin Python binding over the C ABI of ``libdfk.so`` (declared in
``include/dfk.h``): the functions below carry the C entry points' names and
only marshal arguments -- torch tensors become device pointers, the current
torch stream becomes the ``stream`` argument, output tensors are allocated
when not given.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU path.  If ``libdfk.so`` is missing or no sm_100
device is present, every compute call raises ``DfkError``.

The method ("Deep Kernel Fusion for Transformer Decoding", episode
description): gate projection, up projection, SiLU and elementwise multiply
fused into one decode kernel, the down projection left separate, and a
profiler-driven scheduler choosing among row-major and column-major kernel
variants.
"""
import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# DFK_CHECKED=1 selects the bounds-checked build of the same library (every
# result store and activation load tests its index; failures are recorded in
# the device status word, read by dfk_device_error)
LIB_PATH = os.path.join(_PKG, "libdfk_checked.so" if os.environ.get("DFK_CHECKED") == "1"
                        else "libdfk.so")

# dfk_wlayout
DFK_W_ROW_MAJOR = 0
DFK_W_COL_MAJOR = 1
DFK_W_GU_INTERLEAVED = 2
DFK_W_ANY = -1
# dfk_op
DFK_OP_GATE_UP = 0
DFK_OP_RMSNORM_GATE_UP = 1
DFK_OP_DOWN = 2
DFK_OP_GATE_UP_FP8 = 3
DFK_OP_RMSNORM_GATE_UP_FP8 = 4
DFK_OP_DOWN_FP8 = 5
DFK_OP_QKV = 6
DFK_OP_RMSNORM_QKV = 7
# dfk_status
DFK_OK = 0
DFK_ERR_INVALID_ARG = 1
DFK_ERR_UNSUPPORTED_SHAPE = 2
DFK_ERR_UNSUPPORTED_LAYOUT = 3
DFK_ERR_MISALIGNED = 4
DFK_ERR_CUDA = 5
DFK_ERR_ARCH = 6
DFK_ERR_TIMEOUT = 7
DFK_ERR_NO_VARIANT = 8
DFK_ERR_BOUNDS = 9

_LAYOUTS = {"row": DFK_W_ROW_MAJOR, "col": DFK_W_COL_MAJOR, "interleaved": DFK_W_GU_INTERLEAVED,
            "any": DFK_W_ANY}

# Every symbol the header declares (the CPU test checks the library exports them all).
EXPORTED = (
    "dfk_swiglu_gate_up", "dfk_rmsnorm_swiglu_gate_up", "dfk_down_proj", "dfk_select_variant",
    "dfk_swiglu_gate_up_fp8", "dfk_rmsnorm_swiglu_gate_up_fp8", "dfk_down_proj_fp8",
    "dfk_rmsnorm_qkv_proj",
    "dfk_down_proj_static_scratch", "dfk_cached_variant", "dfk_variant_count",
    "dfk_variant_info", "dfk_clear_variant_cache", "dfk_rmsnorm",
    "dfk_gemv", "dfk_silu", "dfk_mul", "dfk_rms_rescale", "dfk_mlp_forward_host",
    "dfk_status_string", "dfk_last_error", "dfk_device_error", "dfk_version",
    "dfk_set_wait_limit", "dfk_selftest_bounded_wait",
    "dfk_tp_group_create", "dfk_tp_group_connect", "dfk_tp_down_proj_allreduce",
    "dfk_tp_group_destroy", "dfk_tp_down_proj_allreduce_emulated",
    "dfk_mlp_stack_workspace_bytes", "dfk_mlp_stack_step",
)


class DfkError(RuntimeError):
    """A libdfk call returned a non-zero dfk_status."""

    def __init__(self, status, msg):
        super().__init__("%s (status %d)" % (msg, status))
        self.status = status


class dfk_variant(ctypes.Structure):
    _fields_ = [("variant_id", ctypes.c_int), ("op", ctypes.c_int), ("layout", ctypes.c_int),
                ("family", ctypes.c_int), ("j_per_thread", ctypes.c_int),
                ("token_tile", ctypes.c_int), ("k_split", ctypes.c_int),
                ("k_tiles_per_stage", ctypes.c_int), ("acc_banks", ctypes.c_int),
                ("paired_fma", ctypes.c_int), ("full_m_tiles", ctypes.c_int),
                ("stages", ctypes.c_int), ("measured_us", ctypes.c_float),
                ("e4m3_mma", ctypes.c_int)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded libdfk.so (ctypes.CDLL); raises DfkError if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise DfkError(DFK_ERR_ARCH, "libdfk.so is not built (%s); run "
                               "`python -m swiglu_mlp_dfk_b200.build`" % LIB_PATH)
            L = ctypes.CDLL(LIB_PATH)
            vp, i, f, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
            sig = {
                "dfk_swiglu_gate_up": [vp, vp, vp, i, vp, i, i, i, i, vp],
                "dfk_rmsnorm_swiglu_gate_up": [vp, vp, f, vp, vp, i, vp, i, i, i, i, vp],
                "dfk_down_proj": [vp, vp, vp, i, i, i, i, vp],
                "dfk_down_proj_static_scratch": [vp, vp, vp, i, i, i, vp],
                "dfk_swiglu_gate_up_fp8": [vp, vp, vp, vp, vp, vp, i, i, i, i, vp],
                "dfk_rmsnorm_swiglu_gate_up_fp8": [vp, vp, f, vp, vp, vp, vp, vp, i, i, i, i,
                                                   vp],
                "dfk_down_proj_fp8": [vp, vp, vp, vp, i, i, i, i, vp],
                "dfk_rmsnorm_qkv_proj": [vp, vp, f, vp, vp, vp, vp, i, i, i, i, i, i, vp],
                "dfk_select_variant": [i, i, i, i, i, ctypes.POINTER(vp), vp,
                                       ctypes.POINTER(dfk_variant)],
                "dfk_cached_variant": [i, i, i, i, i, ctypes.POINTER(dfk_variant)],
                "dfk_variant_count": [],
                "dfk_variant_info": [i, ctypes.POINTER(dfk_variant)],
                "dfk_rmsnorm": [vp, vp, f, vp, i, i, vp],
                "dfk_gemv": [vp, vp, vp, i, i, i, i, vp],
                "dfk_silu": [vp, vp, ll, vp],
                "dfk_mul": [vp, vp, vp, ll, vp],
                "dfk_rms_rescale": [vp, f, vp, i, i, vp],
                "dfk_mlp_forward_host": [vp, vp, f, vp, vp, i, vp, vp, vp, vp, vp, i, i, i, vp],
                "dfk_device_error": [ctypes.POINTER(i)],
                "dfk_set_wait_limit": [ctypes.c_ulonglong],
                "dfk_selftest_bounded_wait": [vp, vp],
                "dfk_tp_group_create": [i, i, i, i, ctypes.POINTER(vp), vp],
                "dfk_tp_group_connect": [vp, vp],
                "dfk_tp_down_proj_allreduce": [vp, vp, vp, vp, i, i, i, vp],
                "dfk_tp_group_destroy": [vp],
                "dfk_tp_down_proj_allreduce_emulated": [i, vp, vp, vp, i, i, i, vp],
                "dfk_mlp_stack_step": [vp, f, vp, vp, i, vp, vp, vp, vp, vp, ll, i, i, i, i, vp],
                "dfk_status_string": [i],
                "dfk_last_error": [],
                "dfk_version": [],
            }
            for name, args in sig.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = i
            for name in ("dfk_status_string", "dfk_last_error", "dfk_version"):
                getattr(L, name).restype = ctypes.c_char_p
            L.dfk_mlp_stack_workspace_bytes.argtypes = [i, i, i, i]
            L.dfk_mlp_stack_workspace_bytes.restype = ll
            L.dfk_clear_variant_cache.argtypes = []
            L.dfk_clear_variant_cache.restype = None
            _lib = L
    return _lib


def _check(status):
    if status != DFK_OK:
        L = lib()
        raise DfkError(status, "%s: %s" % (L.dfk_status_string(status).decode(),
                                           L.dfk_last_error().decode()))


def _ptr(t):
    # a plain int: the c_void_p argtypes convert it (None passes NULL)
    return None if t is None else t.data_ptr()


# The current stream's handle.  torch.cuda.current_stream() builds a Stream
# object (about 3 us a call); the raw accessor under it returns the handle
# directly and is used when this torch has it.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


_BF16 = torch.bfloat16


def _dev_bf16(name, t):
    # on every call of the host-memory entry point: kept to a few attribute reads
    if t is None:
        return
    if not (isinstance(t, torch.Tensor) and t.dtype is _BF16 and t.is_cuda):
        raise DfkError(DFK_ERR_INVALID_ARG, "%s must be a bf16 CUDA tensor" % name)
    if not t.is_contiguous():
        raise DfkError(DFK_ERR_INVALID_ARG, "%s must be contiguous" % name)


def _layout(layout):
    return _LAYOUTS[layout] if isinstance(layout, str) else int(layout)


def _gate_up_shapes(x, w_gate, layout):
    B, D = x.shape
    if layout == DFK_W_ROW_MAJOR:
        F = w_gate.shape[0]
    elif layout == DFK_W_COL_MAJOR:
        F = w_gate.shape[-1]
    else:
        F = w_gate.numel() // (2 * D)
    return B, D, F


def dfk_swiglu_gate_up(x, w_gate, w_up=None, layout=DFK_W_ROW_MAJOR, h=None, variant=0,
                       stream=None):
    """h = SiLU(x W_gate^T) * (x W_up^T) in one kernel; returns h [B, d_ff] bf16."""
    layout = _layout(layout)
    for n, t in (("x", x), ("w_gate", w_gate), ("w_up", w_up), ("h", h)):
        _dev_bf16(n, t)
    B, D, F = _gate_up_shapes(x, w_gate, layout)
    if h is None:
        h = torch.empty((B, F), dtype=torch.bfloat16, device=x.device)
    _check(lib().dfk_swiglu_gate_up(_ptr(x), _ptr(w_gate), _ptr(w_up), layout, _ptr(h), B, D, F,
                                    int(variant), _stream(stream)))
    return h


def dfk_rmsnorm_swiglu_gate_up(x, gamma, eps, w_gate, w_up=None, layout=DFK_W_ROW_MAJOR, h=None,
                               variant=0, stream=None):
    """RMSNorm(x; gamma, eps) fused in front of the gate/up kernel; returns h."""
    layout = _layout(layout)
    for n, t in (("x", x), ("gamma", gamma), ("w_gate", w_gate), ("w_up", w_up), ("h", h)):
        _dev_bf16(n, t)
    B, D, F = _gate_up_shapes(x, w_gate, layout)
    if h is None:
        h = torch.empty((B, F), dtype=torch.bfloat16, device=x.device)
    _check(lib().dfk_rmsnorm_swiglu_gate_up(_ptr(x), _ptr(gamma), float(eps), _ptr(w_gate),
                                            _ptr(w_up), layout, _ptr(h), B, D, F, int(variant),
                                            _stream(stream)))
    return h


def dfk_down_proj(h, w_down, y=None, variant=0, stream=None):
    """y = h W_down^T (separate kernel); w_down [d_model, d_ff]; returns y [B, d_model]."""
    for n, t in (("h", h), ("w_down", w_down), ("y", y)):
        _dev_bf16(n, t)
    B, F = h.shape
    D = w_down.shape[0]
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=h.device)
    _check(lib().dfk_down_proj(_ptr(h), _ptr(w_down), _ptr(y), B, D, F, int(variant),
                               _stream(stream)))
    return y


def dfk_down_proj_static_scratch(h, w_down, y=None, stream=None):
    """y = h W_down^T without device allocation (library-resident scratch array).

    For callers that cannot allocate while running the MLP (a pre-reserved
    memory pool, stream capture); calls that overlap on the GPU race."""
    for n, t in (("h", h), ("w_down", w_down), ("y", y)):
        _dev_bf16(n, t)
    B, F = h.shape
    D = w_down.shape[0]
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=h.device)
    _check(lib().dfk_down_proj_static_scratch(_ptr(h), _ptr(w_down), _ptr(y), B, D, F,
                                              _stream(stream)))
    return y


def _dev_fp8(q, s, rows):
    """FP8 weights: uint8 (or torch.float8_e4m3fn) codes [rows, K] and fp32 scales [rows]."""
    if not isinstance(q, torch.Tensor) or not q.is_cuda or q.dim() != 2 or \
            q.dtype not in (torch.uint8, torch.float8_e4m3fn) or not q.is_contiguous():
        raise DfkError(DFK_ERR_INVALID_ARG, "FP8 weights must be contiguous 2-D uint8 or "
                       "float8_e4m3fn CUDA tensors")
    if not isinstance(s, torch.Tensor) or not s.is_cuda or s.dtype != torch.float32 or \
            not s.is_contiguous() or s.numel() != rows:
        raise DfkError(DFK_ERR_INVALID_ARG, "scales must be contiguous fp32 CUDA tensors of %d "
                       "elements" % rows)


def dfk_swiglu_gate_up_fp8(x, q_gate, s_gate, q_up, s_up, h=None, variant=0, stream=None):
    """h = SiLU(x (s_g Q_g)^T) * (x (s_u Q_u)^T) with FP8 E4M3 codes Q [d_ff, d_model] and
    fp32 row scales s [d_ff]; returns h [B, d_ff] bf16."""
    _dev_bf16("x", x)
    _dev_bf16("h", h)
    B, D = x.shape
    F = q_gate.shape[0]
    _dev_fp8(q_gate, s_gate, F)
    _dev_fp8(q_up, s_up, F)
    if h is None:
        h = torch.empty((B, F), dtype=torch.bfloat16, device=x.device)
    _check(lib().dfk_swiglu_gate_up_fp8(_ptr(x), _ptr(q_gate), _ptr(s_gate), _ptr(q_up),
                                        _ptr(s_up), _ptr(h), B, D, F, int(variant),
                                        _stream(stream)))
    return h


def dfk_rmsnorm_swiglu_gate_up_fp8(x, gamma, eps, q_gate, s_gate, q_up, s_up, h=None, variant=0,
                                   stream=None):
    """RMSNorm(x; gamma, eps) fused in front of the FP8 gate/up kernel; returns h."""
    _dev_bf16("x", x)
    _dev_bf16("gamma", gamma)
    _dev_bf16("h", h)
    B, D = x.shape
    F = q_gate.shape[0]
    _dev_fp8(q_gate, s_gate, F)
    _dev_fp8(q_up, s_up, F)
    if h is None:
        h = torch.empty((B, F), dtype=torch.bfloat16, device=x.device)
    _check(lib().dfk_rmsnorm_swiglu_gate_up_fp8(_ptr(x), _ptr(gamma), float(eps), _ptr(q_gate),
                                                _ptr(s_gate), _ptr(q_up), _ptr(s_up), _ptr(h),
                                                B, D, F, int(variant), _stream(stream)))
    return h


def dfk_down_proj_fp8(h, q_down, s_down, y=None, variant=0, stream=None):
    """y = h (s_d Q_d)^T with FP8 E4M3 codes Q_d [d_model, d_ff] and fp32 row scales s_d
    [d_model]; returns y [B, d_model] bf16."""
    _dev_bf16("h", h)
    _dev_bf16("y", y)
    B, F = h.shape
    D = q_down.shape[0]
    _dev_fp8(q_down, s_down, D)
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=h.device)
    _check(lib().dfk_down_proj_fp8(_ptr(h), _ptr(q_down), _ptr(s_down), _ptr(y), B, D, F,
                                   int(variant), _stream(stream)))
    return y


def dfk_rmsnorm_qkv_proj(x, gamma, eps, w_qkv, n_q, n_k, n_v, q=None, k=None, v=None,
                         variant=0, stream=None):
    """RMSNorm(x; gamma, eps) (skipped when gamma is None) + packed QKV projection with
    w_qkv [n_q + n_k + n_v, d_model]; returns (q, k, v), [B, n_q] / [B, n_k] / [B, n_v]."""
    for n, t in (("x", x), ("gamma", gamma), ("w_qkv", w_qkv), ("q", q), ("k", k), ("v", v)):
        _dev_bf16(n, t)
    B, D = x.shape
    if w_qkv.shape != (n_q + n_k + n_v, D):
        raise DfkError(DFK_ERR_INVALID_ARG, "w_qkv must be [n_q + n_k + n_v, d_model]")
    outs = []
    for t, n in ((q, n_q), (k, n_k), (v, n_v)):
        outs.append(torch.empty((B, n), dtype=torch.bfloat16, device=x.device) if t is None else t)
    _check(lib().dfk_rmsnorm_qkv_proj(_ptr(x), _ptr(gamma), float(eps), _ptr(w_qkv),
                                      _ptr(outs[0]) if n_q else None,
                                      _ptr(outs[1]) if n_k else None,
                                      _ptr(outs[2]) if n_v else None,
                                      B, D, n_q, n_k, n_v, int(variant), _stream(stream)))
    return tuple(outs)


def dfk_gemv(x, w, out=None, variant=0, stream=None):
    """out = x W^T with W [N, K] row-major (unfused-baseline building block)."""
    for n, t in (("x", x), ("w", w), ("out", out)):
        _dev_bf16(n, t)
    B, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((B, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().dfk_gemv(_ptr(x), _ptr(w), _ptr(out), B, K, N, int(variant), _stream(stream)))
    return out


def dfk_rmsnorm(x, gamma, eps, out=None, stream=None):
    """Standalone RMSNorm (unfused-baseline building block)."""
    for n, t in (("x", x), ("gamma", gamma), ("out", out)):
        _dev_bf16(n, t)
    B, D = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(lib().dfk_rmsnorm(_ptr(x), _ptr(gamma), float(eps), _ptr(out), B, D, _stream(stream)))
    return out


def dfk_rms_rescale(y, eps=1e-5, out=None, stream=None):
    """out = y / sqrt(mean(y^2) + eps) per row (decode-stack step input)."""
    for n, t in (("y", y), ("out", out)):
        _dev_bf16(n, t)
    B, D = y.shape
    if out is None:
        out = torch.empty_like(y)
    _check(lib().dfk_rms_rescale(_ptr(y), float(eps), _ptr(out), B, D, _stream(stream)))
    return out


def dfk_silu(a, out=None, stream=None):
    """out = SiLU(a) elementwise (unfused-baseline building block)."""
    _dev_bf16("a", a)
    if out is None:
        out = torch.empty_like(a)
    _dev_bf16("out", out)
    _check(lib().dfk_silu(_ptr(a), _ptr(out), a.numel(), _stream(stream)))
    return out


def dfk_mul(a, b, out=None, stream=None):
    """out = a * b elementwise (unfused-baseline building block)."""
    _dev_bf16("a", a)
    _dev_bf16("b", b)
    if out is None:
        out = torch.empty_like(a)
    _dev_bf16("out", out)
    _check(lib().dfk_mul(_ptr(a), _ptr(b), _ptr(out), a.numel(), _stream(stream)))
    return out


def dfk_mlp_forward_host(x_host, gamma, eps, w_gate, w_up, layout, w_down, y_host, x_dev, h_dev,
                         y_dev, stream=None):
    """One MLP layer from host memory: x_host -> device -> gate/up -> down -> y_host."""
    layout = _layout(layout)
    for n, t in (("gamma", gamma), ("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down),
                 ("x_dev", x_dev), ("h_dev", h_dev), ("y_dev", y_dev)):
        _dev_bf16(n, t)
    B, D = x_host.shape
    F = h_dev.shape[1]
    _check(lib().dfk_mlp_forward_host(_ptr(x_host), _ptr(gamma), float(eps), _ptr(w_gate),
                                      _ptr(w_up), layout, _ptr(w_down), _ptr(y_host),
                                      _ptr(x_dev), _ptr(h_dev), _ptr(y_dev), B, D, F,
                                      _stream(stream)))
    return y_host


def dfk_select_variant(op, B, d_model, d_ff, layout=DFK_W_ROW_MAJOR, sample=None, stream=None):
    """Time the variants of ``op`` for the shape and cache the winner; returns a dict."""
    layout = _layout(layout)
    out = dfk_variant()
    arr = None
    if sample is not None:
        arr = (ctypes.c_void_p * len(sample))(*[None if t is None else t.data_ptr()
                                                for t in sample])
    _check(lib().dfk_select_variant(int(op), int(B), int(d_model), int(d_ff), layout, arr,
                                    _stream(stream), ctypes.byref(out)))
    return out.as_dict()


def dfk_cached_variant(op, B, d_model, d_ff, layout=DFK_W_ROW_MAJOR):
    """The scheduler's cached decision for the shape (dict), or None if none yet."""
    out = dfk_variant()
    st = lib().dfk_cached_variant(int(op), int(B), int(d_model), int(d_ff), _layout(layout),
                                  ctypes.byref(out))
    if st == DFK_ERR_NO_VARIANT:
        return None
    _check(st)
    return out.as_dict()


def dfk_variant_count():
    return lib().dfk_variant_count()


def dfk_variant_info(variant_id):
    out = dfk_variant()
    _check(lib().dfk_variant_info(int(variant_id), ctypes.byref(out)))
    return out.as_dict()


def dfk_clear_variant_cache():
    lib().dfk_clear_variant_cache()


def dfk_device_error():
    """Read and clear the device error word; returns the code (0 = none)."""
    code = ctypes.c_int(0)
    st = lib().dfk_device_error(ctypes.byref(code))
    if st not in (DFK_OK, DFK_ERR_TIMEOUT, DFK_ERR_BOUNDS):
        _check(st)
    return code.value


def dfk_device_status():
    """Read and clear the device error word; returns (dfk_status, code, text)."""
    code = ctypes.c_int(0)
    st = lib().dfk_device_error(ctypes.byref(code))
    return st, code.value, lib().dfk_last_error().decode() if st else ""


def dfk_set_wait_limit(ns):
    """Limit of the kernels' pipeline waits on the current device (0 = default 4 s)."""
    _check(lib().dfk_set_wait_limit(int(ns)))


def dfk_selftest_bounded_wait(elapsed_ns=None, stream=None):
    """Launch the bounded-wait self-test; returns the int64 device tensor that
    receives the time the wait took before giving up (ns)."""
    if elapsed_ns is None:
        elapsed_ns = torch.zeros(1, dtype=torch.int64, device="cuda")
    _check(lib().dfk_selftest_bounded_wait(_ptr(elapsed_ns), _stream(stream)))
    return elapsed_ns


def dfk_version():
    return lib().dfk_version().decode()


# ---- tensor-parallel down projection (see swiglu_mlp_dfk_b200.tp for the MLP)

DFK_TP_HANDLE_BYTES = 64


def dfk_tp_group_create(world, rank, max_B, d_model):
    """Returns (group handle, this rank's IPC handle as bytes)."""
    g = ctypes.c_void_p()
    hb = ctypes.create_string_buffer(DFK_TP_HANDLE_BYTES)
    _check(lib().dfk_tp_group_create(int(world), int(rank), int(max_B), int(d_model),
                                     ctypes.byref(g), hb))
    return g, hb.raw


def dfk_tp_group_connect(group, handles):
    """handles: every rank's IPC handle (bytes), in rank order."""
    blob = b"".join(handles)
    _check(lib().dfk_tp_group_connect(group, ctypes.create_string_buffer(blob, len(blob))))


def dfk_tp_down_proj_allreduce(group, h, w_down_shard, y=None, stream=None):
    B, F = h.shape
    D = w_down_shard.shape[0]
    if y is None:
        y = torch.empty(B, D, dtype=torch.bfloat16, device=h.device)
    _check(lib().dfk_tp_down_proj_allreduce(group, _ptr(h), _ptr(w_down_shard), _ptr(y), B, D,
                                            F, _stream(stream)))
    return y


def dfk_tp_group_destroy(group):
    _check(lib().dfk_tp_group_destroy(group))


def dfk_tp_down_proj_allreduce_emulated(h_all, w_all, y_all=None, stream=None):
    """h_all [world][B][F_shard], w_all [world][D][F_shard] -> y_all [world][B][D]."""
    P, B, F = h_all.shape
    D = w_all.shape[1]
    if y_all is None:
        y_all = torch.empty(P, B, D, dtype=torch.bfloat16, device=h_all.device)
    _check(lib().dfk_tp_down_proj_allreduce_emulated(P, _ptr(h_all), _ptr(w_all), _ptr(y_all),
                                                     B, D, F, _stream(stream)))
    return y_all


# ---- one decode step of a layer stack in one persistent kernel

def dfk_mlp_stack_workspace_bytes(layers, B, d_model, d_ff):
    n = lib().dfk_mlp_stack_workspace_bytes(int(layers), int(B), int(d_model), int(d_ff))
    if n < 0:
        _check(DFK_ERR_UNSUPPORTED_SHAPE)
    return n


def dfk_mlp_stack_step(gammas, eps, w_gate, w_up, w_down, x, h_all, y_all, workspace,
                       layout=DFK_W_ROW_MAJOR, stream=None):
    """gammas [L, D], w_gate / w_up [L, F, D] (row-major) or [L, D, F] (layout "col"),
    w_down [L, D, F], x [B, D] (updated in place), h_all [L, B, F], y_all [L, B, D],
    workspace: uint8 device tensor."""
    layout = _layout(layout)
    L, D, F = w_down.shape
    B = x.shape[0]
    _check(lib().dfk_mlp_stack_step(_ptr(gammas), float(eps), _ptr(w_gate), _ptr(w_up), layout,
                                    _ptr(w_down), _ptr(x), _ptr(h_all), _ptr(y_all),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    L, B, D, F, _stream(stream)))
