"""Kimi Delta Attention (KDA) for NVIDIA B200 -- Python binding of ``libkda.so``.

The functions here only marshal arguments into the C ABI declared in
``include/kda.h`` (same names); every step of the computation runs in the
library's CUDA kernels. PyTorch supplies device memory and the current CUDA
stream. If the library is missing the calls raise -- there is no fallback.

Build the library with ``python -m gated_delta_rule_125_b200.build``.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = ["kda_prefill", "kda_decode_step", "kda_prefill_workspace_size", "kda_prefill_launches",
           "kda_device_error", "kda_prefill_noalloc", "kda_short_conv_swish", "kda_backward",
           "kda_prefill_workspace_min", "kda_set_wait_limit_ns", "kda_status_string", "kda_version", "KDAError",
           "library_path", "load_library", "KDA_OK", "KDA_ERR_INVALID_ARG",
           "KDA_ERR_UNSUPPORTED", "KDA_ERR_MISALIGNED", "KDA_ERR_WORKSPACE", "KDA_ERR_CUDA",
           "KDA_ERR_TIMEOUT", "KDA_FLAG_NO_L2NORM", "KDA_FLAG_EXACT", "KDA_FLAG_SCALAR_GATE"]

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_MISALIGNED = 0, 1, 2, 3
KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = 4, 5, 6
KDA_DTYPE_F32, KDA_DTYPE_BF16 = 0, 1
KDA_FLAG_NO_L2NORM, KDA_FLAG_EXACT, KDA_FLAG_SCALAR_GATE = 0x1, 0x2, 0x4

EXPORTED_SYMBOLS = ("kda_status_string", "kda_version", "kda_prefill_workspace_size",
                    "kda_prefill_workspace_min", "kda_prefill_launches", "kda_prefill",
                    "kda_prefill_ex", "kda_decode_step", "kda_decode_step_ex", "kda_device_error",
                    "kda_prefill_noalloc", "kda_short_conv_swish", "kda_short_conv_launches",
                    "kda_decode_step_conv", "kda_backward_workspace_size", "kda_backward",
                    "kda_set_wait_limit_ns", "kda_prefill_conv")


class OutputGate(ctypes.Structure):
    """``kda_output_gate``: the fused output step (RMSNorm over d_v, sigmoid gate)."""
    _fields_ = [("gate", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("eps", ctypes.c_float)]


class ShortConv(ctypes.Structure):
    """``kda_short_conv``: causal short convolution + Swish (width, weight, states)."""
    _fields_ = [("width", ctypes.c_int32), ("weight", ctypes.c_void_p), ("state_in", ctypes.c_void_p),
                ("state_out", ctypes.c_void_p)]

_lib = None


def library_path() -> str:
    return os.environ.get("KDA_LIBRARY",
                          os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so"))


class KDAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s: %s" % (what, kda_status_string(status)))
        self.status = status


def load_library():
    """Load ``libkda.so`` (raises ``OSError`` if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise OSError("libkda.so not found at %s; build it with "
                      "`python -m gated_delta_rule_125_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    i32, i64, u32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.restype = i32
    for f in (lib.kda_prefill_workspace_size, lib.kda_prefill_workspace_min):
        f.argtypes = [i32, i64, i32, i32, i32, i32, ctypes.c_int, i32, u32]
        f.restype = sz
    lib.kda_prefill_launches.argtypes = [i32, i64, i32, i32, i32, i32, ctypes.c_int, i32, u32, sz]
    lib.kda_prefill_launches.restype = i64
    lib.kda_prefill.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i64, i32, i32, i32, i32,
                                ctypes.c_int, i32, u32, vp, fp, vp, sz, vp]
    lib.kda_prefill.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, i32, i32, i32, i32, ctypes.c_int,
                                    u32, vp, vp]
    lib.kda_decode_step.restype = ctypes.c_int
    og = ctypes.POINTER(OutputGate)
    lib.kda_prefill_ex.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i64, i32, i32, i32, i32,
                                   ctypes.c_int, i32, u32, og, vp, fp, vp, sz, vp]
    lib.kda_prefill_ex.restype = ctypes.c_int
    lib.kda_decode_step_ex.argtypes = [vp, vp, vp, fp, fp, fp, i32, i32, i32, i32, ctypes.c_int,
                                       u32, og, vp, vp]
    lib.kda_decode_step_ex.restype = ctypes.c_int
    lib.kda_prefill_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i64, i32, i32, i32,
                                        i32, ctypes.c_int, i32, u32, vp, fp, vp]
    lib.kda_prefill_noalloc.restype = ctypes.c_int
    lib.kda_device_error.argtypes = [ctypes.POINTER(i32), i32]
    lib.kda_device_error.restype = ctypes.c_int
    sc = ctypes.POINTER(ShortConv)
    lib.kda_short_conv_swish.argtypes = [vp, vp, sc, ip, i32, i64, i32, ctypes.c_int, vp]
    lib.kda_short_conv_swish.restype = ctypes.c_int
    lib.kda_short_conv_launches.argtypes = [i32, i32, i64]
    lib.kda_short_conv_launches.restype = i64
    lib.kda_decode_step_conv.argtypes = [vp, vp, vp, fp, fp, fp, i32, i32, i32, i32, ctypes.c_int,
                                         u32, sc, sc, sc, og, vp, vp]
    lib.kda_decode_step_conv.restype = ctypes.c_int
    lib.kda_prefill_conv.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i64, i32, i32, i32, i32,
                                     ctypes.c_int, i32, u32, sc, sc, sc, og, vp, fp, vp, sz, vp]
    lib.kda_prefill_conv.restype = ctypes.c_int
    lib.kda_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, ctypes.c_int, i32, u32]
    lib.kda_backward_workspace_size.restype = sz
    lib.kda_backward.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, i64, i32, i32, i32, i32, ctypes.c_int, i32, u32,
                                 vp, fp, fp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.kda_backward.restype = ctypes.c_int
    lib.kda_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.kda_set_wait_limit_ns.restype = ctypes.c_uint64
    _lib = lib
    return lib


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(load_library().kda_version())


def kda_device_error(reset: bool = True) -> int:
    """Device error word of the current device (0: no bounded wait ran out). Synchronous."""
    code = ctypes.c_int32(0)
    load_library().kda_device_error(ctypes.byref(code), int(bool(reset)))
    return int(code.value)


def kda_set_wait_limit_ns(ns: int) -> int:
    """Bound (ns) of the prefill's waits between CTAs for later calls; 0 = default (2 s).
    Returns the previous bound (``kda_set_wait_limit_ns`` in ``include/kda.h``)."""
    return int(load_library().kda_set_wait_limit_ns(int(ns)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr() or None


def _out_gate(out_gate):
    """(gate, weight, eps) -> a ``kda_output_gate`` (None -> NULL)."""
    if out_gate is None:
        return None
    g, w, eps = out_gate
    return ctypes.byref(OutputGate(_ptr(g), _ptr(w), float(eps)))


def _conv(conv):
    """(weight [C, W] fp32, state_in or None, state_out or None) -> a ``kda_short_conv`` (None -> NULL)."""
    if conv is None:
        return None
    w, sin, sout = conv
    return ctypes.byref(ShortConv(int(w.shape[-1]), _ptr(w), _ptr(sin), _ptr(sout)))


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _flags(l2norm, exact, scalar_gate=False):
    return ((0 if l2norm else KDA_FLAG_NO_L2NORM) | (KDA_FLAG_EXACT if exact else 0) |
            (KDA_FLAG_SCALAR_GATE if scalar_gate else 0))


def kda_prefill_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype,
                               chunk=64, l2norm=True, exact=False) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load_library().kda_prefill_workspace_size(num_seqs, total_tokens, max_seqlen, H,
                                                        dk, dv, code, chunk,
                                                        _flags(l2norm, exact)))


def kda_prefill_workspace_min(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype,
                              chunk=64, l2norm=True, exact=False) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load_library().kda_prefill_workspace_min(num_seqs, total_tokens, max_seqlen, H,
                                                       dk, dv, code, chunk,
                                                       _flags(l2norm, exact)))


def kda_prefill_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, workspace_bytes,
                         chunk=64, l2norm=True, exact=False) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load_library().kda_prefill_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                                  code, chunk, _flags(l2norm, exact),
                                                  workspace_bytes))


def kda_prefill(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, max_seqlen=None,
                chunk=64, l2norm=True, exact=False, o=None, S_T=None, workspace=None,
                out_gate=None, conv=None, stream=None):
    """Chunkwise KDA prefill (``kda_prefill`` in ``include/kda.h``).

    q, k ``[T,H,dk]``, v ``[T,H,dv]`` (bf16 or fp32), log_alpha ``[T,H,dk]`` fp32
    (or ``[T,H]``: one gate per token and head, the Gated DeltaNet form), beta ``[T,H]`` fp32, S0 ``[N,H,dk,dv]`` fp32 or None, cu_seqlens ``[N+1]`` int32
    on the device or None. Returns ``(o [T,H,dv], S_T [N,H,dk,dv])``. Outputs and
    the workspace are allocated with torch when not given. ``max_seqlen`` (host
    int) avoids a device-to-host read of ``cu_seqlens``. ``out_gate = (gate
    [T,H,dv] (dtype of q), weight [dv] fp32, eps)`` fuses the layer's output step
    (``kda_prefill_ex``): o <- RMSNorm(o) * weight * sigmoid(gate). ``conv=(cq, ck, cv)``,
    each None or ``(weight [H*d, W] fp32, state_in, state_out)`` with states
    ``[N, W-1, H*d]`` (None: zeros / not written): q, k, v are the raw projections and the
    short convolution + Swish runs inside the prefill's loads (``kda_prefill_conv``).
    """
    lib = load_library()
    T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if max_seqlen is None:
        if cu_seqlens is None:
            max_seqlen = T
        else:
            c = cu_seqlens.to("cpu", torch.int64)
            max_seqlen = int((c[1:] - c[:-1]).max()) if N > 0 else 0
    if o is None:
        o = torch.empty((T, H, dv), dtype=q.dtype, device=dev)
    if S_T is None:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    code = _dtype_code(q)
    flags = _flags(l2norm, exact, log_alpha.dim() == 2)
    if workspace is None:
        nbytes = lib.kda_prefill_workspace_size(N, T, max_seqlen, H, dk, dv, code, chunk, flags)
        if nbytes == 0:
            nbytes = 256
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if conv is None:
        rc = lib.kda_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                _ptr(cu_seqlens), N, T, int(max_seqlen), H, dk, dv, code, chunk, flags,
                                _out_gate(out_gate), _ptr(o), _ptr(S_T), _ptr(workspace),
                                workspace.numel(), _stream(stream, dev))
    else:
        cq, ck, cv = conv
        rc = lib.kda_prefill_conv(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                  _ptr(cu_seqlens), N, T, int(max_seqlen), H, dk, dv, code, chunk, flags,
                                  _conv(cq), _conv(ck), _conv(cv), _out_gate(out_gate), _ptr(o), _ptr(S_T),
                                  _ptr(workspace), workspace.numel(), _stream(stream, dev))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_prefill")
    return o, S_T


def kda_prefill_noalloc(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, max_seqlen,
                        chunk=64, l2norm=True, exact=False, o, S_T, stream=None):
    """``kda_prefill_noalloc`` in ``include/kda.h``: the prefill with the library's fixed
    scratch array instead of a workspace, for callers that cannot allocate device
    memory. Outputs ``o`` and ``S_T`` are the caller's; nothing is allocated here.
    Calls sharing the array must not overlap on the GPU."""
    lib = load_library()
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    rc = lib.kda_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                 _ptr(cu_seqlens), N, T, int(max_seqlen), H, dk, dv, _dtype_code(q),
                                 chunk, _flags(l2norm, exact, log_alpha.dim() == 2), _ptr(o), _ptr(S_T),
                                 _stream(stream, q.device))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_prefill_noalloc")
    return o, S_T


def kda_decode_step(q, k, v, log_alpha, beta, S, *, l2norm=True, o=None, out_gate=None,
                    conv=None, stream=None):
    """One KDA decode step (``kda_decode_step`` in ``include/kda.h``), S updated in place.

    q, k ``[N,H,dk]``, v ``[N,H,dv]``, log_alpha ``[N,H,dk]`` (or ``[N,H]``, one gate per
    head) fp32, beta ``[N,H]`` fp32,
    S ``[N,H,dk,dv]`` fp32. Returns o ``[N,H,dv]``. ``conv=(cq, ck, cv)``, each None or
    ``(weight [H*d, W] fp32, state_in, state_out)`` with states ``[N, W-1, H*d]``: the
    short convolution + Swish fused into the loads (``kda_decode_step_conv``).
    """
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    if conv is None:
        rc = lib.kda_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S),
                                    N, H, dk, dv, _dtype_code(q), _flags(l2norm, False, log_alpha.dim() == 2),
                                    _out_gate(out_gate), _ptr(o), _stream(stream, q.device))
    else:
        cq, ck, cv = conv
        rc = lib.kda_decode_step_conv(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S),
                                      N, H, dk, dv, _dtype_code(q), _flags(l2norm, False, log_alpha.dim() == 2),
                                      _conv(cq), _conv(ck), _conv(cv), _out_gate(out_gate), _ptr(o),
                                      _stream(stream, q.device))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_decode_step")
    return o


def kda_short_conv_swish(x, weight, cu_seqlens=None, *, state_in=None, state_out=None, y=None,
                         stream=None):
    """Causal short convolution + Swish (``kda_short_conv_swish`` in ``include/kda.h``).

    x ``[T, C]`` (or ``[T, H, d]``, C = H * d) in bf16 or fp32, weight ``[C, W]`` fp32,
    states ``[N, W-1, C]`` in x's dtype (state_out may be state_in). Returns y like x.
    """
    lib = load_library()
    T = x.shape[0]
    C = int(math.prod(x.shape[1:]))
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if y is None:
        y = torch.empty_like(x)
    c = ShortConv(int(weight.shape[-1]), _ptr(weight), _ptr(state_in), _ptr(state_out))
    rc = lib.kda_short_conv_swish(_ptr(x), _ptr(y), ctypes.byref(c), _ptr(cu_seqlens), N, T, C,
                                  _dtype_code(x), _stream(stream, x.device))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_short_conv_swish")
    return y


def kda_backward(q, k, v, log_alpha, beta, do, dS_T=None, S0=None, cu_seqlens=None, *, max_seqlen=None,
                 l2norm=True, workspace=None, want_dS0=True, stream=None):
    """Backward of the prefill (``kda_backward`` in ``include/kda.h``): the gradients of a
    loss through ``o`` and ``S_T`` given ``do = dL/do`` ``[T,H,dv]`` (io dtype) and
    ``dS_T = dL/dS_T`` ``[N,H,dk,dv]`` fp32 (None: zero). Returns fp32
    ``(dq, dk, dv, dlog_alpha, dbeta, dS0)`` (dS0 None unless ``want_dS0``)."""
    lib = load_library()
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if max_seqlen is None:
        max_seqlen = T if cu_seqlens is None else int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item())
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dkk = torch.empty((T, H, dk), **f32), torch.empty((T, H, dk), **f32)
    dvv = torch.empty((T, H, dv), **f32)
    dla = torch.empty(tuple(log_alpha.shape), **f32)  # [T,H,dk], or [T,H] with one gate per head
    db = torch.empty((T, H), **f32)
    dS0 = torch.empty((N, H, dk, dv), **f32) if want_dS0 else None
    flags = _flags(l2norm, False, log_alpha.dim() == 2)
    code = _dtype_code(q)
    if workspace is None:
        nbytes = lib.kda_backward_workspace_size(N, T, max_seqlen, H, dk, dv, code, 64, flags)
        if nbytes == 0:
            raise KDAError(KDA_ERR_INVALID_ARG, "kda_backward_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    rc = lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                          N, T, max_seqlen, H, dk, dv, code, 64, flags, _ptr(do), _ptr(dS_T),
                          _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(db), _ptr(dS0),
                          _ptr(workspace), workspace.numel(), _stream(stream, q.device))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_backward")
    return dq, dkk, dvv, dla, db, dS0
