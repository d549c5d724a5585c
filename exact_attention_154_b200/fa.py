"""Python binding of ``libfa_sm100.so`` (the C ABI in ``include/fa.h``).

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every step of the attention forward runs in the library's kernel.
There is no fallback: if the library is missing or the device is not an
sm_100 GPU, the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from .synth import BF16, FP16

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_sm100.so")
_lock = threading.Lock()
_lib = None

FA_OK = 0
FA_ERR_ARG, FA_ERR_ALIGN, FA_ERR_HEADDIM, FA_ERR_DTYPE = -1, -2, -3, -4
FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_DEVICE = -5, -6, -7, -8
FA_ERR_SEQLENS = -9

#: every function the C header declares, with (restype, argtypes)
_VP, _FP, _I, _F = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "fa_fwd": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "fa_fwd_qkvpacked": (_I, [_VP, _VP, _FP, _I, _I, _I, _I, _F, _I, _F, _I, _VP]),
    "fa_fwd_ext": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _F, _I, _I, _I, _FP, _I, _VP]),
    "fa_fwd_qkvpacked_ext": (_I, [_VP, _VP, _FP, _I, _I, _I, _I, _F, _I, _F, _I, _I, _FP, _I,
                                  _VP]),
    "fa_fwd_fp8": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _F, _F, _F, _F, _I, _VP]),
    "fa_fwd_varlen": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _I, _I, _I, _I, _I, _F, _I, _I, _I, _FP,
                           _I, _VP]),
    "fa_bwd": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _F, _I, _I,
                    _VP]),
    "fa_bwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I,
                            _I, _VP]),
    "fa_strerror": (ctypes.c_char_p, [_I]),
    "fa_device_status": (_I, [_I, ctypes.POINTER(ctypes.c_uint)]),
    "fa_debug_watchdog_selftest": (_I, [ctypes.c_ulonglong, _VP]),
    "fa_launch_ctas": (_I, [_I, _I, _I, _I, _I]),
    "fa_debug_exp2_poly": (_I, [_VP, _VP, _I, _VP]),
    "fa_debug_set_wait_limit": (_I, [ctypes.c_ulonglong]),
    "fa_version": (_I, []),
}


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} ({status})")
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -c 'import __graft_entry__ as g; g.build()'`")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load().fa_strerror(int(status)).decode()


def version() -> int:
    return int(load().fa_version())


_DT = {torch.float16: FP16, torch.bfloat16: BF16}


def _stream_ptr(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def same_device(named) -> torch.device:
    """The one device every ``(name, tensor)`` pair lives on; raises if they differ.

    The library resolves its per-device state (SM count, kernel attributes, the
    backward's scratch array) from the *current* device, so every call runs
    with the tensors' device made current (see :func:`_on`)."""
    dev = None
    for name, t in named:
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    return dev


def _on(dev: torch.device):
    """Context that makes ``dev`` the current CUDA device for one library call."""
    return torch.cuda.device(dev)


def _check_tensor(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in _DT:
        raise ValueError(f"{name} must be float16 or bfloat16")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _window(window) -> tuple[int, int]:
    left, right = (int(window[0]), int(window[1]))
    return left, right


def _slopes(alibi_slopes, H: int, dev: torch.device):
    """The ``[H]`` fp32 slope tensor on ``dev`` (or None) and its pointer."""
    if alibi_slopes is None:
        return None, None
    if not isinstance(alibi_slopes, torch.Tensor):
        alibi_slopes = torch.as_tensor(alibi_slopes, dtype=torch.float32)
    if alibi_slopes.shape != (H,) or alibi_slopes.dtype != torch.float32:
        raise ValueError("alibi_slopes must be a float32 tensor of shape [H]")
    alibi_slopes = alibi_slopes.to(dev).contiguous()
    return alibi_slopes, alibi_slopes.data_ptr()


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
        causal: bool = False, out: torch.Tensor | None = None,
        lse: torch.Tensor | None = None, return_lse: bool = True,
        window_size=(-1, -1), alibi_slopes=None):
    """Attention forward on ``[B, H, N, d]`` tensors (``[B, N, d]`` is taken as H=1).

    Returns ``(O, LSE)`` (``LSE`` is ``[B, H, N]`` fp32, or None when
    ``return_lse`` is False).  ``scale=None`` means ``1/sqrt(d)``.
    ``window_size=(left, right)``: key j visible from query i iff
    ``i - left <= j <= i + right`` (-1: unbounded).  ``alibi_slopes``: ``[H]``
    fp32; the scaled score gets ``-slope[h] * |i - j|``.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(t, name)
    if not (q.shape == k.shape == v.shape) or q.dtype != k.dtype or q.dtype != v.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    if q.dim() == 3:
        B, N, d = q.shape
        H = 1
    elif q.dim() == 4:
        B, H, N, d = q.shape
    else:
        raise ValueError("expected [B, H, N, d] or [B, N, d]")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_tensor(out, "out")
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out must match q")
    lse_ptr = None
    if return_lse:
        if lse is None:
            lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
        elif lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
            raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
        lse_ptr = lse.data_ptr()
    else:
        lse = None
    dev = same_device([("q", q), ("k", k), ("v", v), ("out", out)] +
                      ([("lse", lse)] if lse is not None else []))
    left, right = _window(window_size)
    slopes, slopes_ptr = _slopes(alibi_slopes, H, dev)
    with _on(dev):
        rc = load().fa_fwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse_ptr, B, H, N, d, 0.0 if scale is None else float(scale),
                               int(bool(causal)), left, right, slopes_ptr, _DT[q.dtype],
                               _stream_ptr(q))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_ext")
    return out, lse


def fwd_qkvpacked(qkv: torch.Tensor, dropout_p: float = 0.0, softmax_scale: float | None = None,
                  causal: bool = False, out: torch.Tensor | None = None,
                  return_lse: bool = True, window_size=(-1, -1), alibi_slopes=None):
    """Packed forward: ``qkv`` is ``[B, N, 3, H, d]``; returns ``(O [B, N, H, d], LSE [B, H, N])``.

    ``window_size`` and ``alibi_slopes`` as :func:`fwd`."""
    _check_tensor(qkv, "qkv")
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must be [B, N, 3, H, d]")
    B, N, _, H, d = qkv.shape
    if out is None:
        out = torch.empty((B, N, H, d), device=qkv.device, dtype=qkv.dtype)
    else:
        _check_tensor(out, "out")
    if out.shape != (B, N, H, d) or out.dtype != qkv.dtype:
        raise ValueError("out must be [B, N, H, d] in qkv's dtype")
    lse = torch.empty((B, H, N), device=qkv.device, dtype=torch.float32) if return_lse else None
    dev = same_device([("qkv", qkv), ("out", out)])
    left, right = _window(window_size)
    slopes, slopes_ptr = _slopes(alibi_slopes, H, dev)
    with _on(dev):
        rc = load().fa_fwd_qkvpacked_ext(
            qkv.data_ptr(), out.data_ptr(), None if lse is None else lse.data_ptr(), B, N, H, d,
            0.0 if softmax_scale is None else float(softmax_scale), int(bool(causal)),
            float(dropout_p), left, right, slopes_ptr, _DT[qkv.dtype], _stream_ptr(qkv))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_qkvpacked_ext")
    return out, lse


def fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, descale_q: float,
            descale_k: float, descale_v: float, scale: float | None = None,
            causal: bool = False, return_lse: bool = True):
    """Forward on fp8 e4m3 ``[B, H, N, d]`` tensors (torch.float8_e4m3fn, or
    uint8 holding the codes) with per-tensor dequantisation factors: the real
    operands are ``descale_x * x``.  Returns ``(O bf16 [B, H, N, d], LSE)``."""
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float8_e4m3fn (or uint8) tensor")
    if not (q8.shape == k8.shape == v8.shape) or q8.dim() != 4:
        raise ValueError("q8, k8, v8 must share one [B, H, N, d] shape")
    B, H, N, d = q8.shape
    dev = same_device([("q8", q8), ("k8", k8), ("v8", v8)])
    out = torch.empty((B, H, N, d), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32) if return_lse else None
    with _on(dev):
        rc = load().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                               None if lse is None else lse.data_ptr(), B, H, N, d,
                               0.0 if scale is None else float(scale), float(descale_q),
                               float(descale_k), float(descale_v), int(bool(causal)),
                               _stream_ptr(q8))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8")
    return out, lse


def fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
               max_seqlen: int, scale: float | None = None, causal: bool = False,
               window_size=(-1, -1), alibi_slopes=None, return_lse: bool = True):
    """Forward over sequences packed back to back: ``q, k, v`` are
    ``[total, H, d]``, sequence b holds rows ``cu_seqlens[b] .. cu_seqlens[b+1]-1``
    (``cu_seqlens``: int32 ``[batch + 1]`` on the same device).  Returns
    ``(O [total, H, d], LSE [H, total])``.  Masks as :func:`fwd`, per sequence."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(t, name)
    if not (q.shape == k.shape == v.shape) or q.dim() != 3 or len({q.dtype, k.dtype, v.dtype}) != 1:
        raise ValueError("q, k, v must share one [total, H, d] shape and dtype")
    if (not isinstance(cu_seqlens, torch.Tensor) or cu_seqlens.dtype != torch.int32
            or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2 or not cu_seqlens.is_contiguous()):
        raise ValueError("cu_seqlens must be a contiguous int32 tensor of batch + 1 offsets")
    total, H, d = q.shape
    batch = cu_seqlens.numel() - 1
    dev = same_device([("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens)])
    out = torch.empty_like(q)
    lse = torch.empty((H, total), device=dev, dtype=torch.float32) if return_lse else None
    left, right = _window(window_size)
    slopes, slopes_ptr = _slopes(alibi_slopes, H, dev)
    with _on(dev):
        rc = load().fa_fwd_varlen(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
            None if lse is None else lse.data_ptr(), cu_seqlens.data_ptr(), batch,
            int(max_seqlen), total, H, d, 0.0 if scale is None else float(scale),
            int(bool(causal)), left, right, slopes_ptr, _DT[q.dtype], _stream_ptr(q))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_varlen")
    return out, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
        dout: torch.Tensor, scale: float | None = None, causal: bool = False):
    """Gradient of :func:`fwd`: returns ``(dQ, dK, dV)`` for an upstream ``dout``.

    ``o`` and ``lse`` are the outputs of :func:`fwd` on the same ``q, k, v``,
    ``scale`` and ``causal``; all tensors ``[B, H, N, d]`` (``lse`` ``[B, H, N]``
    fp32).  The fp32 row-statistic workspace is allocated here.
    """
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(t, name)
    if not (q.shape == k.shape == v.shape == o.shape == dout.shape) or q.dim() != 4:
        raise ValueError("q, k, v, o, dout must share one [B, H, N, d] shape")
    if len({t.dtype for t in (q, k, v, o, dout)}) != 1:
        raise ValueError("q, k, v, o, dout must share one dtype")
    B, H, N, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dev = same_device([("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("dout", dout)])
    work = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    with _on(dev):
        rc = load().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           work.data_ptr(), B, H, N, d, 0.0 if scale is None else float(scale),
                           int(bool(causal)), _DT[q.dtype], _stream_ptr(q))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                lse: torch.Tensor, dout: torch.Tensor, scale: float | None = None,
                causal: bool = False):
    """:func:`bwd` through ``fa_bwd_noalloc``: the row statistic lives in the
    library's own device array instead of a workspace tensor."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(t, name)
    if not (q.shape == k.shape == v.shape == o.shape == dout.shape) or q.dim() != 4:
        raise ValueError("q, k, v, o, dout must share one [B, H, N, d] shape")
    if len({t.dtype for t in (q, k, v, o, dout)}) != 1:
        raise ValueError("q, k, v, o, dout must share one dtype")
    B, H, N, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dev = same_device([("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("dout", dout)])
    with _on(dev):
        rc = load().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, H, N, d,
                                   0.0 if scale is None else float(scale), int(bool(causal)),
                                   _DT[q.dtype], _stream_ptr(q))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_noalloc")
    return dq, dk, dv


def device_status(clear: bool = True):
    """(status, detail) of the current device's watchdog word; synchronises."""
    detail = ctypes.c_uint(0)
    rc = load().fa_device_status(int(bool(clear)), ctypes.byref(detail))
    return int(rc), int(detail.value)


def watchdog_selftest(limit_ns: int = 20_000_000):
    """Run the bounded-wait self test kernel on the current stream."""
    rc = load().fa_debug_watchdog_selftest(int(limit_ns),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_debug_watchdog_selftest")


def set_wait_limit(limit_ns: int = 0):
    """Bound (ns) of every mbarrier wait in the kernels launched next; 0
    restores the default.  A debug hook for testing the kernels' give-up path."""
    rc = load().fa_debug_set_wait_limit(int(limit_ns))
    if rc != FA_OK:
        raise FaError(rc, "fa_debug_set_wait_limit")


def exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """The kernel's software exp2 applied to a float32 CUDA tensor (test hook)."""
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    rc = load().fa_debug_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), _stream_ptr(x))
    if rc != FA_OK:
        raise FaError(rc, "fa_debug_exp2_poly")
    return y


def launch_ctas(B: int, H: int, N: int, d: int, causal: bool = False) -> int:
    return int(load().fa_launch_ctas(B, H, N, d, int(bool(causal))))


def default_scale(d: int) -> float:
    """The fp32 scale the library uses when none is given: 1/sqrt(d) rounded to fp32."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
