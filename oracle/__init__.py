"""fp64 CPU oracle for the exact attention forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  Nothing in the product
package imports this module, and this module imports nothing from it.

Three independent implementations live here:

* :func:`attention` -- the plain definition (scores, row max, exp, sum, P V,
  logsumexp) in C with OpenMP over rows, fp64 throughout
  (``fa_oracle.c``).  Follows the standard attention of
  "2.3 FlashAttention与IO感知注意力(1)" (aiknowledge.cn), section 1.1, and the
  ``standard_attention`` function of "flash_attention.py"
  (forceinjection.github.io).
* :func:`oracle.tiled.flash_forward` -- the tiled online-softmax recurrence of
  ``flash_attention_forward`` in the same file, restated in NumPy fp64 and
  extended with the causal mask and the logsumexp output.
* :func:`oracle.brute.attention_fsum` -- a scalar pure-Python version using
  ``math.fsum`` for tiny inputs.
* :func:`attention_masked` -- the definition with a local window and an
  ALiBi bias (the two masks the packed call names), pinned in
  ``tests/test_oracle_mask_pins.py``.
* :func:`attention_varlen` -- sequences of different lengths packed back to
  back (``[total, H, d]`` with ``cu_seqlens`` offsets): the definition applied
  to each sequence on its own, pinned in ``tests/test_oracle_varlen_pins.py``.
* :func:`decode_e4m3` and :func:`attention_fp8` -- fp8 (e4m3) operands with
  per-tensor dequantisation factors: the codes decoded by the format's
  definition, then the plain definition on the dequantised values; pinned in
  ``tests/test_oracle_fp8_pins.py``.
* :func:`attention_bwd` -- the gradient of the plain definition with respect
  to q, k, v (chain rule written out in ``fa_oracle.c``), pinned in
  ``tests/test_oracle_bwd_pins.py`` by central finite differences of
  :func:`attention`, closed forms and invariants.

Parity status: every function here is pinned by tests in
``tests/test_oracle_pins.py``, ``tests/test_oracle_mask_pins.py``,
``tests/test_oracle_varlen_pins.py``, ``tests/test_oracle_fp8_pins.py`` and
``tests/test_oracle_bwd_pins.py`` (closed
forms, invariants, brute force, finite differences and the
recurrence-equals-definition check); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libfa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``fa_oracle.c`` into ``libfa_oracle.so`` next to it (gcc, OpenMP).

    Plain ``-O2`` with no fast-math flags, so every operation is IEEE fp64.
    """
    if not force and os.path.exists(_LIB_PATH) and (
        os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)
    ):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int)
            lib.oracle_attention_fwd.argtypes = [
                dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int, ip, ctypes.c_int]
            lib.oracle_attention_fwd.restype = ctypes.c_int
            lib.oracle_attention_probs.argtypes = [
                dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                ctypes.c_int, dp]
            lib.oracle_attention_probs.restype = ctypes.c_int
            lib.oracle_attention_fwd_masked.argtypes = [
                dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                dp, ip, ctypes.c_int]
            lib.oracle_attention_fwd_masked.restype = ctypes.c_int
            lib.oracle_attention_bwd.argtypes = [
                dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, ctypes.c_int]
            lib.oracle_attention_bwd.restype = ctypes.c_int
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _as_f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor (CPU); widening fp16/bf16 is exact
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    """OpenMP threads the oracle runs with (``OMP_NUM_THREADS`` or all cores)."""
    return int(_load().oracle_num_threads())


def attention(q, k, v, scale: float | None = None, causal: bool = False,
              rows=None):
    """Exact attention forward in fp64.

    ``q, k, v``: ``[B, H, N, d]`` (or ``[N, d]`` / ``[B, N, d]``, treated as
    H=1 / B=1) arrays or CPU tensors.  ``scale=None`` means ``1/sqrt(d)``.
    ``rows``: optional sequence of query indices; the result then holds only
    those rows, in that order, for every (b, h).

    Returns ``(O, LSE)`` with ``O`` shaped like ``q`` restricted to ``rows`` and
    ``LSE`` shaped ``q.shape[:-1]`` restricted likewise (natural log).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    if q.ndim == 2:
        B, H = 1, 1
    elif q.ndim == 3:
        B, H = q.shape[0], 1
    elif q.ndim == 4:
        B, H = q.shape[0], q.shape[1]
    else:
        raise ValueError("expected 2-D, 3-D or 4-D inputs")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows_arr = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(
        np.asarray(rows, dtype=np.int32))
    nr = int(rows_arr.size)
    o = np.empty((B, H, nr, d), dtype=np.float64)
    lse = np.empty((B, H, nr), dtype=np.float64)
    rc = _load().oracle_attention_fwd(
        _dptr(q), _dptr(k), _dptr(v), _dptr(o), _dptr(lse), B, H, N, d,
        float(scale), int(bool(causal)),
        rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), nr)
    if rc != 0:
        raise ValueError(f"oracle_attention_fwd failed ({rc})")
    return o.reshape(lead + (nr, d)), lse.reshape(lead + (nr,))


def attention_masked(q, k, v, scale: float | None = None, causal: bool = False,
                     window=(-1, -1), alibi_slopes=None, rows=None):
    """:func:`attention` with a local window and an ALiBi bias
    (``oracle_attention_fwd_masked`` in ``fa_oracle.c``).

    ``window = (left, right)``: key j is visible from query i iff
    ``i - left <= j <= i + right`` (-1 = unbounded on that side), intersected
    with the causal mask.  ``alibi_slopes``: one slope per head (``[H]``) or
    None; the scaled score gets ``- slope[h] * |i - j|``.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    if q.ndim == 2:
        B, H = 1, 1
    elif q.ndim == 3:
        B, H = q.shape[0], 1
    elif q.ndim == 4:
        B, H = q.shape[0], q.shape[1]
    else:
        raise ValueError("expected 2-D, 3-D or 4-D inputs")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    left, right = (int(window[0]), int(window[1]))
    if left < -1 or right < -1:
        raise ValueError("window sides must be >= -1")
    slopes = None
    if alibi_slopes is not None:
        slopes = np.ascontiguousarray(np.asarray(alibi_slopes, dtype=np.float64).reshape(-1))
        if slopes.size != H:
            raise ValueError("alibi_slopes needs one slope per head")
    rows_arr = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(
        np.asarray(rows, dtype=np.int32))
    nr = int(rows_arr.size)
    o = np.empty((B, H, nr, d), dtype=np.float64)
    lse = np.empty((B, H, nr), dtype=np.float64)
    rc = _load().oracle_attention_fwd_masked(
        _dptr(q), _dptr(k), _dptr(v), _dptr(o), _dptr(lse), B, H, N, d, float(scale),
        int(bool(causal)), left, right, None if slopes is None else _dptr(slopes),
        rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), nr)
    if rc != 0:
        raise ValueError(f"oracle_attention_fwd_masked failed ({rc})")
    return o.reshape(lead + (nr, d)), lse.reshape(lead + (nr,))


def attention_varlen(q, k, v, cu_seqlens, scale: float | None = None, causal: bool = False,
                     window=(-1, -1), alibi_slopes=None):
    """Attention over sequences packed back to back, in fp64.

    ``q, k, v``: ``[total, H, d]``; sequence b is rows ``cu_seqlens[b]`` to
    ``cu_seqlens[b+1] - 1`` and attends only to itself, with positions counted
    from its first row (the dynamic sequence lengths of item 3, "动态形状优化",
    of "flash-attention与TensorRT 10集成", blog.gitcode.com, read as independent
    self-attention problems of their own lengths).  Each sequence is handed to
    :func:`attention_masked` as one ``[1, H, L, d]`` problem.

    Returns ``(O [total, H, d], LSE [H, total])``; rows outside every sequence
    are NaN.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if not (q.shape == k.shape == v.shape) or q.ndim != 3:
        raise ValueError("q, k, v must share one [total, H, d] shape")
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    total, H, d = q.shape
    if len(cu) < 2 or cu[0] < 0 or cu[-1] > total or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must be nondecreasing offsets within [0, total]")
    O = np.full((total, H, d), np.nan)
    LSE = np.full((H, total), np.nan)
    for s0, s1 in zip(cu, cu[1:]):
        if s1 == s0:
            continue
        seq = [np.ascontiguousarray(t[s0:s1].transpose(1, 0, 2))[None] for t in (q, k, v)]
        o, lse = attention_masked(*seq, scale=scale, causal=causal, window=window,
                                  alibi_slopes=alibi_slopes)
        O[s0:s1] = o[0].transpose(1, 0, 2)
        LSE[:, s0:s1] = lse[0]
    return O, LSE


def decode_e4m3(codes) -> np.ndarray:
    """fp64 values of fp8 e4m3 codes (uint8), from the format's definition:
    bit 7 the sign, bits 6-3 the exponent e (bias 7), bits 2-0 the mantissa m;
    e = 0 gives the subnormals m/8 * 2^-6, otherwise (1 + m/8) * 2^(e-7); the
    one code with e = 15 and m = 7 (per sign) is NaN, and there is no
    infinity (the "E4M3FN" variant, largest finite value 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 7 == 7), np.nan, mag)
    return sign * mag


def attention_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
                  scale: float | None = None, causal: bool = False, rows=None):
    """Attention on fp8 operands in fp64: the real tensors are
    ``descale_x * decode_e4m3(x8)``, and the result is :func:`attention` of
    those (the FP8 inference of item 4, "低精度推理支持", of
    "flash-attention与TensorRT 10集成", blog.gitcode.com, read as e4m3 codes
    with one dequantisation factor per tensor).  ``q8, k8, v8``: uint8 codes
    ``[B, H, N, d]`` (or a torch float8_e4m3fn / uint8 tensor)."""
    def codes(x):
        if hasattr(x, "detach"):
            x = x.detach().cpu()
            if x.dtype != __import__("torch").uint8:
                x = x.view(__import__("torch").uint8)
            x = x.numpy()
        return np.asarray(x, dtype=np.uint8)
    q = float(descale_q) * decode_e4m3(codes(q8))
    k = float(descale_k) * decode_e4m3(codes(k8))
    v = float(descale_v) * decode_e4m3(codes(v8))
    return attention(q, k, v, scale=scale, causal=causal, rows=rows)


def attention_bwd(q, k, v, dout, scale: float | None = None, causal: bool = False):
    """Gradient of :func:`attention`'s O with respect to q, k, v in fp64.

    ``dout`` is the upstream gradient of O, shaped like ``q``.  Returns
    ``(dQ, dK, dV)`` shaped like the inputs.  The chain rule through the same
    plain definition (``oracle_attention_bwd`` in ``fa_oracle.c``).
    """
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    if not (q.shape == k.shape == v.shape == dout.shape):
        raise ValueError("q, k, v, dout must have the same shape")
    shape = q.shape
    N, d = shape[-2], shape[-1]
    if q.ndim < 2 or q.ndim > 4:
        raise ValueError("expected 2-D, 3-D or 4-D inputs")
    heads = int(np.prod(shape[:-2])) if q.ndim > 2 else 1
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq, dk, dv = (np.empty(shape, dtype=np.float64) for _ in range(3))
    rc = _load().oracle_attention_bwd(
        _dptr(q), _dptr(k), _dptr(v), _dptr(dout), _dptr(dq), _dptr(dk), _dptr(dv),
        1, heads, N, d, float(scale), int(bool(causal)))
    if rc != 0:
        raise ValueError(f"oracle_attention_bwd failed ({rc})")
    return dq, dk, dv


def probs(q, k, i: int, scale: float | None = None, causal: bool = False):
    """Normalised attention weights of query row ``i`` for one ``[N, d]`` slice."""
    q, k = _as_f64(q), _as_f64(k)
    N, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    p = np.empty(N, dtype=np.float64)
    rc = _load().oracle_attention_probs(_dptr(q), _dptr(k), N, d, float(scale),
                                        int(bool(causal)), int(i), _dptr(p))
    if rc != 0:
        raise ValueError(f"oracle_attention_probs failed ({rc})")
    return p
