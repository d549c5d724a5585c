"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only draws the inputs (and the
sampled query rows used to check large shapes), so that the CUDA path and the
CPU oracle see exactly the same values.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws
``randn`` in fp32, the values are multiplied by the workload's standard
deviation and rounded once to the compute dtype.  The oracle widens those
rounded values to fp64, so both sides start from identical numbers.

The workloads follow the shapes the pages use: the single-head ``[B, N, d]``
layout of ``flash_attention_forward`` in "flash_attention.py"
(forceinjection.github.io); the packed ``qkv`` call of section 5.2 of
"Windows下RTX 3090编译Flash Attention 2.8.3全指南" (intelliparadigm.com); the
GPT-3-like head count of section 1.2 of "2.3 FlashAttention与IO感知注意力(1)"
(aiknowledge.cn); the sequence-length list of the A100 table of
"flash-attention与TensorRT 10集成" (blog.gitcode.com); and head dim 256, the
largest that page lists.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

FP16, BF16, E4M3 = 0, 1, 2
TORCH_DTYPE = {FP16: torch.float16, BF16: torch.bfloat16, E4M3: torch.float8_e4m3fn}
DTYPE_NAME = {FP16: "f16", BF16: "bf16", E4M3: "e4m3"}


@dataclass(frozen=True)
class Workload:
    """One attention forward problem.

    ``layout`` is ``"bhnd"`` (separate q, k, v of shape [B, H, N, d]),
    ``"packed"`` (one qkv of shape [B, N, 3, H, d]) or ``"varlen"``
    (``lengths`` sequences packed back to back as [total, H, d]; B is the
    number of sequences and N the longest length).  ``window`` is the local
    window (left, right), -1 = unbounded; ``alibi`` adds the usual per-head
    ALiBi slopes (:func:`alibi_slopes`).
    """
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: int
    causal: bool
    seed: int
    layout: str = "bhnd"
    sigma_qk: float = 1.0
    sigma_v: float = 1.0
    extra: dict = field(default_factory=dict, compare=False)
    window: tuple = (-1, -1)
    alibi: bool = False
    lengths: tuple = ()

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def masked(self) -> bool:
        return self.window != (-1, -1) or self.alibi or self.layout == "varlen"

    @property
    def flops(self) -> float:
        """4*B*H*N^2*d, halved for the causal mask; with a local window or
        variable lengths, 4*d*H per (query, visible key) pair, counted exactly."""
        if not self.masked or (self.window == (-1, -1) and self.layout != "varlen"):
            f = 4.0 * self.B * self.H * self.N * self.N * self.d
            return f / 2 if self.causal else f
        lengths = self.lengths if self.layout == "varlen" else (self.N,) * self.B
        return 4.0 * self.d * self.H * sum(visible_pairs(n, self.causal, self.window)
                                           for n in lengths)

    def describe(self) -> dict:
        out = {"workload": self.name, "B": self.B, "H": self.H, "N": self.N,
               "d": self.d, "dtype": DTYPE_NAME[self.dtype],
               "causal": self.causal, "layout": self.layout, "seed": self.seed}
        if self.window != (-1, -1):
            out["window"] = list(self.window)
        if self.alibi:
            out["alibi"] = "2^(-8(h+1)/H)"
        if self.layout == "varlen":
            out["total_tokens"] = int(sum(self.lengths))
        return out


def visible_pairs(n: int, causal: bool, window=(-1, -1)) -> int:
    """Number of (query, key) pairs with key j visible from query i in a
    sequence of n tokens: i - left <= j <= i + right (-1 unbounded), j <= i
    when causal."""
    left, right = window
    if causal:
        right = 0
    i = np.arange(n, dtype=np.int64)
    lo = np.zeros(n, np.int64) if left < 0 else np.maximum(i - left, 0)
    hi = np.full(n, n - 1, np.int64) if right < 0 else np.minimum(i + right, n - 1)
    return int((hi - lo + 1).sum())


def single_head_n256() -> Workload:
    return Workload("single-head fwd [1,256,64] fp16 non-causal", 1, 1, 256, 64,
                    FP16, False, 42)


def packed_qkv_b2_n256_h12() -> Workload:
    return Workload("packed-qkv fwd [2,256,3,12,64] fp16 non-causal", 2, 12, 256, 64,
                    FP16, False, 43, layout="packed")


def many_heads_causal_n2048() -> Workload:
    return Workload("causal fwd [1,128,2048,128] bf16", 1, 128, 2048, 128, BF16,
                    True, 44)


SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)


def seqlen_sweep(N: int, causal: bool) -> Workload:
    if N not in SWEEP_N:
        raise ValueError(f"N must be one of {SWEEP_N}")
    seed = 45 + int(round(math.log2(N // 512)))
    tag = "causal" if causal else "non-causal"
    return Workload(f"seqlen sweep fwd B={16384 // N},H=16,N={N},d=128 bf16 {tag}",
                    16384 // N, 16, N, 128, BF16, causal, seed)


def headdim256_causal() -> Workload:
    return Workload("head-dim 256 causal fwd [1,8,8192,256] bf16, q,k ~ N(0,3^2)",
                    1, 8, 8192, 256, BF16, True, 50, sigma_qk=3.0)


def window_causal_n4096() -> Workload:
    """The N = 4096 sweep shape with a causal sliding window of 256 keys."""
    return Workload("sliding-window causal fwd B=4,H=16,N=4096,d=128 bf16, window (256, 0)",
                    4, 16, 4096, 128, BF16, True, 60, window=(256, 0))


def alibi_causal_n4096() -> Workload:
    """The N = 4096 sweep shape, causal, with per-head ALiBi slopes."""
    return Workload("ALiBi causal fwd B=4,H=16,N=4096,d=128 bf16", 4, 16, 4096, 128, BF16,
                    True, 61, alibi=True)


def varlen_lengths(seed: int, total: int, lo: int, hi: int) -> tuple:
    """Seeded sequence lengths, uniform in [lo, hi], until ``total`` tokens
    (the last one trimmed)."""
    rng = np.random.default_rng(seed)
    out, acc = [], 0
    while acc < total:
        n = int(min(rng.integers(lo, hi + 1), total - acc))
        out.append(n)
        acc += n
    return tuple(out)


def varlen_mix_causal() -> Workload:
    """Sequences of 128..8192 tokens (seeded, uniform) packed to 65536 tokens,
    H=16, d=128, bf16, causal: a dynamic-length batch of the size of the
    N = 4096 sweep point times four."""
    lengths = varlen_lengths(62, 65536, 128, 8192)
    return Workload(f"varlen causal fwd {len(lengths)} sequences of 128..8192 tokens "
                    f"(65536 total), H=16, d=128 bf16", len(lengths), 16, max(lengths), 128,
                    BF16, True, 62, layout="varlen", lengths=lengths)


def fp8_sweep_n4096(causal: bool = False) -> Workload:
    """The N = 4096 sweep shape on fp8 e4m3 operands (per-tensor factors)."""
    tag = "causal" if causal else "non-causal"
    return Workload(f"fp8 e4m3 fwd B=4,H=16,N=4096,d=128 {tag}, bf16 output", 4, 16, 4096, 128,
                    E4M3, causal, 63 + int(causal))


def all_workloads() -> list[Workload]:
    w = [single_head_n256(), packed_qkv_b2_n256_h12(), many_heads_causal_n2048()]
    for n in SWEEP_N:
        for c in (False, True):
            w.append(seqlen_sweep(n, c))
    w.append(headdim256_causal())
    return w


def make_inputs(w: Workload):
    """CPU tensors in the compute dtype.

    ``bhnd`` -> ``(q, k, v)`` each [B, H, N, d]; ``packed`` -> ``(qkv,)`` of
    shape [B, N, 3, H, d] (index 0/1/2 of axis 2 = q/k/v); ``varlen`` ->
    ``(q, k, v, cu_seqlens)`` with q, k, v [total, H, d]; e4m3 workloads
    ``(q8, k8, v8)`` (their factors: :func:`fp8_factors`).
    """
    if w.dtype == E4M3:
        return fp8_inputs(w.B, w.H, w.N, w.d, w.seed, w.sigma_qk, w.sigma_v)[0]
    g = torch.Generator().manual_seed(w.seed)
    dt = TORCH_DTYPE[w.dtype]
    if w.layout == "varlen":
        q, k, v, cu = packed_lengths(w.lengths, w.H, w.d, w.dtype, w.seed, w.sigma_qk, w.sigma_v)
        return q, k, v, cu
    if w.layout == "packed":
        qkv = torch.randn((w.B, w.N, 3, w.H, w.d), generator=g, dtype=torch.float32)
        qkv[:, :, 0:2] *= w.sigma_qk
        qkv[:, :, 2] *= w.sigma_v
        return (qkv.to(dt),)
    shape = (w.B, w.H, w.N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32) * w.sigma_qk
    k = torch.randn(shape, generator=g, dtype=torch.float32) * w.sigma_qk
    v = torch.randn(shape, generator=g, dtype=torch.float32) * w.sigma_v
    return q.to(dt), k.to(dt), v.to(dt)


def unpack_qkv(qkv: torch.Tensor):
    """[B, N, 3, H, d] -> three [B, H, N, d] tensors (a pure re-indexing)."""
    return tuple(qkv[:, :, i].permute(0, 2, 1, 3).contiguous() for i in range(3))


def sample_rows(N: int, seed: int, count: int = 512) -> np.ndarray:
    """Sorted query rows to check at large N: ``count`` distinct rows drawn with
    ``numpy.random.default_rng(seed + 1000)``, always including 0, 127, 128 and
    N-1 (when they exist).  Every row is independent of the others given K and
    V, so a sample checks the rows it names exactly."""
    must = {r for r in (0, 127, 128, N - 1) if 0 <= r < N}
    if N <= count:
        return np.arange(N, dtype=np.int32)
    rng = np.random.default_rng(seed + 1000)
    pick = rng.choice(N, size=count, replace=False)
    return np.array(sorted(must.union(int(x) for x in pick)), dtype=np.int32)


def alibi_slopes(H: int) -> torch.Tensor:
    """The usual ALiBi slopes for H heads, 2^(-8 (h + 1) / H), as an fp32 [H]
    tensor (an input like q, k, v; the pages give the keyword, not values)."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


def packed_lengths(lengths, H, d, dtype, seed, sigma_qk=1.0, sigma_v=1.0, extra_rows=0):
    """Sequences of the given lengths packed back to back: ``(q, k, v)`` each
    ``[total, H, d]`` (same recipe as :func:`make_inputs`), plus the int32
    offsets ``cu_seqlens`` ``[len(lengths) + 1]``.  ``extra_rows`` trailing rows
    belong to no sequence."""
    total = int(sum(lengths)) + extra_rows
    g = torch.Generator().manual_seed(seed)
    dt = TORCH_DTYPE[dtype]
    q = torch.randn((total, H, d), generator=g, dtype=torch.float32) * sigma_qk
    k = torch.randn((total, H, d), generator=g, dtype=torch.float32) * sigma_qk
    v = torch.randn((total, H, d), generator=g, dtype=torch.float32) * sigma_v
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return q.to(dt), k.to(dt), v.to(dt), cu


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor fp8 quantisation of an fp32 tensor: descale = amax / 448
    rounded to fp32, codes = round-to-nearest e4m3 of x / descale (torch's
    float8_e4m3fn conversion).  Returns (codes as float8_e4m3fn, descale)."""
    amax = float(x.abs().max())
    descale = float(torch.tensor(max(amax, 1e-30) / 448.0, dtype=torch.float32))
    return (x / descale).to(torch.float8_e4m3fn), descale


def fp8_factors(w: Workload):
    """The (descale_q, descale_k, descale_v) of an e4m3 workload's inputs."""
    return fp8_inputs(w.B, w.H, w.N, w.d, w.seed, w.sigma_qk, w.sigma_v)[1]


def fp8_inputs(B, H, N, d, seed, sigma_qk=1.0, sigma_v=1.0):
    """[B, H, N, d] fp8 q, k, v and their descale factors: the draws of
    :func:`make_inputs` (fp32 randn times sigma), each quantised per tensor by
    :func:`quantize_e4m3`.  Returns ``((q8, k8, v8), (dq, dk, dv))``."""
    g = torch.Generator().manual_seed(seed)
    shape = (B, H, N, d)
    xs = [torch.randn(shape, generator=g, dtype=torch.float32) * s
          for s in (sigma_qk, sigma_qk, sigma_v)]
    out = [quantize_e4m3(x) for x in xs]
    return tuple(c for c, _ in out), tuple(f for _, f in out)


def random_inputs(B, H, N, d, dtype, seed, sigma_qk=1.0, sigma_v=1.0):
    """[B, H, N, d] q, k, v for ad-hoc test shapes (same recipe)."""
    w = Workload("adhoc", B, H, N, d, dtype, False, seed, sigma_qk=sigma_qk,
                 sigma_v=sigma_v)
    return make_inputs(w)
