"""Tiled online-softmax recurrence in NumPy fp64 (second, independent oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Restates ``flash_attention_forward`` of "flash_attention.py"
(forceinjection.github.io): an outer loop over query blocks of ``Br`` rows and
an inner loop over key/value blocks of ``Bc`` rows, keeping per row a running
max ``m``, a running sum ``l`` and an unnormalised output ``O``.  For every key
block the page's five steps are, in order:

1. ``m_new = max(m, rowmax(S_ij))``
2. ``P_ij = exp(S_ij - m_new)``
3. ``correction = exp(m - m_new)``
4. ``l = correction * l + rowsum(P_ij)`` and ``O = correction * O + P_ij V_j``
5. ``m = m_new``

and the block's result is ``O / l``.  Ragged tails are handled by clipping the
block end at ``N``, as the page does with ``min``.

Two extensions the page does not print, kept as small as possible:

* the causal mask -- key ``j`` is visible from query ``i`` iff ``j <= i``; the
  masked scores are ``-inf`` (the ``masked_fill`` hook of the standard attention
  on the aiknowledge.cn page, section 1.1);
* the natural-log logsumexp ``LSE = m + ln(l)`` of the scaled scores.

Unlike the page, the state stays in fp64 (the page keeps it in the input dtype).
A row that has seen only masked keys keeps ``m = -inf``; its ``P`` and
``correction`` are then taken as 0 instead of ``exp(nan)``.
"""
from __future__ import annotations

import math

import numpy as np


def flash_forward(q, k, v, scale: float | None = None, causal: bool = False,
                  Br: int = 64, Bc: int = 64):
    """``q, k, v``: ``[N, d]`` or ``[..., N, d]`` fp64 arrays.  Returns (O, LSE)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim > 2:
        lead = q.shape[:-2]
        qs = q.reshape((-1,) + q.shape[-2:])
        ks = k.reshape((-1,) + k.shape[-2:])
        vs = v.reshape((-1,) + v.shape[-2:])
        outs = [flash_forward(a, b, c, scale, causal, Br, Bc) for a, b, c in zip(qs, ks, vs)]
        O = np.stack([o for o, _ in outs]).reshape(lead + q.shape[-2:])
        L = np.stack([l for _, l in outs]).reshape(lead + q.shape[-2:-1])
        return O, L

    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Tr = (N + Br - 1) // Br
    Tc = (N + Bc - 1) // Bc
    O = np.zeros((N, d))
    LSE = np.zeros(N)
    for i in range(Tr):
        q0, q1 = i * Br, min(i * Br + Br, N)
        Qi = q[q0:q1]
        mi = np.full(q1 - q0, -np.inf)
        li = np.zeros(q1 - q0)
        Oi = np.zeros((q1 - q0, d))
        for j in range(Tc):
            k0, k1 = j * Bc, min(j * Bc + Bc, N)
            Sij = (Qi @ k[k0:k1].T) * scale
            if causal:
                rows = np.arange(q0, q1)[:, None]
                cols = np.arange(k0, k1)[None, :]
                Sij = np.where(cols <= rows, Sij, -np.inf)
            m_new = np.maximum(mi, Sij.max(axis=1))
            ref = np.where(np.isfinite(m_new), m_new, 0.0)
            Pij = np.exp(Sij - ref[:, None])
            correction = np.where(np.isfinite(mi), np.exp(mi - ref), 0.0)
            li = correction * li + Pij.sum(axis=1)
            Oi = correction[:, None] * Oi + Pij @ v[k0:k1]
            mi = m_new
        O[q0:q1] = Oi / li[:, None]
        LSE[q0:q1] = mi + np.log(li)
    return O, LSE
