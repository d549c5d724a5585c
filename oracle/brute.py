"""Scalar pure-Python attention with ``math.fsum`` (third oracle, tiny inputs).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The definition of "2.3 FlashAttention与IO感知注意力(1)" (aiknowledge.cn),
section 1.1, evaluated one scalar at a time with correctly rounded sums
(``math.fsum``) and without subtracting the row max, so that it shares no
evaluation order with the C oracle.  Meant for N <= 8 and small d, where
``exp`` of the raw scores cannot overflow.
"""
from __future__ import annotations

import math


def attention_fsum(q, k, v, scale=None, causal=False):
    """``q, k, v``: nested lists (or arrays) ``[N][d]``.  Returns (O, LSE) lists."""
    N = len(q)
    d = len(q[0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O, LSE = [], []
    for i in range(N):
        nvis = i + 1 if causal else N
        s = [scale * math.fsum(float(q[i][c]) * float(k[j][c]) for c in range(d))
             for j in range(nvis)]
        e = [math.exp(x) for x in s]
        z = math.fsum(e)
        O.append([math.fsum(e[j] * float(v[j][c]) for j in range(nvis)) / z
                  for c in range(d)])
        LSE.append(math.log(z))
    return O, LSE


def attention_fsum_masked(q, k, v, scale=None, causal=False, window=(-1, -1), slope=0.0):
    """:func:`attention_fsum` with a local window ``(left, right)`` (-1 =
    unbounded) and an ALiBi bias ``-slope * |i - j|`` on the scaled scores,
    one scalar at a time with ``math.fsum``.  Returns (O, LSE) lists."""
    N = len(q)
    d = len(q[0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    left, right = window
    O, LSE = [], []
    for i in range(N):
        vis = [j for j in range(N)
               if (left < 0 or j >= i - left) and (right < 0 or j <= i + right)
               and (not causal or j <= i)]
        s = [scale * math.fsum(float(q[i][c]) * float(k[j][c]) for c in range(d))
             - slope * abs(i - j) for j in vis]
        e = [math.exp(x) for x in s]
        z = math.fsum(e)
        O.append([math.fsum(e[n] * float(v[j][c]) for n, j in enumerate(vis)) / z
                  for c in range(d)])
        LSE.append(math.log(z))
    return O, LSE
