"""Pins of the variable-length oracle (``oracle.attention_varlen``) to facts
that do not come from the oracle itself.

* Brute force: each sequence, evaluated one scalar at a time with
  ``math.fsum`` on its own rows, with masks and ALiBi.
* Closed forms: a one-token sequence returns its own value row, with LSE the
  scaled self-score; all-equal keys inside a sequence give the (causal:
  running) mean of that sequence's values only.
* Independence: changing the tokens of one sequence leaves every other
  sequence's rows bit for bit unchanged; equal lengths reproduce the
  fixed-length [B, H, N, d] problem after a transposition.

``test_planted_mistakes_are_caught`` checks that an off-by-one sequence
boundary and a transposed LSE layout each break a pin.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import brute


def _packed(lengths, H, d, seed, sigma=1.0):
    total = int(sum(lengths)) + 3  # trailing rows outside every sequence
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((total, H, d)) * s for s in (sigma, sigma, 1.0))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return q, k, v, cu


@pytest.mark.parametrize("causal,window,slopes", [
    (False, (-1, -1), None), (True, (-1, -1), None), (False, (2, 1), [0.25, 0.5]),
    (True, (3, -1), [0.4, 0.0])])
def test_each_sequence_matches_fsum_brute_force(causal, window, slopes):
    lengths = [1, 4, 0, 7, 5]
    H, d = 2, 3
    q, k, v, cu = _packed(lengths, H, d, seed=11)
    scale = 0.7
    O, L = oracle.attention_varlen(q, k, v, cu, scale=scale, causal=causal, window=window,
                                   alibi_slopes=slopes)
    for b in range(len(lengths)):
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        for h in range(H):
            Ob, Lb = brute.attention_fsum_masked(q[s0:s1, h], k[s0:s1, h], v[s0:s1, h],
                                                 scale=scale, causal=causal, window=window,
                                                 slope=0.0 if slopes is None else slopes[h])
            assert np.abs(O[s0:s1, h] - np.array(Ob)).max() <= 1e-13
            assert np.abs(L[h, s0:s1] - np.array(Lb)).max() <= 1e-13
    # rows outside every sequence stay undefined
    assert np.isnan(O[cu[-1]:]).all() and np.isnan(L[:, cu[-1]:]).all()


def test_one_token_sequence_returns_its_value_row():
    q, k, v, cu = _packed([3, 1, 2], 2, 4, seed=12)
    scale = 0.5
    O, L = oracle.attention_varlen(q, k, v, cu, scale=scale, causal=False)
    r = cu[1]
    assert np.array_equal(O[r], v[r])
    assert np.abs(L[:, r] - scale * np.einsum("hd,hd->h", q[r], k[r])).max() <= 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_equal_keys_average_only_the_own_sequence(causal):
    lengths = [5, 6, 4]
    q, k, v, cu = _packed(lengths, 1, 3, seed=13)
    k[:] = 0.37  # every score of a row is the same number
    O, _ = oracle.attention_varlen(q, k, v, cu, causal=causal)
    for s0, s1 in zip(cu, cu[1:]):
        vs = v[s0:s1, 0]
        want = (np.cumsum(vs, 0) / np.arange(1, s1 - s0 + 1)[:, None]) if causal else \
            np.broadcast_to(vs.mean(0), vs.shape)
        assert np.abs(O[s0:s1, 0] - want).max() <= 1e-14


def test_sequences_are_independent():
    lengths = [6, 9, 5]
    q, k, v, cu = _packed(lengths, 2, 4, seed=14)
    O1, L1 = oracle.attention_varlen(q, k, v, cu, causal=True, window=(3, -1))
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    sl = slice(cu[1], cu[2])
    for t in (q2, k2, v2):
        t[sl] = np.random.default_rng(99).standard_normal(t[sl].shape)
    O2, L2 = oracle.attention_varlen(q2, k2, v2, cu, causal=True, window=(3, -1))
    keep = np.r_[0:cu[1], cu[2]:cu[3]]
    assert np.array_equal(O1[keep], O2[keep]) and np.array_equal(L1[:, keep], L2[:, keep])
    assert not np.array_equal(O1[sl], O2[sl])


def test_equal_lengths_are_the_fixed_length_problem():
    B, H, N, d = 3, 2, 9, 4
    rng = np.random.default_rng(15)
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    O, L = oracle.attention(q, k, v, causal=True)
    packed = [t.transpose(0, 2, 1, 3).reshape(B * N, H, d) for t in (q, k, v)]
    cu = np.arange(0, B * N + 1, N)
    Ov, Lv = oracle.attention_varlen(*packed, cu, causal=True)
    assert np.abs(Ov.reshape(B, N, H, d).transpose(0, 2, 1, 3) - O).max() <= 1e-14
    assert np.abs(Lv.reshape(H, B, N).transpose(1, 0, 2) - L).max() <= 1e-13


def _varlen_planted(q, k, v, cu, slip, **kw):
    """A copy of the varlen composition with one planted slip."""
    total, H, d = q.shape
    O = np.full((total, H, d), np.nan)
    L = np.full((H, total), np.nan)
    for s0, s1 in zip(cu, cu[1:]):
        e = min(s1 + 1, total) if slip == "boundary" else s1
        seq = [np.ascontiguousarray(t[s0:e].transpose(1, 0, 2))[None] for t in (q, k, v)]
        o, lse = oracle.attention_masked(*seq, **kw)
        O[s0:s1] = o[0].transpose(1, 0, 2)[: s1 - s0]
        L[:, s0:s1] = lse[0][:, : s1 - s0]
    if slip == "lse_layout":
        L = L.T.copy().reshape(H, total)
    return O, L


def test_planted_mistakes_are_caught():
    # a sequence boundary off by one (each sequence also sees the next row):
    # the equal-keys pin fails
    q, k, v, cu = _packed([5, 6, 4], 1, 3, seed=16)
    k[:] = 0.37
    O, _ = _varlen_planted(q, k, v, cu, "boundary")
    assert np.abs(O[cu[0]:cu[1], 0] - v[cu[0]:cu[1], 0].mean(0)).max() > 1e-3
    O, _ = _varlen_planted(q, k, v, cu, None)
    assert np.abs(O[cu[0]:cu[1], 0] - v[cu[0]:cu[1], 0].mean(0)).max() <= 1e-14
    # the LSE stored [total, H] instead of [H, total]: the one-token pin fails
    q, k, v, cu = _packed([3, 1, 2], 2, 4, seed=12)
    _, L = _varlen_planted(q, k, v, cu, "lse_layout", scale=0.5)
    r = cu[1]
    assert not (np.abs(L[:, r] - 0.5 * np.einsum("hd,hd->h", q[r], k[r])).max() <= 1e-15)
