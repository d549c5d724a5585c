"""Pins of the windowed / ALiBi oracle (``oracle.attention_masked``) to facts
that do not come from the oracle itself.

* Limits: the unbounded window is the plain definition; a window at least N
  wide on the left and 0 on the right is the causal mask; slope 0 adds nothing.
* Closed forms: window (0, 0) leaves each row one key, so O = V and LSE = the
  diagonal score; with all scores equal, ALiBi weights are a two-sided (or,
  causal, one-sided) geometric series, whose sums are textbook formulas.
* Brute force: a scalar ``math.fsum`` evaluation on tiny inputs.
* Invariants: adding one vector to every key leaves O unchanged (the bias
  depends only on positions); per-head slopes act head by head.

``test_planted_mistakes_are_caught`` checks that plausible slips (a window
off by one, the bias sign flipped, the bias without the absolute value, the
bias scaled with the scores) each break at least one pin.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import brute


def _rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


@pytest.mark.parametrize("causal", [False, True])
def test_unbounded_window_is_the_definition(causal):
    q, k, v = (_rand((2, 3, 37, 8), s) for s in (1, 2, 3))
    O, L = oracle.attention(q, k, v, causal=causal)
    Om, Lm = oracle.attention_masked(q, k, v, causal=causal, window=(-1, -1))
    assert np.abs(Om - O).max() <= 1e-14 and np.abs(Lm - L).max() <= 1e-13


def test_wide_left_window_is_causal_and_slope_zero_adds_nothing():
    q, k, v = (_rand((1, 2, 29, 8), s) for s in (4, 5, 6))
    Oc, Lc = oracle.attention(q, k, v, causal=True)
    Ow, Lw = oracle.attention_masked(q, k, v, window=(29, 0))
    assert np.abs(Ow - Oc).max() <= 1e-14 and np.abs(Lw - Lc).max() <= 1e-13
    Of, Lf = oracle.attention(q, k, v)
    Oz, Lz = oracle.attention_masked(q, k, v, window=(40, 40), alibi_slopes=[0.0, 0.0])
    assert np.abs(Oz - Of).max() <= 1e-14 and np.abs(Lz - Lf).max() <= 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_window_zero_keeps_the_diagonal_only(causal):
    q, k, v = (_rand((2, 2, 11, 5), s) for s in (7, 8, 9))
    scale = 0.3
    O, L = oracle.attention_masked(q, k, v, scale=scale, causal=causal, window=(0, 0),
                                   alibi_slopes=[0.7, 1.3])
    assert np.array_equal(O, v)
    diag = scale * np.einsum("bhid,bhid->bhi", q, k)
    assert np.abs(L - diag).max() <= 1e-14


def _geometric(r, n):
    """sum_{k<n} r^k and sum_{k<n} k r^k (textbook closed forms)."""
    s0 = (1.0 - r ** n) / (1.0 - r)
    s1 = r * (1.0 - n * r ** (n - 1) + (n - 1) * r ** n) / (1.0 - r) ** 2
    return s0, s1


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("slope", [0.25, 1.0])
def test_alibi_on_equal_scores_is_a_geometric_series(slope, causal):
    N, d = 23, 2
    q = np.zeros((N, d))  # every score is 0, so only the bias differs
    k = _rand((N, d), 10)
    v = np.stack([np.arange(N, dtype=float), np.ones(N)], axis=1)  # v_j = (j, 1)
    O, L = oracle.attention_masked(q, k, v, causal=causal, alibi_slopes=[slope])
    r = math.exp(-slope)
    for i in range(N):
        # keys left of i (k = 0..i steps back) and, non-causal, right of i
        a0, a1 = _geometric(r, i + 1)
        den, num = a0, i * a0 - a1
        if not causal:
            b0, b1 = _geometric(r, N - i)  # k = 0..N-1-i; drop k = 0 below
            den += b0 - 1.0
            num += i * (b0 - 1.0) + b1
        assert abs(O[i, 0] - num / den) <= 1e-12 * max(1.0, abs(num / den))
        assert abs(O[i, 1] - 1.0) <= 1e-14
        assert abs(L[i] - math.log(den)) <= 1e-13


@pytest.mark.parametrize("window", [(-1, -1), (2, 1), (0, 3), (4, 0), (1, -1)])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_fsum_brute_force(window, causal):
    N, d = 7, 3
    q, k, v = (_rand((N, d), 20 + s) for s in range(3))
    O, L = oracle.attention_masked(q, k, v, scale=0.6, causal=causal, window=window,
                                   alibi_slopes=[0.45])
    Ob, Lb = brute.attention_fsum_masked(q.tolist(), k.tolist(), v.tolist(), scale=0.6,
                                         causal=causal, window=window, slope=0.45)
    assert np.abs(O - np.array(Ob)).max() <= 1e-13
    assert np.abs(L - np.array(Lb)).max() <= 1e-13


def test_key_shift_invariance_and_per_head_slopes():
    q, k, v = (_rand((1, 3, 31, 6), 30 + s) for s in range(3))
    slopes = [0.1, 0.5, 2.0]
    O, _ = oracle.attention_masked(q, k, v, window=(5, 3), alibi_slopes=slopes)
    u = _rand((6,), 40)
    Os, _ = oracle.attention_masked(q, k + u, v, window=(5, 3), alibi_slopes=slopes)
    assert np.abs(Os - O).max() <= 1e-12
    for h, sl in enumerate(slopes):
        Oh, _ = oracle.attention_masked(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1],
                                        window=(5, 3), alibi_slopes=[sl])
        assert np.abs(Oh[:, 0] - O[:, h]).max() <= 1e-15


def test_bad_arguments_rejected():
    x = _rand((4, 4), 50)
    with pytest.raises(ValueError):
        oracle.attention_masked(x, x, x, window=(-2, 0))
    with pytest.raises(ValueError):
        oracle.attention_masked(x[None, None], x[None, None], x[None, None], alibi_slopes=[1.0, 2.0])


def _mutant(q, k, v, scale, causal, window, slope, slip):
    """A deliberately wrong copy of the masked definition, for the pin self-test."""
    N = q.shape[0]
    left, right = window
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = np.ones((N, N), dtype=bool)
    lo = i - left + (1 if slip == "window_off_by_one" else 0)
    if left >= 0:
        vis &= j >= lo
    if right >= 0:
        vis &= j <= i + right
    if causal:
        vis &= j <= i
    dist = (i - j) if slip == "bias_without_abs" else np.abs(i - j)
    bias = (1 if slip == "bias_sign" else -1) * slope * dist
    s = (q @ k.T + bias) * scale if slip == "bias_scaled" else scale * (q @ k.T) + bias
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return (e @ v) / z, (m + np.log(z))[:, 0]


@pytest.mark.parametrize("slip", ["window_off_by_one", "bias_sign", "bias_without_abs",
                                  "bias_scaled"])
def test_planted_mistakes_are_caught(slip):
    """Every planted slip disagrees with the fsum brute force or a closed form."""
    N, d, scale, slope = 8, 3, 0.6, 0.45
    q, k, v = (_rand((N, d), 60 + s) for s in range(3))
    caught = []
    for causal in (False, True):
        for window in ((2, 1), (-1, -1)):
            O, L = _mutant(q, k, v, scale, causal, window, slope, slip)
            Ob, Lb = brute.attention_fsum_masked(q.tolist(), k.tolist(), v.tolist(), scale=scale,
                                                 causal=causal, window=window, slope=slope)
            caught.append(not (np.allclose(O, Ob, atol=1e-12) and np.allclose(L, Lb, atol=1e-12)))
    assert any(caught), f"slip {slip} went unnoticed"
