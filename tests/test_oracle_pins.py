"""Pins for the fp64 oracle, checked against facts that do not come from it.

Each test fixes one property that the definition of attention (standard
attention of "2.3 FlashAttention与IO感知注意力(1)", aiknowledge.cn, section 1.1;
``standard_attention`` of "flash_attention.py", forceinjection.github.io)
forces, chosen so that a plausible slip in the oracle (a dropped scale, a
transposed operand, a wrong mask edge, a missing max shift, a wrong log base)
breaks at least one of them.  ``test_planted_mistakes_are_caught`` checks that
claim by planting such slips in copies of the oracle on the CPU.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import brute, tiled

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _rand(*shape, sigma=1.0):
    return rng.standard_normal(shape) * sigma


@pytest.mark.parametrize("causal", [False, True])
def test_golden_two_key_example(oracle_mod, causal):
    g = json.load(open(os.path.join(GOLDEN, "two_key_worked_example.json")))
    O, L = oracle_mod.attention(np.array(g["q"], float), np.array(g["k"], float),
                                np.array(g["v"], float), scale=g["scale"], causal=causal)
    ref = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(O, ref["O"], rtol=0, atol=g["tolerance"])
    np.testing.assert_allclose(L, ref["LSE"], rtol=0, atol=g["tolerance"])


@pytest.mark.parametrize("causal", [False, True])
def test_n1_returns_v0(oracle_mod, causal):
    q, k, v = _rand(1, 64), _rand(1, 64), _rand(1, 64)
    O, L = oracle_mod.attention(q, k, v, causal=causal)
    np.testing.assert_array_equal(O, v)
    assert abs(L[0] - (q[0] @ k[0]) / 8.0) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_all_equal_keys_give_mean_of_visible_v(oracle_mod, causal):
    N, d = 37, 16
    q, v = _rand(N, d), _rand(N, d)
    c = _rand(d)
    k = np.tile(c, (N, 1))
    scale = 0.3
    O, L = oracle_mod.attention(q, k, v, scale=scale, causal=causal)
    for i in range(N):
        nv = i + 1 if causal else N
        np.testing.assert_allclose(O[i], v[:nv].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(L[i] - (scale * (q[i] @ c) + math.log(nv))) < 1e-12


def test_causal_row0_is_v0(oracle_mod):
    q, k, v = _rand(50, 32, sigma=3.0), _rand(50, 32, sigma=3.0), _rand(50, 32)
    O, L = oracle_mod.attention(q, k, v, causal=True)
    np.testing.assert_array_equal(O[0], v[0])
    assert abs(L[0] - (q[0] @ k[0]) / math.sqrt(32)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(oracle_mod, causal):
    N, d = 61, 24
    q, k = _rand(N, d, sigma=2.0), _rand(N, d, sigma=2.0)
    for i in (0, 1, 30, 60):
        p = oracle_mod.probs(q, k, i, causal=causal)
        assert abs(p.sum() - 1.0) < 1e-15 * N
        assert np.all(p >= 0)
        if causal:
            assert np.all(p[i + 1:] == 0) and np.all(p[: i + 1] > 0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_uniform_average(oracle_mod, causal):
    N, d = 45, 8
    q, k, v = np.zeros((N, d)), _rand(N, d), _rand(N, d)
    O, L = oracle_mod.attention(q, k, v, causal=causal)
    for i in range(N):
        nv = i + 1 if causal else N
        np.testing.assert_allclose(O[i], v[:nv].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(L[i] - math.log(nv)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_and_linearity_in_v(oracle_mod, causal):
    N, d = 33, 16
    q, k = _rand(N, d), _rand(N, d)
    O, _ = oracle_mod.attention(q, k, np.full((N, d), 2.5), causal=causal)
    np.testing.assert_allclose(O, 2.5, rtol=0, atol=1e-14)
    v1, v2 = _rand(N, d), _rand(N, d)
    O1, _ = oracle_mod.attention(q, k, v1, causal=causal)
    O2, _ = oracle_mod.attention(q, k, v2, causal=causal)
    O12, _ = oracle_mod.attention(q, k, 3.0 * v1 - 0.5 * v2, causal=causal)
    np.testing.assert_allclose(O12, 3.0 * O1 - 0.5 * O2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(oracle_mod, causal):
    N, d = 40, 16
    q, k, v = _rand(N, d), _rand(N, d), _rand(N, d)
    u = _rand(d)
    scale = 0.25
    O, L = oracle_mod.attention(q, k, v, scale=scale, causal=causal)
    O2, L2 = oracle_mod.attention(q, k + u, v, scale=scale, causal=causal)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L + scale * (q @ u), rtol=0, atol=1e-12)


def test_permutation_equivariance(oracle_mod):
    N, d = 29, 8
    q, k, v = _rand(N, d), _rand(N, d), _rand(N, d)
    O, L = oracle_mod.attention(q, k, v)
    perm = rng.permutation(N)
    Ok, Lk = oracle_mod.attention(q, k[perm], v[perm])
    np.testing.assert_allclose(Ok, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lk, L, rtol=0, atol=1e-13)
    Oq, Lq = oracle_mod.attention(q[perm], k, v)
    np.testing.assert_allclose(Oq, O[perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lq, L[perm], rtol=0, atol=1e-13)


def test_two_keys_closed_form(oracle_mod):
    d = 12
    q, k, v = _rand(2, d), _rand(2, d), _rand(2, d)
    scale = 0.7
    O, L = oracle_mod.attention(q, k, v, scale=scale)
    for i in range(2):
        s0, s1 = scale * (q[i] @ k[0]), scale * (q[i] @ k[1])
        w0 = scipy.special.expit(s0 - s1)
        np.testing.assert_allclose(O[i], w0 * v[0] + (1 - w0) * v[1], rtol=0, atol=1e-14)
        assert abs(L[i] - np.logaddexp(s0, s1)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
def test_brute_force_fsum(oracle_mod, N, causal):
    d = 6
    q, k, v = _rand(N, d), _rand(N, d), _rand(N, d)
    O, L = oracle_mod.attention(q, k, v, causal=causal)
    Ob, Lb = brute.attention_fsum(q.tolist(), k.tolist(), v.tolist(), causal=causal)
    np.testing.assert_allclose(O, np.array(Ob), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, np.array(Lb), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_matches_library_logsumexp(oracle_mod, causal):
    N, d = 70, 32
    q, k, v = _rand(N, d, sigma=3.0), _rand(N, d, sigma=3.0), _rand(N, d)
    scale = 1.0 / math.sqrt(d)
    _, L = oracle_mod.attention(q, k, v, causal=causal)
    S = scale * (q @ k.T)
    for i in range(N):
        nv = i + 1 if causal else N
        assert abs(L[i] - scipy.special.logsumexp(S[i, :nv])) < 1e-12


# The shapes and seed of compare_and_verify in "flash_attention.py"
# (forceinjection.github.io), (B, N, d) = (1,256,64), (1,512,64), (1,1024,64),
# (4,512,64) with seed 42 (with its 64 x 64 blocks; smaller blocks on smaller
# shapes, and two ragged shapes, so the pure-NumPy loop stays fast).
@pytest.mark.parametrize("B,N,d", [(1, 256, 64), (1, 96, 64), (2, 130, 64)])
@pytest.mark.parametrize("Br,Bc", [(64, 64), (1, 3), (3, 1), (64, 17)])
@pytest.mark.parametrize("causal", [False, True])
def test_tiled_recurrence_equals_definition(oracle_mod, B, N, d, Br, Bc, causal):
    if (Br, Bc) in ((1, 3), (3, 1)) and N > 96:
        pytest.skip("tiny blocks only on the smallest shape (pure Python loop)")
    r = np.random.default_rng(42)
    q, k, v = (r.standard_normal((B, N, d)) for _ in range(3))
    O, L = oracle_mod.attention(q, k, v, causal=causal)
    Ot, Lt = tiled.flash_forward(q, k, v, causal=causal, Br=Br, Bc=Bc)
    np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lt, L, rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,N,d", [(1, 512, 64), (1, 1024, 64), (4, 512, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_tiled_recurrence_on_the_pages_shapes(oracle_mod, B, N, d, causal):
    r = np.random.default_rng(42)
    q, k, v = (r.standard_normal((B, N, d)) for _ in range(3))
    O, L = oracle_mod.attention(q, k, v, causal=causal)
    Ot, Lt = tiled.flash_forward(q, k, v, causal=causal, Br=64, Bc=64)
    np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lt, L, rtol=0, atol=1e-12)


def test_row_subset_matches_full(oracle_mod):
    B, H, N, d = 2, 3, 50, 8
    q, k, v = (_rand(B, H, N, d) for _ in range(3))
    O, L = oracle_mod.attention(q, k, v, causal=True)
    rows = [49, 0, 17, 17]
    Os, Ls = oracle_mod.attention(q, k, v, causal=True, rows=rows)
    np.testing.assert_array_equal(Os, O[:, :, rows])
    np.testing.assert_array_equal(Ls, L[:, :, rows])


def test_large_logits_are_stable(oracle_mod):
    # scores near +-1000 would overflow exp() without the max shift
    N, d = 20, 4
    q, k, v = _rand(N, d, sigma=30.0), _rand(N, d, sigma=30.0), _rand(N, d)
    O, L = oracle_mod.attention(q, k, v, scale=1.0)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    S = q @ k.T
    np.testing.assert_allclose(L, scipy.special.logsumexp(S, axis=1), rtol=1e-14, atol=0)


def test_bad_arguments_rejected(oracle_mod):
    q = _rand(4, 4)
    with pytest.raises(ValueError):
        oracle_mod.attention(q, q, _rand(5, 4))
    with pytest.raises(ValueError):
        oracle_mod.attention(q, q, q, rows=[4])


def _mutant_attention(q, k, v, scale, causal, slip):
    """A deliberately wrong copy of the definition, for the pin self-test."""
    N, d = q.shape
    S = (q @ (k if slip == "transpose_k" else k).T)
    if slip == "transpose_k":
        S = S.T
    if slip != "drop_scale":
        S = S * scale
    nv = np.arange(N) + (2 if slip == "mask_off_by_one" else 1)
    if causal:
        S = np.where(np.arange(N)[None, :] < nv[:, None], S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    P = np.exp(S - m)
    l = P.sum(axis=1, keepdims=True)
    O = (P @ v) / l
    L = (m + np.log(l))[:, 0]
    if slip == "log2_lse":
        L = (m[:, 0] + np.log2(l[:, 0]))
    if slip == "lse_without_max":
        L = np.log(l[:, 0])
    return O, L


@pytest.mark.parametrize("slip", ["drop_scale", "transpose_k", "mask_off_by_one",
                                  "log2_lse", "lse_without_max"])
def test_planted_mistakes_are_caught(slip):
    """Every planted slip breaks at least one of the pinned properties."""
    N, d = 9, 4
    r = np.random.default_rng(7)
    q, k, v = r.standard_normal((N, d)), r.standard_normal((N, d)), r.standard_normal((N, d))
    caught = []
    for causal in (False, True):
        O, L = _mutant_attention(q, k, v, 0.5, causal, slip)
        Ob, Lb = brute.attention_fsum(q.tolist(), k.tolist(), v.tolist(), scale=0.5,
                                      causal=causal)
        caught.append(not (np.allclose(O, Ob, atol=1e-12) and np.allclose(L, Lb, atol=1e-12)))
    assert any(caught), f"slip {slip} went unnoticed"
