"""Pins of the fp64 backward oracle (``oracle.attention_bwd``) to facts that do
not come from the oracle itself.

* Central finite differences of the *forward* oracle's loss sum(O * dO): the
  gradient of the plain definition, whatever code computes it.
* Reverse-mode differentiation of the same definition by torch's autograd in
  fp64 (a library routine, written independently of the oracle).
* Closed forms: N = 1 (O = V), constant V, dO = 0, causal row 0.
* Invariants: the key gradients sum to zero (O does not change when the same
  vector is added to every key), the value gradients sum to the sum of dO
  (every row of P sums to one), linearity in dO.

``test_planted_mistakes_are_caught`` checks that each of a set of plausible
slips in a backward pass (a dropped scale, a wrong sign in the softmax
Jacobian, an unnormalised P, an off-by-one causal mask, dS in place of P for
dV) breaks at least one of these pins.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


def _loss(q, k, v, dout, scale, causal):
    o, _ = oracle.attention(q, k, v, scale=scale, causal=causal)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("causal", [False, True])
def test_matches_central_finite_differences(causal):
    shape, scale, h = (1, 2, 6, 5), 0.37, 1e-5
    q, k, v, dout = (_rand(shape, s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=causal)
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            up = _loss(q, k, v, dout, scale, causal)
            x[idx] = keep - h
            down = _loss(q, k, v, dout, scale, causal)
            x[idx] = keep
            num[idx] = (up - down) / (2 * h)
        assert np.abs(num - g).max() <= 1e-7 * max(1.0, np.abs(g).max())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 8), (7, 4), (33, 16), (130, 64)])
def test_matches_fp64_autograd_of_the_definition(N, d, causal):
    shape = (2, 3, N, d)
    q, k, v, dout = (_rand(shape, 10 + s, sigma=1.5) for s in range(4))
    scale = 1.0 / np.sqrt(d)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    s = (tq @ tk.transpose(-1, -2)) * scale
    if causal:
        mask = torch.ones(N, N, dtype=torch.bool).tril()
        s = s.masked_fill(~mask, float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(dout))
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=causal)
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(got - ref.numpy()).max() <= 1e-12 * max(1.0, float(ref.abs().max()))


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_gives_dv_equal_dout_and_no_score_gradient(causal):
    q, k, v, dout = (_rand((3, 1, 6), s) for s in range(4))
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, causal=causal)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    assert np.allclose(dv, dout, rtol=0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_key_gradients_sum_to_zero_and_value_gradients_to_sum_of_dout(causal):
    shape = (2, 2, 40, 8)
    q, k, v, dout = (_rand(shape, 20 + s, sigma=2.0) for s in range(4))
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, causal=causal)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-12 * np.abs(dk).max()
    assert np.abs(dv.sum(axis=2) - dout.sum(axis=2)).max() <= 1e-12 * np.abs(dout).sum(axis=2).max()


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_give_no_score_gradient(causal):
    shape = (1, 2, 17, 8)
    q, k, dout = (_rand(shape, 30 + s) for s in range(3))
    v = np.broadcast_to(_rand((1, 2, 1, 8), 33), shape).copy()
    dq, dk, _ = oracle.attention_bwd(q, k, v, dout, causal=causal)
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13


def test_zero_and_linear_in_dout():
    shape = (1, 3, 23, 8)
    q, k, v, g1, g2 = (_rand(shape, 40 + s) for s in range(5))
    zero = oracle.attention_bwd(q, k, v, np.zeros(shape), causal=True)
    assert all(not np.any(z) for z in zero)
    a = oracle.attention_bwd(q, k, v, g1, causal=True)
    b = oracle.attention_bwd(q, k, v, g2, causal=True)
    c = oracle.attention_bwd(q, k, v, 2.0 * g1 - 3.0 * g2, causal=True)
    for x, y, z in zip(a, b, c):
        assert np.abs(z - (2.0 * x - 3.0 * y)).max() <= 1e-12 * np.abs(z).max()


def test_causal_row0_query_gets_no_gradient():
    q, k, v, dout = (_rand((2, 2, 9, 4), 50 + s) for s in range(4))
    dq, _, _ = oracle.attention_bwd(q, k, v, dout, causal=True)
    assert np.array_equal(dq[:, :, 0], np.zeros_like(dq[:, :, 0]))


def test_bad_arguments_rejected():
    x = _rand((4, 4), 60)
    with pytest.raises(ValueError):
        oracle.attention_bwd(x, x, x, _rand((5, 4), 61))


def _mutant_bwd(q, k, v, dout, scale, causal, slip):
    """A deliberately wrong backward of one [N, d] slice, for the pin self-test."""
    N = q.shape[0]
    s = (q @ k.T) * scale
    nv = np.arange(N) + (2 if slip == "mask_off_by_one" else 1)
    if causal:
        s = np.where(np.arange(N)[None, :] < nv[:, None], s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p = e if slip == "unnormalised_p" else e / e.sum(axis=1, keepdims=True)
    dv = p.T @ dout
    dp = dout @ v.T
    D = np.sum(p * dp, axis=1, keepdims=True)
    ds = p * (dp + D) if slip == "jacobian_sign" else p * (dp - D)
    if slip == "ds_for_dv":
        dv = ds.T @ dout
    dq = ds @ k * (1.0 if slip == "drop_scale" else scale)
    dk = ds.T @ q * scale
    return dq, dk, dv


@pytest.mark.parametrize("slip", ["drop_scale", "jacobian_sign", "unnormalised_p",
                                  "mask_off_by_one", "ds_for_dv"])
def test_planted_mistakes_are_caught(slip):
    """Every planted slip breaks the finite-difference pin or an invariant."""
    N, d, scale, h = 7, 4, 0.6, 1e-6
    q, k, v, dout = (_rand((N, d), 70 + s) for s in range(4))
    caught = []
    for causal in (False, True):
        dq, dk, dv = _mutant_bwd(q, k, v, dout, scale, causal, slip)
        ok = abs(dk.sum(axis=0)).max() < 1e-12 and abs(dv.sum(axis=0) - dout.sum(axis=0)).max() < 1e-12
        for x, g in ((q, dq), (k, dk), (v, dv)):
            for idx in [(0, 0), (N // 2, 1), (N - 1, d - 1)]:
                keep = x[idx]
                x[idx] = keep + h
                up = _loss(q, k, v, dout, scale, causal)
                x[idx] = keep - h
                down = _loss(q, k, v, dout, scale, causal)
                x[idx] = keep
                ok = ok and abs((up - down) / (2 * h) - g[idx]) < 1e-6
        caught.append(not ok)
    assert any(caught), f"slip {slip} went unnoticed"
