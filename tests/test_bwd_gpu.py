"""GPU parity of the attention backward (``fa_bwd``) against the fp64 gradient
oracle (``oracle.attention_bwd``, pinned in ``tests/test_oracle_bwd_pins.py``).

The forward of this library supplies O and LSE, as a user's training step
would.  The bound is derived from the arithmetic, per element: the kernel
rounds P and dS to the 16-bit input type before the tensor-core products and
reads D = rowsum(dO * O) from the forward's 16-bit O; each rounding is at most
u = 2^-8 (bf16) or 2^-11 (fp16) relative.  With E[i,j] = P[i,j] *
(2u |dP[i,j] - D_i| + u sum_c |dO[i,c] O[i,c]|) the error of dS, the bounds are

    |err dV_j| <= u sum_i P[i,j] |dO_i| ,   |err dK_j| <= scale sum_i E[i,j] |q_i| ,
    |err dQ_i| <= scale sum_j E[i,j] |k_j| ,

each plus the output rounding u |ref|; the test allows twice the bound plus
1e-6 (fp32 accumulation and exp2 approximation are orders of magnitude below).
"""
import numpy as np
import pytest
import torch

from exact_attention_154_b200 import fa, synth
from exact_attention_154_b200.synth import BF16, FP16
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load()
    yield
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_OK, f"watchdog fired: {detail:#x}"


def _bounds(q, k, v, dout, scale, causal, u):
    q, k, v, g = (t.double().numpy() for t in (q, k, v, dout))
    N = q.shape[-2]
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    if causal:
        s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    o = p @ v
    dp = np.einsum("bhid,bhjd->bhij", g, v)
    D = (g * o).sum(-1, keepdims=True)
    Dabs = np.abs(g * o).sum(-1, keepdims=True)
    E = p * (2 * u * np.abs(dp - D) + u * Dabs)
    bdv = u * np.einsum("bhij,bhid->bhjd", p, np.abs(g))
    bdk = scale * np.einsum("bhij,bhid->bhjd", E, np.abs(q))
    bdq = scale * np.einsum("bhij,bhjd->bhid", E, np.abs(k))
    return bdq, bdk, bdv


def _check(q, k, v, dout, causal, dtype, label):
    scale = fa.default_scale(q.shape[-1])
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.bwd(qc, kc, vc, o, lse, gc, causal=causal)
    torch.cuda.synchronize()
    ref = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=causal)
    u = 2.0 ** -8 if dtype == BF16 else 2.0 ** -11
    bounds = _bounds(q, k, v, dout, scale, causal, u)
    for name, got, r, bnd in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref, bounds):
        g = got.cpu().double().numpy()
        assert np.isfinite(g).all(), f"{label} {name}: non-finite"
        err = np.abs(g - r)
        allowed = 2.0 * (bnd + u * np.abs(r)) + 1e-6
        worst = float((err / allowed).max())
        assert worst <= 1.0, f"{label} {name}: error {err.max():.3e}, {worst:.2f} x the bound"


@pytest.mark.parametrize("dtype", [FP16, BF16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 64, 128, 129, 200, 256, 300, 513])
def test_small_shapes(N, d, causal, dtype):
    q, k, v = synth.random_inputs(1, 2, N, d, dtype, seed=3000 + N + d + int(causal))
    dout = synth.random_inputs(1, 2, N, d, dtype, seed=4000 + N + d)[0]
    _check(q, k, v, dout, causal, dtype, f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_several_heads_long_sequence(causal):
    q, k, v = synth.random_inputs(2, 3, 1024, 128, BF16, seed=5000 + int(causal), sigma_qk=1.5)
    dout = synth.random_inputs(2, 3, 1024, 128, BF16, seed=5100)[0]
    _check(q, k, v, dout, causal, BF16, f"B=2 H=3 N=1024 causal={causal}")


def test_single_key_closed_form():
    # N = 1: O = V, so dV = dO and dQ = dK = 0.  On the GPU P = exp2(s - LSE)
    # is 1 up to fp32 rounding and dP - D cancels up to fp32 summation order,
    # so dV equals dO to 16-bit rounding and dQ, dK vanish to ~1e-7.
    q, k, v = synth.random_inputs(2, 2, 1, 128, BF16, seed=61)
    dout = synth.random_inputs(2, 2, 1, 128, BF16, seed=62)[0]
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.fwd(qc, kc, vc)
    dq, dk, dv = fa.bwd(qc, kc, vc, o, lse, gc)
    torch.cuda.synchronize()
    g = dout.double()
    assert (dv.cpu().double() - g).abs().max() <= 2.0 ** -8 * g.abs().max()
    assert dq.abs().max() <= 1e-4 and dk.abs().max() <= 1e-4


def test_key_gradients_sum_to_zero():
    # adding one vector to every key leaves O unchanged: sum_j dK_j = 0
    q, k, v = synth.random_inputs(1, 2, 384, 64, FP16, seed=71)
    dout = synth.random_inputs(1, 2, 384, 64, FP16, seed=72)[0]
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.fwd(qc, kc, vc, causal=True)
    _, dk, _ = fa.bwd(qc, kc, vc, o, lse, gc, causal=True)
    torch.cuda.synchronize()
    dkd = dk.double()
    assert dkd.sum(dim=2).abs().max() <= 2e-2 * dkd.abs().sum(dim=2).max()


@pytest.mark.parametrize("d,dtype,N", [(128, BF16, 512), (64, FP16, 512), (128, BF16, 500)])
@pytest.mark.parametrize("causal", [False, True])
def test_more_units_than_ctas(causal, d, dtype, N):
    """160 key blocks and 160 query blocks (B=1, H=40, N=512, or N=500 with a
    ragged last block) on a persistent grid of at most one CTA per SM: some
    CTAs take a second unit, carrying the ring slots and the per-step barrier
    phases over from the first (d = 64: the dK/dV kernel with two dP regions
    as well)."""
    q, k, v = synth.random_inputs(1, 40, N, d, dtype, seed=5200 + int(causal) + d + N)
    dout = synth.random_inputs(1, 40, N, d, dtype, seed=5300 + d + N)[0]
    assert 40 * ((N + 127) // 128) > torch.cuda.get_device_properties(0).multi_processor_count
    _check(q, k, v, dout, causal, dtype, f"B=1 H=40 N={N} d={d} causal={causal}")
