"""GPU parity of the fp8 (e4m3) forward (fa_fwd_fp8) against the fp64 fp8
oracle (``oracle.attention_fp8``: the same codes and factors, dequantised).

Tolerance, derived from the arithmetic.  The kernel forms S from the e4m3
codes with fp32 accumulation (products of two e4m3 values are exact in fp32),
takes the softmax weights p_j = 2^(t_j - m_ref) in fp32 and rounds them to
e4m3 before P V, dividing by the fp32 sum l of the unrounded weights.  e4m3
round-to-nearest of p <= 256 errs by at most max(2^-4 p, 2^-10) (3 mantissa
bits; subnormal spacing 2^-9), and 1/l <= w_max, the row's largest softmax
weight (the row max's weight is >= 1 in the kernel's units).  So each output
element obeys

    |O - O_ref| <= sum_j max(2^-4 w_j, 2^-10 w_max) |v_j| + 2^-8 |O_ref|

with w_j the oracle's softmax weights, v_j the dequantised values and the
last term the bf16 output rounding.  The test allows 1.25x that plus 1e-5
(fp32 sums, ex2.approx).  The LSE uses the unrounded sum: 1e-3 relative as
the 16-bit path.  At the bench size (N = 4096) the P rounding errors average
over thousands of keys, and the 16-bit path's mean-abs bound (2e-3) is checked
as well.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_154_b200 import fa, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load()
    yield
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_OK, f"watchdog fired: {detail:#x}"


def _dequant(c, f):
    return f * oracle.decode_e4m3(c.view(torch.uint8).numpy())


def _check(o, lse, codes, factors, scale, causal, rows=None, mean_abs=None, label=""):
    q, k, v = (_dequant(c, f) for c, f in zip(codes, factors))
    O_ref, L_ref = oracle.attention_fp8(*codes, *factors, scale=scale, causal=causal, rows=rows)
    B, H, N, d = q.shape
    rr = np.arange(N) if rows is None else np.asarray(rows)
    o = o.double().numpy()[:, :, rr]
    err = np.abs(o - O_ref)
    worst = 0.0
    for b in range(B):
        for h in range(H):
            W = np.stack([oracle.probs(q[b, h], k[b, h], int(i), scale=scale, causal=causal)
                          for i in rr])
            A = np.maximum(2.0 ** -4 * W, 2.0 ** -10 * W.max(axis=1, keepdims=True))
            bound = A @ np.abs(v[b, h]) + 2.0 ** -8 * np.abs(O_ref[b, h])
            worst = max(worst, float((err[b, h] / (1.25 * bound + 1e-5)).max()))
    lerr = np.abs(lse.double().numpy()[:, :, rr] - L_ref) / np.maximum(1.0, np.abs(L_ref))
    res = {"o_max_abs": float(err.max()), "o_mean_abs": float(err.mean()),
           "worst_over_bound": worst, "lse_rel": float(lerr.max())}
    assert np.isfinite(o).all() and worst <= 1.0 and res["lse_rel"] <= 1e-3, f"{label}: {res}"
    if mean_abs is not None:
        assert res["o_mean_abs"] <= mean_abs, f"{label}: {res}"
    return res


def _run(codes, factors, causal, scale=None):
    o, lse = fa.fwd_fp8(*(c.cuda() for c in codes), *factors, scale=scale, causal=causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("N", [1, 129, 513, 1000])
def test_fp8_small_shapes_full(N, d, causal):
    codes, factors = synth.fp8_inputs(2, 2, N, d, seed=4000 + N + d)
    o, lse = _run(codes, factors, causal)
    _check(o, lse, codes, factors, fa.default_scale(d), causal, label=f"N={N} d={d} causal={causal}")


def test_fp8_one_key_is_the_value_row():
    codes, factors = synth.fp8_inputs(2, 3, 1, 128, seed=4100)
    o, lse = _run(codes, factors, False)
    want = torch.from_numpy(_dequant(codes[2], factors[2])).to(torch.bfloat16)
    assert torch.equal(o, want)


def test_fp8_skewed_logits_head_dim_256_causal():
    # q, k ~ N(0, 3^2) as the head-dim 256 workload: nearly one-hot rows
    codes, factors = synth.fp8_inputs(1, 2, 2048, 256, seed=4101, sigma_qk=3.0)
    o, lse = _run(codes, factors, True)
    rows = synth.sample_rows(2048, 4101, count=128)
    _check(o, lse, codes, factors, fa.default_scale(256), True, rows=rows, label="skewed d=256")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_bench_size_sampled(causal):
    # the N = 4096 sweep shape (B=4, H=16, d=128)
    codes, factors = synth.fp8_inputs(4, 16, 4096, 128, seed=4102 + int(causal))
    o, lse = _run(codes, factors, causal)
    rows = synth.sample_rows(4096, 4102, count=64)
    res = _check(o, lse, codes, factors, fa.default_scale(128), causal, rows=rows,
                 mean_abs=2e-3, label=f"bench size causal={causal}")
    print("fp8 bench-size errors:", res)


def test_fp8_deterministic_and_explicit_scale():
    codes, factors = synth.fp8_inputs(1, 4, 700, 128, seed=4103)
    o1, l1 = _run(codes, factors, True, scale=0.05)
    o2, l2 = _run(codes, factors, True, scale=0.05)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    _check(o1, l1, codes, factors, float(torch.tensor(0.05, dtype=torch.float32)), True,
           label="explicit scale")
