"""GPU parity of the local-window and ALiBi forward (fa_fwd_ext,
fa_fwd_qkvpacked_ext) against the fp64 masked oracle, element by element.

Windows cover the degenerate (0, 0) (one key per row), narrow two-sided,
one-sided, block-sized and wider-than-a-block windows, each with and without
the causal mask and per-head ALiBi slopes, at N = 1, a ragged two-tile N and
a ragged multi-block N, for every head dim.  Bounds as the plain forward:
O max-abs <= 2e-2, mean-abs <= 2e-3, |dLSE| <= 1e-3 max(1, |LSE|).
"""
import numpy as np
import pytest
import torch

from exact_attention_154_b200 import fa, synth
from exact_attention_154_b200.synth import BF16, FP16

from parity import check

pytestmark = pytest.mark.gpu

WINDOWS = [(-1, -1), (0, 0), (2, 1), (128, 0), (300, -1), (-1, 5), (64, 64), (200, 130)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load()
    yield
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_OK, f"watchdog fired: {detail:#x}"


def _run(q, k, v, causal, window, slopes, scale=None):
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=causal,
                    window_size=window, alibi_slopes=slopes)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("alibi", [False, True])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", WINDOWS)
def test_window_alibi_small(window, causal, alibi, d):
    H = 3
    dtype = BF16 if (d + window[0]) % 2 == 0 else FP16
    for N in (1, 129, 513):
        q, k, v = synth.random_inputs(2, H, N, d, dtype, seed=2000 + N + d + window[0])
        slopes = synth.alibi_slopes(H) if alibi else None
        o, lse = _run(q, k, v, causal, window, slopes)
        check(o, lse, q, k, v, fa.default_scale(d), causal, window=window,
              alibi_slopes=None if slopes is None else slopes.double().numpy(),
              label=f"N={N} d={d} causal={causal} window={window} alibi={alibi}")


def test_steep_slopes_and_explicit_scale():
    # slopes up to 4 make each row's weights nearly one-hot on its diagonal
    H, N, d = 4, 700, 128
    q, k, v = synth.random_inputs(1, H, N, d, BF16, seed=2101, sigma_qk=2.0)
    slopes = torch.tensor([0.0, 0.5, 1.5, 4.0])
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, (-1, -1), slopes, scale=0.1)
        check(o, lse, q, k, v, float(torch.tensor(0.1, dtype=torch.float32)), causal,
              window=(-1, -1), alibi_slopes=slopes.double().numpy(), label="steep slopes")


def test_window_zero_returns_v():
    for d in (64, 128, 256):
        q, k, v = synth.random_inputs(2, 2, 300, d, FP16, seed=2102)
        o, lse = _run(q, k, v, False, (0, 0), synth.alibi_slopes(2))
        assert torch.equal(o, v)


def test_packed_ext_matches_oracle():
    g = torch.Generator().manual_seed(2103)
    B, N, H, d = 2, 333, 4, 64
    qkv = torch.randn(B, N, 3, H, d, generator=g).to(torch.float16)
    slopes = synth.alibi_slopes(H)
    o, lse = fa.fwd_qkvpacked(qkv.cuda(), causal=True, window_size=(100, 0),
                              alibi_slopes=slopes.cuda())
    torch.cuda.synchronize()
    q, k, v = synth.unpack_qkv(qkv)
    check(o.cpu().permute(0, 2, 1, 3), lse.cpu(), q, k, v, fa.default_scale(d), True,
          window=(100, 0), alibi_slopes=slopes.double().numpy(), label="packed ext")


@pytest.mark.parametrize("causal,window,alibi", [(True, (256, 0), True), (False, (512, 512), False),
                                                 (True, (-1, -1), True)])
def test_bench_size_sampled(causal, window, alibi):
    # the sweep's N = 4096 shape (B=4, H=16, d=128), >= 512 sampled rows per head
    w = synth.seqlen_sweep(4096, causal)
    q, k, v = synth.make_inputs(w)
    slopes = synth.alibi_slopes(w.H) if alibi else None
    o, lse = _run(q, k, v, causal, window, slopes)
    rows = synth.sample_rows(w.N, w.seed)
    check(o, lse, q, k, v, fa.default_scale(w.d), causal, rows=rows, window=window,
          alibi_slopes=None if slopes is None else slopes.double().numpy(),
          label=f"bench size {window} alibi={alibi}")


def test_unbounded_ext_is_bitwise_the_plain_forward():
    q, k, v = (t.cuda() for t in synth.random_inputs(2, 4, 1000, 128, BF16, seed=2104))
    for causal in (False, True):
        o1, l1 = fa.fwd(q, k, v, causal=causal)
        o2, l2 = fa.fwd(q, k, v, causal=causal, window_size=(5000, 5000))
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
