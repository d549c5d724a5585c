"""GPU parity of the variable-length forward (fa_fwd_varlen) against the
fp64 oracle run per sequence (``oracle.attention_varlen``), element by element.

Length mixes include empty and one-token sequences, lengths on and just past
a tile boundary and several-tile ragged lengths, with trailing rows that
belong to no sequence (which must stay untouched), a max_seqlen above the
longest length, and every head dim.  Bounds as the plain forward.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_154_b200 import fa, synth
from exact_attention_154_b200.synth import BF16, FP16

from parity import compare, to_f64

pytestmark = pytest.mark.gpu

LENGTHS = [1, 7, 128, 0, 129, 300, 513, 256]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load()
    yield
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_OK, f"watchdog fired: {detail:#x}"


def _varlen(q, k, v, cu, max_seqlen, sentinel=7.0, **kw):
    qc, kc, vc, cuc = q.cuda(), k.cuda(), v.cuda(), cu.cuda()
    out = torch.full_like(qc, sentinel)
    total, H, d = q.shape
    lse = torch.full((H, total), sentinel, device="cuda", dtype=torch.float32)
    lib = fa.load()
    slopes = kw.get("alibi_slopes")
    sl = None if slopes is None else slopes.cuda()
    left, right = kw.get("window", (-1, -1))
    rc = lib.fa_fwd_varlen(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), out.data_ptr(),
                           lse.data_ptr(), cuc.data_ptr(), cu.numel() - 1, max_seqlen, total, H,
                           d, 0.0, int(kw.get("causal", False)), left, right,
                           None if sl is None else sl.data_ptr(),
                           BF16 if q.dtype == torch.bfloat16 else FP16,
                           torch.cuda.current_stream().cuda_stream)
    assert rc == fa.FA_OK, fa.strerror(rc)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window,alibi", [
    (False, (-1, -1), False), (True, (-1, -1), False), (False, (64, 3), True),
    (True, (200, -1), True), (False, (0, 0), False)])
def test_varlen_mix(d, causal, window, alibi):
    H = 3
    dtype = BF16 if d != 64 else FP16
    q, k, v, cu = synth.packed_lengths(LENGTHS, H, d, dtype, seed=3000 + d, extra_rows=5)
    slopes = synth.alibi_slopes(H) if alibi else None
    o, lse = _varlen(q, k, v, cu, max(LENGTHS) + 40, causal=causal, window=window,
                     alibi_slopes=slopes)
    O, L = oracle.attention_varlen(q, k, v, cu.numpy(), scale=fa.default_scale(d), causal=causal,
                                   window=window,
                                   alibi_slopes=None if slopes is None else slopes.double().numpy())
    end = int(cu[-1])
    compare(to_f64(o[:end]), o.dtype, to_f64(lse[:, :end]), O[:end], L[:, :end],
            label=f"varlen d={d} causal={causal} window={window} alibi={alibi}")
    # rows outside every sequence are not written
    assert (o[end:] == 7.0).all() and (lse[:, end:] == 7.0).all()


def test_equal_lengths_are_bitwise_the_fixed_forward():
    B, H, N, d = 3, 4, 300, 128
    q, k, v = synth.random_inputs(B, H, N, d, BF16, seed=3101)
    o_ref, l_ref = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    packed = [t.transpose(1, 2).reshape(B * N, H, d).contiguous() for t in (q, k, v)]
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32)
    o, lse = fa.fwd_varlen(*(t.cuda() for t in packed), cu.cuda(), N, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o.cpu().reshape(B, N, H, d).transpose(1, 2), o_ref.cpu())
    assert torch.equal(lse.cpu().reshape(H, B, N).transpose(0, 1), l_ref.cpu())


def test_bad_offsets_are_reported_and_skipped():
    H, d = 2, 64
    q, k, v, _ = synth.packed_lengths([100, 300], H, d, FP16, seed=3102)
    # sequence 1 has length -50 (decreasing offsets): skipped and reported;
    # sequence 0 is computed as usual, rows past it stay untouched
    cu = torch.tensor([0, 100, 50, 50], dtype=torch.int32)
    o, lse = _varlen(q, k, v, cu, 256)
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_ERR_SEQLENS and detail == (5 << 8) | 14
    O, L = oracle.attention_varlen(q[:100], k[:100], v[:100], np.array([0, 100]),
                                   scale=fa.default_scale(d))
    compare(to_f64(o[:100]), o.dtype, to_f64(lse[:, :100]), O, L, label="before bad offsets")
    assert (o[100:] == 7.0).all() and (lse[:, 100:] == 7.0).all()
    # a sequence longer than max_seqlen is skipped as well
    cu = torch.tensor([0, 100, 400], dtype=torch.int32)
    o, _ = _varlen(q, k, v, cu, 256)
    rc, _ = fa.device_status(clear=True)
    assert rc == fa.FA_ERR_SEQLENS and (o[100:] == 7.0).all()
    assert np.abs(to_f64(o[:100]) - O).max() <= 2e-2
    # the context is fine afterwards
    q2, k2, v2, cu2 = synth.packed_lengths([33, 200], H, d, FP16, seed=3103)
    o2, l2 = _varlen(q2, k2, v2, cu2, 200)
    O, L = oracle.attention_varlen(q2, k2, v2, cu2.numpy(), scale=fa.default_scale(d))
    compare(to_f64(o2), o2.dtype, to_f64(l2), O, L, label="after bad offsets")
    assert fa.device_status(clear=True)[0] == fa.FA_OK


def test_many_sequences_sampled_lengths():
    # 64 sequences with lengths drawn from 1..2048 (seeded), H = 8, d = 128
    rng = np.random.default_rng(3104)
    lengths = [int(x) for x in rng.integers(1, 2049, size=64)]
    H, d = 8, 128
    q, k, v, cu = synth.packed_lengths(lengths, H, d, BF16, seed=3104)
    o, lse = fa.fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), causal=True)
    torch.cuda.synchronize()
    # check four whole sequences (first, last, longest, shortest)
    pick = sorted({0, len(lengths) - 1, int(np.argmax(lengths)), int(np.argmin(lengths))})
    for b in pick:
        s0, s1 = int(cu[b]), int(cu[b + 1])
        sub = [t[s0:s1] for t in (q, k, v)]
        O, L = oracle.attention_varlen(*sub, np.array([0, s1 - s0]), scale=fa.default_scale(d),
                                       causal=True)
        compare(to_f64(o[s0:s1].cpu()), o.dtype, to_f64(lse[:, s0:s1].cpu()), O, L,
                label=f"sequence {b} (length {s1 - s0})")
