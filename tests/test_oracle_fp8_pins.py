"""Pins of the fp8 oracle (``oracle.decode_e4m3``, ``oracle.attention_fp8``)
to facts that do not come from the oracle itself.

* Decoding: every one of the 256 codes against torch's float8_e4m3fn
  conversion (a library routine), and the format's landmark values (1, the
  largest finite 448, the smallest normal 2^-6 and subnormal 2^-9, NaN).
* Dequantisation: a one-key problem returns descale_v * v and the LSE
  scale * descale_q * descale_k * q.k in closed form; O is linear in
  descale_v with the LSE unchanged; descale_q and descale_k act only through
  their product; on codes whose values bf16 represents exactly (all e4m3
  values), unit factors give the bf16 definition.

``test_planted_mistakes_are_caught``: a dropped exponent bias, a subnormal
decoded as normal, descale_v applied to the scores, and descale_k dropped
each break a pin.
"""
import numpy as np
import torch

import oracle


def test_all_codes_match_torch_float8_e4m3fn():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])


def test_landmark_values():
    d = oracle.decode_e4m3
    assert d(0x38) == 1.0 and d(0xB8) == -1.0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x08) == 2.0 ** -6 and d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9
    assert d(0x00) == 0.0 and np.signbit(d(0x80))
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))


def _codes(shape, seed):
    # finite codes only (NaN excluded), both signs
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3F
    return c


def test_one_key_closed_form():
    q, k, v = (_codes((2, 3, 1, 16), s) for s in (1, 2, 3))
    dq, dk, dv, scale = 0.01, 0.02, 0.5, 0.25
    O, L = oracle.attention_fp8(q, k, v, dq, dk, dv, scale=scale)
    dec = oracle.decode_e4m3
    assert np.array_equal(O, dv * dec(v))
    want = scale * dq * dk * np.einsum("bhnd,bhnd->bhn", dec(q), dec(k))
    assert np.abs(L - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


def test_descale_v_is_linear_and_leaves_lse():
    q, k, v = (_codes((1, 2, 33, 16), s) for s in (4, 5, 6))
    O1, L1 = oracle.attention_fp8(q, k, v, 0.01, 0.01, 1.0, causal=True)
    O2, L2 = oracle.attention_fp8(q, k, v, 0.01, 0.01, 2.5, causal=True)
    assert np.abs(O2 - 2.5 * O1).max() <= 1e-12 * np.abs(O1).max()
    assert np.array_equal(L1, L2)


def test_q_and_k_factors_act_through_their_product():
    q, k, v = (_codes((1, 2, 29, 16), s) for s in (7, 8, 9))
    O1, L1 = oracle.attention_fp8(q, k, v, 0.02, 0.005, 1.0)
    O2, L2 = oracle.attention_fp8(q, k, v, 0.01, 0.01, 1.0)
    assert np.abs(O1 - O2).max() <= 1e-12 and np.abs(L1 - L2).max() <= 1e-12


def test_unit_factors_give_the_bf16_definition():
    q, k, v = (_codes((2, 2, 40, 32), s) for s in (10, 11, 12))
    as_bf16 = [torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.bfloat16) for c in (q, k, v)]
    # every e4m3 value is a bf16 value: the conversion is exact
    for c, b in zip((q, k, v), as_bf16):
        assert np.array_equal(b.double().numpy(), oracle.decode_e4m3(c))
    O1, L1 = oracle.attention_fp8(q, k, v, 1.0, 1.0, 1.0, scale=2.0 ** -12, causal=True)
    O2, L2 = oracle.attention(*as_bf16, scale=2.0 ** -12, causal=True)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def _decode_planted(codes, slip):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    if slip == "bias":
        mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    else:  # "subnormal": e = 0 taken as a normal number
        mag = (1.0 + m / 8.0) * np.exp2(np.maximum(e, 1) - 7.0)
    return sign * mag


def test_planted_mistakes_are_caught():
    assert _decode_planted(0x38, "bias") != 1.0  # landmark pin
    assert _decode_planted(0x01, "subnormal") != 2.0 ** -9
    q, k, v = (_codes((1, 1, 1, 16), s) for s in (13, 14, 15))
    dec = oracle.decode_e4m3
    dq, dk, dv, scale = 0.01, 0.02, 0.5, 0.25
    # descale_v applied to the scores: the one-key LSE pin fails
    L_bad = oracle.attention(dq * dec(q), dk * dec(k) * dv, dv * dec(v), scale=scale)[1]
    want = scale * dq * dk * np.einsum("bhnd,bhnd->bhn", dec(q), dec(k))
    assert np.abs(L_bad - want).max() > 1e-9
    # descale_k dropped: the product pin fails
    q, k, v = (_codes((1, 2, 29, 16), s) for s in (7, 8, 9))
    O1 = oracle.attention(0.02 * dec(q), dec(k), dec(v))[0]
    O2 = oracle.attention(0.01 * dec(q), dec(k), dec(v))[0]
    assert np.abs(O1 - O2).max() > 1e-6
