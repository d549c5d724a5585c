"""Host-only checks of the build inputs, the binding's device checks and the
software exp2's coefficients.  No GPU."""
import os
import re

import numpy as np
import pytest
import torch

from exact_attention_154_b200 import _build, fa

CSRC = _build.CSRC


def _includes(path):
    text = open(path).read()
    return re.findall(r'#include\s+"([^"]+)"', text)


def test_every_included_header_is_a_build_input():
    inputs = {os.path.realpath(p) for p in _build._inputs()}
    seen, todo = set(), [os.path.join(CSRC, s) for s in _build.SOURCES]
    while todo:
        path = os.path.realpath(todo.pop())
        if path in seen:
            continue
        seen.add(path)
        for inc in _includes(path):
            todo.append(os.path.join(os.path.dirname(path), inc))
    assert seen <= inputs, f"not tracked by the build: {sorted(seen - inputs)}"


def test_same_device_accepts_one_device_and_names_the_odd_tensor():
    a, b = torch.empty(2), torch.empty(2)
    assert fa.same_device([("q", a), ("k", b)]) == torch.device("cpu")
    m = torch.empty(2, device="meta")
    with pytest.raises(ValueError, match="k is on meta"):
        fa.same_device([("q", a), ("k", m)])


def _exp2_coefficients():
    text = open(os.path.join(CSRC, "fa_fwd_sm100.cuh")).read()
    m = re.search(r"constexpr float c0 = ([0-9.eE+-]+)f, c1 = ([0-9.eE+-]+)f,\s*"
                  r"c2 = ([0-9.eE+-]+)f, c3 = ([0-9.eE+-]+)f;", text)
    assert m, "exp2 polynomial coefficients not found"
    return [np.float32(float(x)) for x in m.groups()]


def test_exp2_polynomial_meets_its_stated_relative_bound_in_fp32():
    """2^f on [-1/2, 1/2] by the kernel's degree-3 polynomial, evaluated with
    fp32 fused multiply-adds as the kernel does (Horner, rounded once per
    step), against 2^f in fp64: the stated 7.5e-5 relative bound."""
    c0, c1, c2, c3 = _exp2_coefficients()
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64).astype(np.float32)

    def fma32(a, b, c):  # one rounding, as the hardware FFMA
        return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)

    q = fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = fma32(q, f, np.full_like(f, c1))
    q = fma32(q, f, np.full_like(f, c0))
    rel = np.abs(q.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5
    # and it is a genuine fit, not a loose one: the error is within 2x of the bound
    assert rel.max() >= 3e-5
    # equioscillation of a minimax fit: the extreme error recurs across the interval
    peaks = rel > 0.9 * rel.max()
    assert peaks[: len(f) // 3].any() and peaks[len(f) // 3: 2 * len(f) // 3].any() \
        and peaks[2 * len(f) // 3:].any()
