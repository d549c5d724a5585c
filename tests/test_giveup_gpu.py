"""The attention kernels' own give-up path, on the GPU, without a fault or a
hang: with every mbarrier wait bounded to 200 ns (far below one tile load),
the forward and the backward kernels' waits run out.  Each CTA then raises
its abort flag, drains what it issued, frees tensor memory and returns; the
device word reports FA_ERR_TIMEOUT with the role and site of the first wait
that gave up.  The next normal calls in the same process must be
parity-green and leave the device word clean."""
import numpy as np
import pytest
import torch

from exact_attention_154_b200 import fa, synth
from exact_attention_154_b200.synth import BF16

from parity import check

pytestmark = pytest.mark.gpu

ROLES = {1: "producer", 2: "mma", 3: "softmax", 6: "store"}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.load()
    fa.device_status(clear=True)
    yield
    fa.set_wait_limit(0)
    assert fa.device_status(clear=True)[0] == fa.FA_OK


def _timed_out():
    rc, detail = fa.device_status(clear=True)
    assert rc == fa.FA_ERR_TIMEOUT, (rc, hex(detail))
    assert (detail >> 8) in ROLES and 1 <= (detail & 0xFF) <= 16, hex(detail)
    return detail


def test_forward_gives_up_then_recovers():
    q, k, v = synth.random_inputs(4, 16, 4096, 128, BF16, seed=5000)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    try:
        fa.set_wait_limit(200)
        for causal in (False, True):
            fa.fwd(qc, kc, vc, causal=causal)
            _timed_out()
    finally:
        fa.set_wait_limit(0)
    o, lse = fa.fwd(qc, kc, vc, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True)[0] == fa.FA_OK
    check(o.cpu(), lse.cpu(), q, k, v, fa.default_scale(128), True,
          rows=[0, 127, 128, 2047, 4095], label="after give-up")


def test_backward_gives_up_then_recovers():
    B, H, N, d = 2, 8, 2048, 128
    q, k, v = (t.cuda() for t in synth.random_inputs(B, H, N, d, BF16, seed=5001))
    g = synth.random_inputs(B, H, N, d, BF16, seed=5002)[0].cuda()
    o, lse = fa.fwd(q, k, v, causal=True)
    ref = fa.bwd(q, k, v, o, lse, g, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True)[0] == fa.FA_OK
    try:
        fa.set_wait_limit(200)
        fa.bwd(q, k, v, o, lse, g, causal=True)
        _timed_out()
    finally:
        fa.set_wait_limit(0)
    again = fa.bwd(q, k, v, o, lse, g, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status(clear=True)[0] == fa.FA_OK
    for a, b in zip(again, ref):
        assert torch.equal(a, b)  # the same kernels on the same inputs
