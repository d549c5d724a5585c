"""fa_bwd_noalloc (library-owned row-statistic array) against fa_bwd (caller
workspace): the same kernels on the same inputs, so the gradients must match
bit for bit, on two consecutive calls with different inputs."""
import pytest
import torch

from exact_attention_154_b200 import fa, synth
from exact_attention_154_b200.synth import BF16, FP16


def test_noalloc_capacity_checked_on_the_host():
    lib = fa.load()
    P = 1 << 20
    # B * H * N above the array's 8,388,608 floats is refused before any launch
    assert lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 64, 64, 4096, 64, 0.0, 0, 1, None) == fa.FA_ERR_ARG
    assert lib.fa_bwd_noalloc(None, P, P, P, P, P, P, P, P, 1, 1, 128, 64, 0.0, 0, 1, None) == fa.FA_ERR_ARG


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [((2, 3, 700, 128), BF16, True, 81), ((1, 4, 1000, 64), FP16, False, 82)]
    for (B, H, N, d), dtype, causal, seed in cases:
        q, k, v = (t.cuda() for t in synth.random_inputs(B, H, N, d, dtype, seed=seed))
        g = synth.random_inputs(B, H, N, d, dtype, seed=seed + 100)[0].cuda()
        o, lse = fa.fwd(q, k, v, causal=causal)
        ref = fa.bwd(q, k, v, o, lse, g, causal=causal)
        got = fa.bwd_noalloc(q, k, v, o, lse, g, causal=causal)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert fa.device_status(clear=True)[0] == fa.FA_OK
