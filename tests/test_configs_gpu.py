"""GPU parity on the five benchmark workloads at full size.

The two small workloads are compared on every element.  The large ones are
compared on >= 512 seeded query rows per (b, h) (always including rows 0,
127, 128 and N-1): each row of the output depends only on its own query and
the head's K and V, so the sampled rows are checked exactly as in a full
comparison.  Launch configuration is the one ``bench.py`` times.
"""
import pytest
import torch

from exact_attention_154_b200 import fa, synth

from parity import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert fa.device_status(clear=True)[0] == fa.FA_OK


def _run(w, rows=None):
    if w.layout == "packed":
        (qkv,) = synth.make_inputs(w)
        o, lse = fa.fwd_qkvpacked(qkv.cuda(), causal=w.causal)
        torch.cuda.synchronize()
        q, k, v = synth.unpack_qkv(qkv)
        o = o.cpu().permute(0, 2, 1, 3)
    else:
        q, k, v = synth.make_inputs(w)
        o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal)
        torch.cuda.synchronize()
        o = o.cpu()
    return check(o, lse.cpu(), q, k, v, fa.default_scale(w.d), w.causal, rows=rows,
                 label=w.name)


def test_single_head_n256_full():
    _run(synth.single_head_n256())


def test_packed_qkv_full():
    _run(synth.packed_qkv_b2_n256_h12())


def test_many_heads_causal_sampled():
    w = synth.many_heads_causal_n2048()
    _run(w, rows=synth.sample_rows(w.N, w.seed))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", synth.SWEEP_N)
def test_seqlen_sweep_sampled(N, causal):
    w = synth.seqlen_sweep(N, causal)
    _run(w, rows=synth.sample_rows(w.N, w.seed))


def test_headdim256_skewed_causal_sampled():
    w = synth.headdim256_causal()
    res = _run(w, rows=synth.sample_rows(w.N, w.seed))
    print("head-dim 256 errors:", res)
