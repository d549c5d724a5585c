"""The kernel's software exp2 (degree-3 minimax polynomial after rint range
reduction, run on the FMA pipe for part of the softmax weights) against CUDA's
exp2f, over the argument range the softmax can produce."""
import pytest
import torch

from exact_attention_154_b200 import fa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_relative_error_bound():
    # arguments are x = s*scale*log2(e) - m_ref <= 8 (lazy rescale threshold)
    x = torch.linspace(-120.0, 8.0, 2_000_001, device="cuda", dtype=torch.float32)
    y = fa.exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1.0e-4, rel     # minimax bound of the fit is 7.5e-5
    # exact powers of two stay within the same bound; 2^0 is the common case
    xi = torch.arange(-100, 9, device="cuda", dtype=torch.float32)
    yi = fa.exp2_poly(xi).double()
    assert ((yi - torch.exp2(xi.double())).abs() / torch.exp2(xi.double())).max() < 1.0e-4


def test_underflow_is_clamped_not_wrapped():
    x = torch.tensor([-126.0, -150.0, -1e4, -3.0e38], device="cuda")
    y = fa.exp2_poly(x)
    assert torch.all(y >= 0) and torch.all(y <= 2.0 ** -125)


def test_odd_length():
    x = torch.tensor([0.0, 1.0, -1.0], device="cuda")
    y = fa.exp2_poly(x)
    assert torch.allclose(y, torch.tensor([1.0, 2.0, 0.5], device="cuda"), rtol=1e-4)
