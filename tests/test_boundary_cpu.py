"""Host-only checks of the C ABI: the library loads, exports every function
``include/fa.h`` declares, and rejects bad arguments before touching a GPU.

No call here launches work: every call either fails an argument check or
queries static data."""
import os
import re

import pytest

from exact_attention_154_b200 import fa
from exact_attention_154_b200._build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return fa.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = header_functions()
    for required in ("fa_fwd", "fa_fwd_qkvpacked", "fa_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert names, "no declarations parsed"
    for name in names:
        assert hasattr(lib, name), f"{name} not exported"
    assert set(names) == set(fa.SIGNATURES), "binding and header disagree"


def test_version_and_strerror(lib):
    assert fa.version() >= 10000
    for code in range(-8, 1):
        assert fa.strerror(code) != "unknown status"
    assert fa.strerror(-99) == "unknown status"


# fake, never dereferenced device addresses (16-byte aligned unless stated)
P = 1 << 20


def _fwd(lib, q=P, k=P, v=P, o=P, lse=None, B=1, H=1, N=128, d=128, scale=0.0, causal=0, dtype=1):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, q=None) == fa.FA_ERR_ARG
    assert _fwd(lib, o=None) == fa.FA_ERR_ARG
    assert _fwd(lib, B=0) == fa.FA_ERR_ARG
    assert _fwd(lib, H=-1) == fa.FA_ERR_ARG
    assert _fwd(lib, N=0) == fa.FA_ERR_ARG
    assert _fwd(lib, d=96) == fa.FA_ERR_HEADDIM
    assert _fwd(lib, d=32) == fa.FA_ERR_HEADDIM
    assert _fwd(lib, dtype=2) == fa.FA_ERR_DTYPE
    assert _fwd(lib, scale=-1.0) == fa.FA_ERR_ARG
    assert _fwd(lib, scale=float("nan")) == fa.FA_ERR_ARG
    assert _fwd(lib, scale=float("inf")) == fa.FA_ERR_ARG
    assert _fwd(lib, causal=2) == fa.FA_ERR_ARG
    assert _fwd(lib, q=P + 8) == fa.FA_ERR_ALIGN
    assert _fwd(lib, o=P + 2) == fa.FA_ERR_ALIGN
    assert _fwd(lib, lse=P + 2) == fa.FA_ERR_ALIGN
    # sizes whose tile count no longer fits the device index type
    assert _fwd(lib, B=1 << 20, H=1 << 12, N=1 << 12) == fa.FA_ERR_ARG


def test_packed_argument_errors(lib):
    def call(qkv=P, o=P, B=2, N=256, H=12, d=64, scale=0.0, causal=0, dropout=0.0, dtype=0):
        return lib.fa_fwd_qkvpacked(qkv, o, None, B, N, H, d, scale, causal, dropout, dtype, None)
    assert call(qkv=None) == fa.FA_ERR_ARG
    assert call(dropout=0.1) == fa.FA_ERR_UNSUPPORTED
    assert call(dropout=float("nan")) == fa.FA_ERR_ARG
    assert call(d=80) == fa.FA_ERR_HEADDIM
    assert call(dtype=7) == fa.FA_ERR_DTYPE
    assert call(qkv=P + 4) == fa.FA_ERR_ALIGN


def test_selftest_argument_check(lib):
    assert lib.fa_debug_watchdog_selftest(0, None) == fa.FA_ERR_ARG
    assert lib.fa_debug_watchdog_selftest(10**11, None) == fa.FA_ERR_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.fwd(x, x, x)


def test_library_has_no_torch_dependency():
    """The C ABI library links no torch or Python symbols."""
    import subprocess
    out = subprocess.run(["ldd", fa.lib_path()], capture_output=True, text=True).stdout
    assert "torch" not in out and "python" not in out


def test_exp2_hook_argument_check(lib):
    assert lib.fa_debug_exp2_poly(None, P, 4, None) == fa.FA_ERR_ARG
    assert lib.fa_debug_exp2_poly(P, P, -1, None) == fa.FA_ERR_ARG


def test_bwd_argument_errors(lib):
    def call(q=P, o=P, lse=P, ws=P, B=1, H=1, N=128, d=128, scale=0.0, causal=0, dtype=1):
        return lib.fa_bwd(q, P, P, o, lse, P, P, P, P, ws, B, H, N, d, scale, causal, dtype, None)
    assert call(q=None) == fa.FA_ERR_ARG
    assert call(lse=None) == fa.FA_ERR_ARG
    assert call(ws=None) == fa.FA_ERR_ARG
    assert call(N=0) == fa.FA_ERR_ARG
    assert call(d=256) == fa.FA_ERR_HEADDIM
    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(dtype=3) == fa.FA_ERR_DTYPE
    assert call(scale=float("nan")) == fa.FA_ERR_ARG
    assert call(q=P + 8) == fa.FA_ERR_ALIGN
    assert call(o=P + 2) == fa.FA_ERR_ALIGN
    assert call(lse=P + 2) == fa.FA_ERR_ALIGN
    assert call(ws=P + 1) == fa.FA_ERR_ALIGN
