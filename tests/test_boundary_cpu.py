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
    for code in range(-9, 1):
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


def test_ext_argument_errors(lib):
    def call(q=P, left=-1, right=-1, slopes=None, N=256, causal=0, lse=None):
        return lib.fa_fwd_ext(q, P, P, P, lse, 1, 2, N, 64, 0.0, causal, left, right, slopes, 1,
                              None)
    assert call(q=None) == fa.FA_ERR_ARG
    assert call(left=-2) == fa.FA_ERR_ARG
    assert call(right=-3, causal=1) == fa.FA_ERR_ARG
    assert call(slopes=P + 2) == fa.FA_ERR_ALIGN
    assert call(q=P + 4, left=5) == fa.FA_ERR_ALIGN

    def packed(qkv=P, dropout=0.0, left=-1, right=-1, slopes=None):
        return lib.fa_fwd_qkvpacked_ext(qkv, P, None, 2, 256, 4, 64, 0.0, 0, dropout, left, right,
                                        slopes, 0, None)
    assert packed(qkv=None) == fa.FA_ERR_ARG
    assert packed(dropout=0.5) == fa.FA_ERR_UNSUPPORTED
    assert packed(left=-7) == fa.FA_ERR_ARG
    assert packed(slopes=P + 1) == fa.FA_ERR_ALIGN


def test_varlen_argument_errors(lib):
    def call(q=P, cu=P, batch=2, max_seqlen=128, total=200, H=2, d=64, dtype=0, slopes=None,
             left=-1):
        return lib.fa_fwd_varlen(q, P, P, P, None, cu, batch, max_seqlen, total, H, d, 0.0, 0, left,
                                 -1, slopes, dtype, None)
    assert call(cu=None) == fa.FA_ERR_ARG
    assert call(q=None) == fa.FA_ERR_ARG
    assert call(batch=0) == fa.FA_ERR_ARG
    assert call(max_seqlen=0) == fa.FA_ERR_ARG
    assert call(total=0) == fa.FA_ERR_ARG
    assert call(d=48) == fa.FA_ERR_HEADDIM
    assert call(dtype=5) == fa.FA_ERR_DTYPE
    assert call(left=-4) == fa.FA_ERR_ARG
    assert call(cu=P + 2) == fa.FA_ERR_ALIGN
    assert call(slopes=P + 2) == fa.FA_ERR_ALIGN
    assert call(q=P + 8) == fa.FA_ERR_ALIGN


def test_python_varlen_rejects_bad_offsets_tensor():
    import torch
    x = torch.zeros(8, 2, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.fwd_varlen(x, x, x, torch.tensor([0, 8], dtype=torch.int64), 8)


def test_fp8_argument_errors(lib):
    def call(q=P, d=128, scale=0.0, dq=0.01, dk=0.01, dv=0.01, causal=0, lse=None, N=256):
        return lib.fa_fwd_fp8(q, P, P, P, lse, 1, 2, N, d, scale, dq, dk, dv, causal, None)
    assert call(q=None) == fa.FA_ERR_ARG
    assert call(d=64) == fa.FA_ERR_HEADDIM
    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(dq=0.0) == fa.FA_ERR_ARG
    assert call(dk=-1.0) == fa.FA_ERR_ARG
    assert call(dv=float("inf")) == fa.FA_ERR_ARG
    assert call(dq=float("nan")) == fa.FA_ERR_ARG
    assert call(scale=-0.5) == fa.FA_ERR_ARG
    assert call(dq=1e30, dk=1e30) == fa.FA_ERR_ARG  # scale * dq * dk overflows
    assert call(causal=3) == fa.FA_ERR_ARG
    assert call(q=P + 4) == fa.FA_ERR_ALIGN
    assert call(lse=P + 1) == fa.FA_ERR_ALIGN
    # the 16-bit entry points refuse the e4m3 dtype
    assert lib.fa_fwd(P, P, P, P, None, 1, 1, 128, 128, 0.0, 0, 2, None) == fa.FA_ERR_DTYPE
    assert lib.fa_fwd_qkvpacked(P, P, None, 1, 128, 1, 128, 0.0, 0, 0.0, 2, None) == fa.FA_ERR_DTYPE


def test_wait_limit_hook_argument_check(lib):
    assert lib.fa_debug_set_wait_limit(50) == fa.FA_ERR_ARG
    assert lib.fa_debug_set_wait_limit(10**11) == fa.FA_ERR_ARG
    assert lib.fa_debug_set_wait_limit(0) == fa.FA_OK  # the default
