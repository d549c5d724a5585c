"""B200 (sm_100a) exact attention: the forward and its gradient.

``fwd`` / ``fwd_qkvpacked`` / ``fwd_varlen`` / ``fwd_fp8`` and ``bwd`` / ``bwd_noalloc`` call the C ABI of
``libfa_sm100.so`` (declared in ``include/fa.h``); ``synth`` draws the seeded
synthetic inputs.
"""
from .fa import (FaError, bwd, bwd_noalloc, device_status, fwd, fwd_fp8, fwd_qkvpacked,
                 fwd_varlen, launch_ctas, load, strerror, version, watchdog_selftest)

__all__ = ["FaError", "bwd", "bwd_noalloc", "device_status", "fwd", "fwd_fp8",
           "fwd_qkvpacked", "fwd_varlen", "launch_ctas", "load", "strerror", "version", "watchdog_selftest"]
