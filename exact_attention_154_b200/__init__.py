"""B200 (sm_100a) exact attention forward.

``fwd`` / ``fwd_qkvpacked`` call the C ABI of ``libfa_sm100.so`` (declared in
``include/fa.h``); ``synth`` draws the seeded synthetic inputs.
"""
from .fa import (FaError, device_status, fwd, fwd_qkvpacked, launch_ctas, load, strerror,
                 version, watchdog_selftest)

__all__ = ["FaError", "device_status", "fwd", "fwd_qkvpacked", "launch_ctas", "load",
           "strerror", "version", "watchdog_selftest"]
