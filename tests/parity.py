"""Shared parity helpers for the GPU tests (CUDA path vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Acceptance bounds on N(0,1)-class inputs: O max-abs and mean-abs error, and
# LSE error relative to max(1, |LSE|).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_REL = 1e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def check(o_gpu: torch.Tensor, lse_gpu, q, k, v, scale, causal, rows=None, label="",
          window=None, alibi_slopes=None):
    """Compare GPU O ([B, H, N, d]) and LSE ([B, H, N]) with the oracle on the
    given query rows (all rows when ``rows`` is None).  With ``window`` or
    ``alibi_slopes`` the reference is the masked oracle.  Returns an error dict."""
    if window is None and alibi_slopes is None:
        O_ref, L_ref = oracle.attention(q, k, v, scale=scale, causal=causal, rows=rows)
    else:
        O_ref, L_ref = oracle.attention_masked(
            q, k, v, scale=scale, causal=causal, rows=rows,
            window=(-1, -1) if window is None else window,
            alibi_slopes=None if alibi_slopes is None else np.asarray(alibi_slopes, np.float64))
    o = to_f64(o_gpu if rows is None else o_gpu[:, :, torch.as_tensor(rows, dtype=torch.long)])
    lg = None
    if lse_gpu is not None:
        lg = to_f64(lse_gpu if rows is None else
                    lse_gpu[:, :, torch.as_tensor(rows, dtype=torch.long)])
    return compare(o, o_gpu.dtype, lg, O_ref, L_ref, label)


def compare(o, dtype, lg, O_ref, L_ref, label=""):
    """Element-wise comparison of fp64 copies of the GPU output ``o`` (and LSE
    ``lg`` or None) with the oracle's ``O_ref`` / ``L_ref``."""
    err = np.abs(o - O_ref)
    res = {"o_max_abs": float(err.max()), "o_mean_abs": float(err.mean())}
    # error floor: the oracle rounded once to the output dtype
    floor = np.abs(to_f64(torch.from_numpy(O_ref).to(dtype)) - O_ref)
    res["floor_max_abs"] = float(floor.max())
    res["floor_mean_abs"] = float(floor.mean())
    if lg is not None:
        lerr = np.abs(lg - L_ref) / np.maximum(1.0, np.abs(L_ref))
        res["lse_rel"] = float(lerr.max())
    ok = (np.isfinite(o).all() and res["o_max_abs"] <= O_MAX_ABS
          and res["o_mean_abs"] <= O_MEAN_ABS
          and (lg is None or res["lse_rel"] <= LSE_REL))
    assert ok, f"{label} parity failed: {res}"
    return res
