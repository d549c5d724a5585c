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


def check(o_gpu: torch.Tensor, lse_gpu, q, k, v, scale, causal, rows=None, label=""):
    """Compare GPU O ([B, H, N, d]) and LSE ([B, H, N]) with the oracle on the
    given query rows (all rows when ``rows`` is None).  Returns an error dict."""
    O_ref, L_ref = oracle.attention(q, k, v, scale=scale, causal=causal, rows=rows)
    o = to_f64(o_gpu if rows is None else o_gpu[:, :, torch.as_tensor(rows, dtype=torch.long)])
    err = np.abs(o - O_ref)
    res = {"o_max_abs": float(err.max()), "o_mean_abs": float(err.mean())}
    # error floor: the oracle rounded once to the output dtype
    floor = np.abs(to_f64(torch.from_numpy(O_ref).to(o_gpu.dtype)) - O_ref)
    res["floor_max_abs"] = float(floor.max())
    res["floor_mean_abs"] = float(floor.mean())
    if lse_gpu is not None:
        lg = to_f64(lse_gpu if rows is None else lse_gpu[:, :, torch.as_tensor(rows, dtype=torch.long)])
        lerr = np.abs(lg - L_ref) / np.maximum(1.0, np.abs(L_ref))
        res["lse_rel"] = float(lerr.max())
    ok = (np.isfinite(o).all() and res["o_max_abs"] <= O_MAX_ABS
          and res["o_mean_abs"] <= O_MEAN_ABS
          and (lse_gpu is None or res["lse_rel"] <= LSE_REL))
    assert ok, f"{label} parity failed: {res}"
    return res
