"""Helpers for the GPU parity tests: device upload and error metrics.
No method arithmetic lives here."""

import numpy as np
import torch

# Tolerances of the parity bar: bf16 outputs against the float64 oracle
# (max-abs and relative L2), fp32 outputs, and the natural-log LSE.
TOL = {
    "bf16": dict(max_abs=2e-2, rel_l2=5e-3, lse_abs=1e-3),
    "f32": dict(max_abs=1e-4, rel_l2=1e-5, lse_abs=1e-4),
}
NEAR_TIE_REL = 1e-3


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float32)
    return t.cuda()


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def mask_of(idx, cnt, nk):
    """Dense boolean [..., nk] kept-block mask from (idx, cnt) lists."""
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    m = np.zeros(cnt.shape + (nk,), dtype=bool)
    for pos in np.ndindex(cnt.shape):
        m[pos][idx[pos][: cnt[pos]]] = True
    return m
