"""Budget constants from data: the log-linear fit ln k = a*H + b over the
(entropy, retained count) pairs that tra_calibrate_topk returns.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2, Intuition I: the number of keys a query needs grows as
tau * exp(H_i); the fit generalises the slope to a.  The fitted (a, b) go
straight into tra_plan_create, whose budget is exp(a*H + b).
"""
from __future__ import annotations

import numpy as np


def fit_log_linear(H, k) -> tuple[float, float]:
    """Least-squares (a, b) of ln k = a*H + b over the valid rows (k >= 1,
    finite H).  Returns floats; raises if fewer than two valid rows."""
    H = np.asarray(H, dtype=np.float64).reshape(-1)
    k = np.asarray(k, dtype=np.float64).reshape(-1)
    ok = (k >= 1) & np.isfinite(H)
    if ok.sum() < 2:
        raise ValueError("need at least two valid (H, k) pairs")
    A = np.stack([H[ok], np.ones(int(ok.sum()))], axis=1)
    (a, b), *_ = np.linalg.lstsq(A, np.log(k[ok]), rcond=None)
    return float(a), float(b)
