"""Budget constants from data: the log-linear fit ln k = a*H + b over the
(entropy, retained count) pairs that tra_calibrate_topk returns.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2, Intuition I: the number of keys a query needs grows as
tau * exp(H_i); the fit generalises the slope to a.  The fitted (a, b) go
straight into tra_plan_create, whose budget is exp(a*H + b).

The fit itself is the library's tra_calibrate_fit (host code behind the C
ABI); this module only copies the pairs to contiguous host buffers.
"""
from __future__ import annotations

import torch

from . import tra_calibrate_fit


def fit_log_linear(H, k) -> tuple[float, float]:
    """(a, b) of ln k = a*H + b over the rows with k >= 1 and a finite H.
    H, k: tensors or arrays of any shape (device tensors are copied to the
    host).  Raises TraError if fewer than two usable rows remain."""
    Hh = torch.as_tensor(H).detach().to("cpu", torch.float32).contiguous().reshape(-1)
    kh = torch.as_tensor(k).detach().to("cpu", torch.int32).contiguous().reshape(-1)
    if Hh.numel() != kh.numel():
        raise ValueError("H and k need the same number of rows")
    a, b, _ = tra_calibrate_fit(Hh.data_ptr(), kh.data_ptr(), Hh.numel())
    return a, b
