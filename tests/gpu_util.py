"""Shared helpers of the GPU parity tests (no attention arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the parity bar, per output tensor, both must hold:
#   normwise  ||x - ref||_2 / ||ref||_2
#   max-abs   max|x - ref| / max|ref|
TOL = {torch.bfloat16: (1e-2, 2e-2), torch.float32: (1e-4, 1e-4)}


def errors(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0, 0.0
    dn = float(np.linalg.norm(ref.ravel()))
    dm = float(np.max(np.abs(ref)))
    nrm = float(np.linalg.norm((x - ref).ravel())) / (dn if dn > 0 else 1.0)
    mx = float(np.max(np.abs(x - ref))) / (dm if dm > 0 else 1.0)
    return nrm, mx


def check(name, got, ref, dtype):
    """Assert the parity bar for one output; `got` may be a torch tensor."""
    if isinstance(got, torch.Tensor):
        got = got.detach().float().cpu().numpy()
    tn, tm = TOL[dtype]
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    nrm, mx = errors(got, ref)
    assert nrm <= tn and mx <= tm, (
        f"{name}: normwise {nrm:.3e} (tol {tn:.0e}), max {mx:.3e} (tol {tm:.0e})")
    return nrm, mx


def host(t):
    return t.detach().float().cpu().numpy()
