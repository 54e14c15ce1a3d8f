"""Shared helpers for the GPU parity tests (no oracle arithmetic here)."""
import os

import numpy as np

FWD_TOL = 1e-5   # max|gpu - oracle| / max|oracle| for forward outputs
GRAD_TOL = 1e-4  # same measure for gradients and forces
THREADS = max(1, len(os.sched_getaffinity(0)))


def rel_err(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return 0.0
    scale = np.max(np.abs(want))
    diff = np.max(np.abs(got - want))
    if scale == 0.0:
        return diff
    return diff / scale


def cuda(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()
