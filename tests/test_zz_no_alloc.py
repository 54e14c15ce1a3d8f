"""The allocation-free tensor-product backward against the workspace one and
against the oracle.

cgtp_tp_backward_noalloc serves callers that cannot allocate device memory
when they call the library (a framework that owns all device memory through
its own allocator, or a time-stepping loop that must not allocate after
set-up): its grad_w partial sums live in a fixed array inside the library
instead of a caller workspace.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import tp as otp
from tests.gpu_common import GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _noalloc(api, plan, x, y, w, gz, want_w=True):
    import torch
    from equivariant_mlip_tensor_b200._lib import lib
    gx, gy = torch.empty_like(x), torch.empty_like(y)
    gw = torch.empty_like(w) if want_w else None
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib().cgtp_tp_backward_noalloc(plan.handle("pair"), x.shape[0], p(x), p(y), p(w), p(gz), p(gx), p(gy), p(gw),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    return gx, gy, gw


def test_noalloc_matches_workspace_entry_point_on_two_calls(api):
    wl = synthetic.tp_batch()
    L = (wl.lmax_in, wl.lmax_sh, wl.lmax_out)
    plan = api.Plan(*L, wl.mult)
    rng = np.random.default_rng(90)
    inputs = [(wl.x, wl.y, wl.w, wl.grad_z),
              tuple(rng.standard_normal(a.shape).astype(np.float32) for a in (wl.x, wl.y, wl.w, wl.grad_z))]
    for x, y, w, gz in inputs:  # two calls in a row share (and overwrite) the built-in scratch
        xd, yd, wd, gzd = cuda(x), cuda(y), cuda(w), cuda(gz)
        ref = plan.tp_backward(xd, yd, wd, gzd)
        got = _noalloc(api, plan, xd, yd, wd, gzd)
        for g, r in zip(got, ref):
            assert rel_err(host(g), host(r)) <= GRAD_TOL


def test_noalloc_matches_the_oracle_with_and_without_grad_w(api):
    wl = synthetic.tp_batch(seed=11, batch=203, mult=64)  # ragged against the 8-pair chunks
    L = (wl.lmax_in, wl.lmax_sh, wl.lmax_out)
    plan = api.Plan(*L, wl.mult)
    ox, oy, ow = otp.tp_backward(wl.x, wl.y, wl.w, wl.grad_z, *L)
    xd, yd, wd, gzd = cuda(wl.x), cuda(wl.y), cuda(wl.w), cuda(wl.grad_z)
    gx, gy, gw = _noalloc(api, plan, xd, yd, wd, gzd)
    assert rel_err(host(gx), ox) <= GRAD_TOL
    assert rel_err(host(gy), oy) <= GRAD_TOL
    assert rel_err(host(gw), ow) <= GRAD_TOL
    # without grad_w the scratch is not touched; the input gradients are unchanged
    gx2, gy2, none = _noalloc(api, plan, xd, yd, wd, gzd, want_w=False)
    assert none is None
    assert rel_err(host(gx2), ox) <= GRAD_TOL
    assert rel_err(host(gy2), oy) <= GRAD_TOL


def test_noalloc_rejects_requests_beyond_its_scratch(api):
    from equivariant_mlip_tensor_b200._lib import lib
    plan = api.Plan(3, 3, 3, 256)  # 64 chunks x 34 paths x 256 channels > 2 MiB of floats
    import torch
    B = 1024
    x = torch.zeros((B, 16, 256), device="cuda")
    w = torch.zeros((34, 256), device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib().cgtp_tp_backward_noalloc(plan.handle("pair"), B, p(x), p(x), p(w), p(x), None, None, p(w), None)
    assert st == 7  # CGTP_ERR_WORKSPACE
