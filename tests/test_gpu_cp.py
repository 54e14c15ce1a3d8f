"""GPU parity of the CP-decomposed tensor product against the oracle's dense
formula: forward and every gradient (inputs and factors) at several shapes,
ranks, batches and multiplicities (ragged against the 64- and 128-item
blocks), factors fitted by the oracle's least-squares fit, the exact
factorisation against the exact edge-free product, nullable outputs, an empty
batch, and the host-side errors."""
import ctypes

import numpy as np
import pytest

from oracle import cg as ocg
from oracle import cp as ocp
from oracle import tp as otp
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _problem(L, R, batch, mult, seed):
    d1, d2, d3 = ocp.dims(*L)
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return f(d3, R) / np.float32(np.sqrt(R)), f(d1, R), f(d2, R), f(batch, d1, mult), f(batch, d2, mult), \
        f(batch, d3, mult)


@pytest.mark.parametrize("L,R,batch,mult", [((1, 1, 1), 1, 3, 8), ((1, 1, 1), 16, 37, 8), ((2, 2, 2), 40, 100, 128),
                                            ((2, 2, 2), 7, 5, 32), ((1, 2, 1), 20, 33, 16),
                                            ((2, 4, 2), 64, 50, 128), ((3, 3, 3), 96, 21, 64)])
def test_matches_oracle(api, L, R, batch, mult):
    A, B, C, x, y, g = _problem(L, R, batch, mult, 10 * R + batch)
    plan = api.Plan(*L, mult)
    z = plan.cp_forward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y))
    assert rel_err(host(z), ocp.cp_forward(A, B, C, x, y)) <= FWD_TOL
    got = plan.cp_backward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y), cuda(g))
    want = ocp.cp_backward(A, B, C, x, y, g)
    for name, a, b in zip(("grad_x", "grad_y", "grad_A", "grad_B", "grad_C"), got, want):
        assert a.shape == b.shape, name
        assert rel_err(host(a), b) <= GRAD_TOL, (name, rel_err(host(a), b))


def test_fitted_factors_at_the_timed_shape(api):
    """Factors from the oracle's batch least-squares fit at (2,2,2), rank 40:
    the GPU forward follows the dense formula, and both stay close to the exact
    product (the fit's error)."""
    L, R, mult = (2, 2, 2), 40, 128
    A, B, C = (v.astype(np.float32) for v in ocp.fit_als(*L, R, np.random.default_rng(11), n_iter=12))
    err = ocp.rel_error(A, B, C, *L)
    assert err < 0.05
    rng = np.random.default_rng(12)
    x = rng.standard_normal((64, 9, mult)).astype(np.float32)
    y = rng.standard_normal((64, 9, mult)).astype(np.float32)
    plan = api.Plan(*L, mult)
    z = host(plan.cp_forward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y)))
    assert rel_err(z, ocp.cp_forward(A, B, C, x, y)) <= FWD_TOL
    exact = otp.tp_forward(x, y, np.ones((len(ocg.paths(*L)), mult)), *L)
    assert rel_err(z, exact) <= 4 * err


def test_exact_factorisation_is_the_tensor_product(api):
    L, mult = (1, 2, 1), 32
    M = ocp.exact_tensor(*L)
    d3, d1, d2 = M.shape
    A = M.reshape(d3, d1 * d2).astype(np.float32)
    B = np.repeat(np.eye(d1), d2, axis=1).astype(np.float32)
    C = np.tile(np.eye(d2), (1, d1)).astype(np.float32)
    rng = np.random.default_rng(13)
    x = rng.standard_normal((20, d1, mult)).astype(np.float32)
    y = rng.standard_normal((20, d2, mult)).astype(np.float32)
    plan = api.Plan(*L, mult)
    z = host(plan.cp_forward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y)))
    exact = otp.tp_forward(x, y, np.ones((len(ocg.paths(*L)), mult)), *L)
    assert rel_err(z, exact) <= FWD_TOL


def test_nullable_outputs(api):
    L, R, batch, mult = (2, 2, 2), 12, 9, 32
    A, B, C, x, y, g = _problem(L, R, batch, mult, 14)
    plan = api.Plan(*L, mult)
    args = (cuda(A), cuda(B), cuda(C), cuda(x), cuda(y), cuda(g))
    full = plan.cp_backward(*args)
    gx, gy, gA, gB, gC = plan.cp_backward(*args, want_x=False, want_y=False)
    assert gx is None and gy is None
    for a, b in zip((gA, gB, gC), full[2:]):
        assert np.array_equal(host(a), host(b))  # same blocks, same order: bitwise
    gx, gy, gA, gB, gC = plan.cp_backward(*args, want_factors=False)
    assert gA is None and gB is None and gC is None
    assert np.array_equal(host(gx), host(full[0]))
    assert np.array_equal(host(gy), host(full[1]))


def test_empty_batch(api):
    L, R, mult = (1, 1, 1), 5, 8
    A, B, C, x, y, g = _problem(L, R, 0, mult, 15)
    plan = api.Plan(*L, mult)
    z = plan.cp_forward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y))
    assert z.shape == (0, 4, mult)
    gx, gy, gA, gB, gC = plan.cp_backward(cuda(A), cuda(B), cuda(C), cuda(x), cuda(y), cuda(g))
    for a in (gA, gB, gC):
        assert not np.any(host(a))


def test_host_errors(api):
    import torch
    from equivariant_mlip_tensor_b200._lib import lib
    L, R, batch, mult = (1, 1, 1), 4, 6, 8
    A, B, C, x, y, g = _problem(L, R, batch, mult, 16)
    plan = api.Plan(*L, mult)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    Ad, Bd, Cd, xd, yd, gd = (cuda(v) for v in (A, B, C, x, y, g))
    z = torch.empty((batch, 4, mult), device="cuda")
    f = lib().cgtp_cp_forward
    assert f(plan.handle("pair"), 0, batch, p(Ad), p(Bd), p(Cd), p(xd), p(yd), p(z), None) == 1      # rank < 1
    assert f(plan.handle("pair"), R, -1, p(Ad), p(Bd), p(Cd), p(xd), p(yd), p(z), None) == 1     # negative batch
    assert f(plan.handle("pair"), R, batch, None, p(Bd), p(Cd), p(xd), p(yd), p(z), None) == 1   # missing factor
    assert f(plan.handle("pair"), 100000, batch, p(Ad), p(Bd), p(Cd), p(xd), p(yd), p(z), None) == 2  # factors exceed smem
    gA = torch.empty_like(Ad)
    nb = plan.cp_backward_workspace_bytes(R, batch)
    ws = torch.empty(nb // 4 + 64, device="cuda")
    b = lib().cgtp_cp_backward
    args = (plan.handle("pair"), R, batch, p(Ad), p(Bd), p(Cd), p(xd), p(yd), p(gd), None, None, p(gA), None, None)
    assert b(*args, None, 0, None) == 7              # factor gradient without workspace
    assert b(*args, p(ws), nb - 256, None) == 7      # workspace too small
    assert b(*args, p(ws), nb, None) == 0
    assert f(plan.handle("pair"), R, batch, p(Ad), p(Bd), p(Cd), p(xd), p(yd), p(z), None) == 0
