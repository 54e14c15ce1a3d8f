"""Pins of the oracle's CP-decomposed tensor product: factors that spell out
the exact tensor reproduce the oracle's exact edge-free product, the dot-product
path's closed form in the dense tensor, the adjoints against Euler's identity
for a map linear in each argument and against central differences, and the
batch least-squares fit against exactly representable tensors, the
Eckart-Young bound of a matrix-shaped tensor, the expected N(0,1) batch
loss = squared Frobenius distance, and the equivariance error (zero for the
exact factorisation, shrinking with the fit's error)."""
import numpy as np
import pytest

from oracle import cg as ocg
from oracle import cp
from oracle import tp


def _exact_factors(L):
    """A rank-d1*d2 decomposition that is exact by construction: one component
    per input pair (i, j), with B = e_i, C = e_j and A = M[:, i, j]."""
    M = cp.exact_tensor(*L)
    d3, d1, d2 = M.shape
    A = M.reshape(d3, d1 * d2)
    B = np.repeat(np.eye(d1), d2, axis=1)
    C = np.tile(np.eye(d2), (1, d1))
    return A, B, C


@pytest.mark.parametrize("L", [(1, 1, 1), (1, 2, 1), (2, 2, 2)])
def test_exact_factors_reproduce_the_tensor_product(L):
    A, B, C = _exact_factors(L)
    d1, d2, d3 = cp.dims(*L)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, d1, 3))
    y = rng.standard_normal((5, d2, 3))
    w = np.ones((len(ocg.paths(*L)), 3))
    want = tp.tp_forward(x, y, w, *L)
    got = cp.cp_forward(A, B, C, x, y)
    assert np.abs(got - want).max() <= 1e-13 * np.abs(want).max()
    assert cp.rel_error(A, B, C, *L) <= 1e-15


def test_dot_product_path_closed_form():
    # (1,1,0): the l = 0 output is 1*x0 y0 + c (x . y) over the three l = 1 rows,
    # c = +-1/sqrt(3) (the 1 x 1 -> 0 coupling is proportional to the dot product)
    M = cp.exact_tensor(1, 1, 0)
    assert M.shape == (1, 4, 4)
    assert M[0, 0, 0] == pytest.approx(1.0)
    c = M[0, 1, 1]
    assert abs(abs(c) - 1 / np.sqrt(3)) <= 1e-14
    assert np.allclose(M[0], np.diag([1.0, c, c, c]), atol=1e-15)


def _random_problem(L, R, seed, batch=4, u=3):
    d1, d2, d3 = cp.dims(*L)
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((d3, R))
    B = rng.standard_normal((d1, R))
    C = rng.standard_normal((d2, R))
    x = rng.standard_normal((batch, d1, u))
    y = rng.standard_normal((batch, d2, u))
    g = rng.standard_normal((batch, d3, u))
    return A, B, C, x, y, g


@pytest.mark.parametrize("L,R", [((1, 1, 1), 5), ((2, 4, 2), 7)])
def test_backward_euler_identities(L, R):
    A, B, C, x, y, g = _random_problem(L, R, 3)
    z = cp.cp_forward(A, B, C, x, y)
    gz_z = float(np.sum(g * z))
    for v, gv in zip((x, y, A, B, C), cp.cp_backward(A, B, C, x, y, g)):
        assert gv.shape == v.shape
        # z is linear in each argument, so <dL/dv, v> = <g, z>
        assert abs(float(np.sum(gv * v)) - gz_z) <= 1e-11 * max(1.0, abs(gz_z))


@pytest.mark.parametrize("L,R", [((1, 1, 1), 5), ((2, 2, 2), 9)])
def test_backward_central_differences(L, R):
    A, B, C, x, y, g = _random_problem(L, R, 4)
    args = dict(A=A, B=B, C=C, x=x, y=y)
    grads = dict(zip(("x", "y", "A", "B", "C"), cp.cp_backward(A, B, C, x, y, g)))
    f = lambda a: float(np.sum(g * cp.cp_forward(a["A"], a["B"], a["C"], a["x"], a["y"])))
    rng = np.random.default_rng(5)
    h = 1e-6
    for key in ("x", "y", "A", "B", "C"):
        d = rng.standard_normal(args[key].shape)
        p, m = dict(args), dict(args)
        p[key] = args[key] + h * d
        m[key] = args[key] - h * d
        fd = (f(p) - f(m)) / (2 * h)
        an = float(np.sum(grads[key] * d))
        assert abs(fd - an) <= 1e-7 * np.linalg.norm(grads[key]) * np.linalg.norm(d), key


@pytest.mark.parametrize("L,R", [((0, 0, 0), 1), ((1, 1, 0), 4)])
def test_fit_is_exact_when_the_rank_suffices(L, R):
    A, B, C = cp.fit_als(*L, R, np.random.default_rng(6))
    assert cp.rel_error(A, B, C, *L) <= 1e-8


def test_fit_respects_the_eckart_young_bound():
    # (1,1,0) is a 4 x 4 matrix with singular values 1, 1/sqrt(3) (three times):
    # no rank-3 map gets closer than (1/sqrt(3)) / sqrt(1 + 3/3) = 0.40825
    A, B, C = cp.fit_als(1, 1, 0, 3, np.random.default_rng(7))
    err = cp.rel_error(A, B, C, 1, 1, 0)
    assert err >= np.sqrt(1 / 3) / np.sqrt(2) - 1e-9
    assert err <= 0.5


def test_error_curve_reaches_zero():
    L = (1, 1, 1)
    errs = [cp.rel_error(*cp.fit_als(*L, R, np.random.default_rng(8)), *L) for R in (3, 8, 16)]
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] <= 1e-8  # rank d1 * d2 = 16 always suffices


def test_batch_loss_estimates_the_frobenius_distance():
    L, R = (1, 1, 1), 5
    A, B, C, _, _, _ = _random_problem(L, R, 9)
    M = cp.exact_tensor(*L)
    frob2 = float(np.sum((M - cp.cp_tensor(A, B, C)) ** 2))
    est = cp.batch_loss(A, B, C, *L, np.random.default_rng(10), 40000)
    assert abs(est - frob2) <= 0.03 * frob2


def test_equivariance_error_of_exact_and_fitted_factors():
    """The exact factorisation is equivariant to rounding; random factors are
    not; a fit's equivariance error shrinks with its Frobenius error (both vanish
    together), here at (1,1,1) ranks 6 and 10."""
    L = (1, 1, 1)
    rng = np.random.default_rng(20)
    assert cp.equivariance_error(*_exact_factors(L), *L, rng) <= 1e-13
    A, B, C, _, _, _ = _random_problem(L, 6, 21)
    assert cp.equivariance_error(A, B, C, *L, rng) > 0.1
    e6 = cp.equivariance_error(*cp.fit_als(*L, 6, np.random.default_rng(22)), *L, rng)
    f10 = cp.fit_als(*L, 10, np.random.default_rng(23))
    e10 = cp.equivariance_error(*f10, *L, rng)
    assert e10 < e6
    assert e10 <= 4 * cp.rel_error(*f10, *L) + 1e-12
