"""Pins of the oracle's second derivatives: the harmonic Hessian and the
adjoint of the convolution backward (double backward).

The Hessian is pinned by identities that hold for any correct second
derivative of the real harmonics of a direction: symmetry, Euler's identity
for a function homogeneous of degree 0 (sum_k r_k d2Y/dr_j dr_k = -dY/dr_j),
the sphere's Laplacian eigenvalue (the Cartesian Laplacian of Y(r/|r|) is
-l(l+1) Y / |r|^2), and central differences of the complex-step Jacobian.
The double backward is pinned by central differences of the oracle's own
first backward (itself pinned in test_oracle_conv), one input and one
cotangent at a time, so that a dropped or mis-signed term fails by itself.
"""
import numpy as np
import pytest

from oracle import cg as ocg
from oracle import conv as oconv
from oracle import graph as ograph
from oracle import sh as osh


def _vectors(seed, n=7):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((n, 3)) * rng.uniform(0.3, 3.0, size=(n, 1))
    return v


@pytest.mark.parametrize("lmax", [1, 2, 4])
def test_hessian_symmetric_and_euler_identity(lmax):
    v = _vectors(1)
    H = osh.real_sh_hessian(v, lmax)
    J = osh.real_sh_jacobian(v, lmax)
    scale = np.abs(H).max()
    assert np.abs(H - np.swapaxes(H, -1, -2)).max() < 1e-12 * scale
    assert np.abs(np.einsum("ek,ebjk->ebj", v, H) + J).max() < 1e-12 * scale


def test_hessian_laplacian_is_sphere_eigenvalue():
    v = _vectors(2)
    lmax = 4
    H = osh.real_sh_hessian(v, lmax)
    Y = osh.real_sh(v, lmax)
    ls = np.concatenate([[l] * (2 * l + 1) for l in range(lmax + 1)])
    r2 = np.sum(v * v, axis=1)
    lap = np.trace(H, axis1=-2, axis2=-1)
    assert np.abs(lap + ls * (ls + 1) * Y / r2[:, None]).max() < 1e-11 * np.abs(lap).max()


def test_hessian_l1_closed_form():
    # Y_1 = sqrt(3) (y, z, x) / r:  d2(r_a / r)/dr_j dr_k = (3 r_a r_j r_k / r^2 - r_a d_jk - r_j d_ak - r_k d_aj) / r^3
    v = _vectors(3)
    H = osh.real_sh_hessian(v, 1)[:, 1:4]
    r = np.linalg.norm(v, axis=1)
    I = np.eye(3)
    for b, a in enumerate((1, 2, 0)):
        ref = (3 * v[:, a, None, None] * v[:, :, None] * v[:, None, :] / r[:, None, None] ** 2
               - v[:, a, None, None] * I - v[:, :, None] * I[a][None, None, :] - I[a][None, :, None] * v[:, None, :])
        ref = np.sqrt(3) * ref / r[:, None, None] ** 3
        assert np.abs(H[:, b] - ref).max() < 1e-12 * np.abs(ref).max()


def test_hessian_matches_differences_of_jacobian():
    v = _vectors(4)
    d = np.random.default_rng(5).standard_normal(3)
    h = 1e-5
    Hd = (osh.real_sh_jacobian(v + h * d, 4) - osh.real_sh_jacobian(v - h * d, 4)) / (2 * h)
    H = osh.real_sh_hessian(v, 4)
    assert np.abs(np.einsum("ebjk,k->ebj", H, d) - Hd).max() < 1e-7 * np.abs(Hd).max()


def test_hessian_of_zero_vector_is_zero():
    H = osh.real_sh_hessian(np.zeros((2, 3)), 3)
    assert not np.any(H)


def _problem(seed, L, u=3, n=9):
    rng = np.random.default_rng(seed)
    pos = rng.random((n, 3)) * 4.0
    o = ograph.neighbour_list(pos, 3.0)
    E, P = o["col"].size, len(ocg.paths(*L))
    ni, no = (L[0] + 1) ** 2, (L[2] + 1) ** 2
    d = dict(rp=o["row_ptr"], col=o["col"], ev=o["edge_vec"].astype(np.float64),
             x=rng.standard_normal((n, ni, u)), W=rng.standard_normal((E, P, u)),
             g=rng.standard_normal((n, no, u)),
             ggx=rng.standard_normal((n, ni, u)), ggw=rng.standard_normal((E, P, u)),
             ggr=rng.standard_normal((E, 3)))
    return d


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 2, 2), (1, 2, 1)])
@pytest.mark.parametrize("cot", ["ggx", "ggw", "ggr"])
def test_double_backward_matches_differences_of_backward(L, cot):
    d = _problem(10 + len(cot), L)
    cots = {k: (d[k] if k == cot else None) for k in ("ggx", "ggw", "ggr")}

    def objective(x, W, g, ev):
        gx, gw, gr = oconv.conv_backward(d["rp"], d["col"], ev, x, W, g, *L)
        return sum(float(np.sum(c * o)) for c, o in ((cots["ggx"], gx), (cots["ggw"], gw), (cots["ggr"], gr))
                   if c is not None)

    grads = oconv.conv_double_backward(d["rp"], d["col"], d["ev"], d["x"], d["W"], d["g"],
                                       cots["ggx"], cots["ggw"], cots["ggr"], *L)
    rng = np.random.default_rng(99)
    h = 1e-6
    for key, grad in zip(("x", "W", "g", "ev"), grads):
        direction = rng.standard_normal(d[key].shape)
        plus = {k: d[k] for k in ("x", "W", "g", "ev")}
        minus = dict(plus)
        plus[key] = d[key] + h * direction
        minus[key] = d[key] - h * direction
        fd = (objective(**plus) - objective(**minus)) / (2 * h)
        an = float(np.sum(grad * direction))
        scale = np.linalg.norm(grad) * np.linalg.norm(direction) + 1e-300
        assert abs(fd - an) <= 1e-7 * scale, (key, fd, an)


def test_double_backward_is_linear_in_the_cotangents():
    L = (2, 2, 2)
    d = _problem(20, L)
    args = (d["rp"], d["col"], d["ev"], d["x"], d["W"], d["g"])
    whole = oconv.conv_double_backward(*args, d["ggx"], d["ggw"], d["ggr"], *L)
    parts = [oconv.conv_double_backward(*args, d["ggx"], None, None, *L),
             oconv.conv_double_backward(*args, None, d["ggw"], None, *L),
             oconv.conv_double_backward(*args, None, None, d["ggr"], *L)]
    for k in range(4):
        s = parts[0][k] + parts[1][k] + parts[2][k]
        assert np.abs(whole[k] - s).max() <= 1e-12 * max(np.abs(whole[k]).max(), 1.0)
    zero = oconv.conv_double_backward(*args, None, None, None, *L)
    assert all(not np.any(z) for z in zero)
