"""Pins for the oracle's real harmonics and Wigner-D matrices (CPU only)."""
import math

import numpy as np
import pytest

from oracle import cg, sh
from oracle.wigner import (random_rotation, rotation_zyz, wigner_d_fit, wigner_d_real)

LMAX = 4


def _dirs(n=64, seed=0):
    return np.random.default_rng(seed).normal(size=(n, 3))


def test_against_scipy_through_real_basis():
    ss = pytest.importorskip("scipy.special")
    v = _dirs()
    u = v / np.linalg.norm(v, axis=1)[:, None]
    th, ph = np.arccos(u[:, 2]), np.arctan2(u[:, 1], u[:, 0])
    Y = sh.real_sh(v, LMAX)
    for l in range(LMAX + 1):
        Yc = np.stack([ss.sph_harm_y(l, m, th, ph) for m in range(-l, l + 1)], axis=-1)
        Yr = math.sqrt(4 * math.pi) * (Yc @ cg.real_basis_q(l).T)
        assert np.abs(Yr.imag).max() < 1e-13
        assert np.allclose(Yr.real, Y[:, l * l:(l + 1) ** 2], atol=1e-13)


def test_legendre_recurrence_route_agrees():
    v = _dirs(seed=1)
    assert np.allclose(sh.real_sh(v, LMAX), sh.real_sh_legendre(v, LMAX), atol=1e-13)


def test_low_degree_closed_forms():
    v = _dirs(seed=2)
    u = v / np.linalg.norm(v, axis=1)[:, None]
    Y = sh.real_sh(v, 2)
    assert np.allclose(Y[:, 0], 1.0)
    assert np.allclose(Y[:, 1:4], math.sqrt(3) * u[:, [1, 2, 0]], atol=1e-15)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    s15 = math.sqrt(15)
    want2 = np.stack([s15 * x * y, s15 * y * z, math.sqrt(5) / 2 * (3 * z * z - 1),
                      s15 * x * z, s15 / 2 * (x * x - y * y)], axis=1)
    assert np.allclose(Y[:, 4:9], want2, atol=1e-14)


def test_addition_theorem_and_norm():
    a, b = _dirs(seed=3), _dirs(seed=4)
    Ya, Yb = sh.real_sh(a, LMAX), sh.real_sh(b, LMAX)
    ua = a / np.linalg.norm(a, axis=1)[:, None]
    ub = b / np.linalg.norm(b, axis=1)[:, None]
    c = np.sum(ua * ub, axis=1)
    for l in range(LMAX + 1):
        sl = slice(l * l, (l + 1) ** 2)
        Pl = np.polynomial.legendre.legval(c, [0] * l + [1])
        assert np.allclose(np.sum(Ya[:, sl] * Yb[:, sl], axis=1), (2 * l + 1) * Pl, atol=1e-12)
        assert np.allclose(np.sum(Ya[:, sl] ** 2, axis=1), 2 * l + 1, atol=1e-12)


def test_parity_and_scale_invariance():
    v = _dirs(seed=5)
    Y = sh.real_sh(v, LMAX)
    Ym = sh.real_sh(-v, LMAX)
    for l in range(LMAX + 1):
        sl = slice(l * l, (l + 1) ** 2)
        assert np.allclose(Ym[:, sl], (-1) ** l * Y[:, sl], atol=1e-14)
    assert np.allclose(sh.real_sh(3.7 * v, LMAX), Y, atol=1e-14)


def test_jacobian_complex_step_vs_central_differences():
    v = _dirs(16, seed=6)
    J = sh.real_sh_jacobian(v, LMAX)
    h = 1e-6
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        fd = (sh.real_sh(v + e, LMAX) - sh.real_sh(v - e, LMAX)) / (2 * h)
        assert np.allclose(J[..., k], fd, atol=1e-7)
    # the harmonics depend on direction only: no derivative along r
    assert np.allclose(np.einsum("ebk,ek->eb", J, v), 0.0, atol=1e-12)


def test_zero_vector_convention():
    Y = sh.real_sh(np.zeros((2, 3)), LMAX)
    assert np.all(Y[:, 0] == 1.0) and np.all(Y[:, 1:] == 0.0)
    assert np.all(sh.real_sh_jacobian(np.zeros((1, 3)), LMAX) == 0.0)


def test_wigner_rotates_harmonics():
    rng = np.random.default_rng(8)
    u = _dirs(32, seed=9)
    for _ in range(4):
        R = random_rotation(rng)
        for l in range(LMAX + 1):
            sl = slice(l * l, (l + 1) ** 2)
            D = wigner_d_real(l, R)
            assert np.allclose(sh.real_sh(u @ R.T, LMAX)[:, sl], sh.real_sh(u, LMAX)[:, sl] @ D.T,
                               atol=1e-12)
            assert np.allclose(D, wigner_d_fit(l, R), atol=1e-12)
            assert np.allclose(D @ D.T, np.eye(2 * l + 1), atol=1e-12)


def test_wigner_homomorphism_and_z_rotation_closed_form():
    rng = np.random.default_rng(10)
    R1, R2 = random_rotation(rng), random_rotation(rng)
    for l in range(LMAX + 1):
        assert np.allclose(wigner_d_real(l, R1 @ R2), wigner_d_real(l, R1) @ wigner_d_real(l, R2),
                           atol=1e-12)
    # rotation about z by t mixes (m, -m) as a plane rotation by m t
    t = 0.7
    R = rotation_zyz(t, 0.0, 0.0)
    for l in range(LMAX + 1):
        D = wigner_d_real(l, R)
        want = np.zeros((2 * l + 1, 2 * l + 1))
        want[l, l] = 1.0
        for m in range(1, l + 1):
            c, s = math.cos(m * t), math.sin(m * t)
            want[l + m, l + m] = c
            want[l - m, l - m] = c
            want[l + m, l - m] = -s
            want[l - m, l + m] = s
        assert np.allclose(D, want, atol=1e-13)
