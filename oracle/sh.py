"""Real spherical harmonics of edge directions and their Cartesian Jacobian.

Test infrastructure only (see ``oracle/__init__``).

The convolution combines neighbour features with the spherical harmonics of
the edge direction ("LunaTP: Enabling Efficient and Scalable Tensor Product
for Equivariant MLIPs", abstract: CGTP convolutions).  The pages fix no
convention, so the plainest one is used:

* component normalisation: sum_m Y_lm(u)^2 = 2l + 1 and Y_00 = 1;
* the real basis of ``oracle.cg.real_basis_q`` (Condon-Shortley complex
  harmonics), which gives Y_1 = sqrt(3) (y, z, x) with positive signs;
* for a unit vector u = (x, y, z):
      Y_l0  = sqrt(2l+1) P_l(z)
      Y_lm  = sqrt(2(2l+1)(l-m)!/(l+m)!) (d^m P_l/dz^m)(z) Re[(x+iy)^m]   (m>0)
      Y_l-m = sqrt(2(2l+1)(l-m)!/(l+m)!) (d^m P_l/dz^m)(z) Im[(x+iy)^m]   (m>0)
  with P_l from the explicit binomial sum and Re/Im of (x+iy)^m expanded as
  real polynomials (so that complex-step differentiation applies);
* a zero vector has no direction: its harmonics are taken as the
  homogeneous polynomials at the origin, Y_00 = 1 and Y_lm = 0 for l > 0,
  with a zero Jacobian.
"""
import math

import numpy as np


def _legendre_deriv_coeffs(l, m):
    """Coefficients c_p of d^m P_l / dz^m = sum_p c_p z^p (exact rationals as floats)."""
    coeffs = {}
    for k in range(0, l // 2 + 1):
        power = l - 2 * k
        if power < m:
            continue
        c = ((-1) ** k * math.comb(l, k) * math.comb(2 * l - 2 * k, l)
             * math.factorial(power) // math.factorial(power - m))
        coeffs[power - m] = coeffs.get(power - m, 0) + c
    return {p: c / 2 ** l for p, c in coeffs.items()}


def _re_im_power(x, y, m):
    """Re and Im of (x + i y)^m as real polynomials in x and y (binomial sum)."""
    re = 0 * x
    im = 0 * x
    for p in range(m + 1):
        term = math.comb(m, p) * x ** (m - p) * y ** p
        # i^p cycles 1, i, -1, -i
        r = p % 4
        if r == 0:
            re = re + term
        elif r == 1:
            im = im + term
        elif r == 2:
            re = re - term
        else:
            im = im - term
    return re, im


def _sh_blocks(x, y, z, lmax):
    """The (lmax+1)^2 real harmonics of a unit vector given by x, y, z, as a
    list in lm order; x, y, z may be real or complex arrays or any number type
    with +, -, * and integer powers."""
    out = []
    for l in range(lmax + 1):
        block = [None] * (2 * l + 1)
        for m in range(0, l + 1):
            dP = sum(c * z ** p for p, c in _legendre_deriv_coeffs(l, m).items())
            if m == 0:
                block[l] = math.sqrt(2 * l + 1) * dP + 0 * x
            else:
                norm = math.sqrt(2 * (2 * l + 1) * math.factorial(l - m) / math.factorial(l + m))
                re, im = _re_im_power(x, y, m)
                block[l + m] = norm * dP * re
                block[l - m] = norm * dP * im
        out.extend(block)
    return out


def _sh_unit(x, y, z, lmax):
    """Real harmonics of a unit vector given by arrays x, y, z (real or complex)."""
    return np.stack(_sh_blocks(x, y, z, lmax), axis=-1)


def real_sh(vec, lmax):
    """Y_lm(vec / |vec|) for every l <= lmax, shape [..., (lmax+1)^2], fp64."""
    v = np.asarray(vec, dtype=np.float64)
    r = np.sqrt(np.sum(v * v, axis=-1))
    safe = np.where(r > 0, r, 1.0)
    u = v / safe[..., None]
    Y = _sh_unit(u[..., 0], u[..., 1], u[..., 2], lmax)
    zero = r == 0
    if np.any(zero):
        Y[zero] = 0.0
        Y[zero, 0] = 1.0
    return Y


def real_sh_jacobian(vec, lmax, h=1e-30):
    """dY_lm(vec/|vec|)/dvec by complex-step differentiation.

    Shape [..., (lmax+1)^2, 3].  Every operation on the way (the square root
    of the squared norm, the division, the polynomials) is analytic near the
    real input, so Im f(v + i h e_k) / h is the derivative to roundoff.
    """
    v = np.asarray(vec, dtype=np.float64)
    r = np.sqrt(np.sum(v * v, axis=-1))
    J = np.zeros(v.shape[:-1] + ((lmax + 1) ** 2, 3))
    for k in range(3):
        vc = v.astype(np.complex128)
        vc[..., k] += 1j * h
        rc = np.sqrt(vc[..., 0] ** 2 + vc[..., 1] ** 2 + vc[..., 2] ** 2)
        rc = np.where(r > 0, rc, 1.0)
        u = vc / rc[..., None]
        Yc = _sh_unit(u[..., 0], u[..., 1], u[..., 2], lmax)
        J[..., k] = Yc.imag / h
    J[r == 0] = 0.0
    return J


def real_sh_legendre(vec, lmax):
    """Second route to the same harmonics: spherical angles and the three-term
    associated-Legendre recurrence (no Condon-Shortley phase), for cross-checks."""
    v = np.asarray(vec, dtype=np.float64)
    r = np.sqrt(np.sum(v * v, axis=-1))
    ct = v[..., 2] / r
    st = np.sqrt(np.maximum(0.0, 1.0 - ct * ct))
    phi = np.arctan2(v[..., 1], v[..., 0])
    P = {}
    P[(0, 0)] = np.ones_like(ct)
    for m in range(1, lmax + 1):
        P[(m, m)] = (2 * m - 1) * st * P[(m - 1, m - 1)]
    for m in range(0, lmax + 1):
        if m + 1 <= lmax:
            P[(m + 1, m)] = (2 * m + 1) * ct * P[(m, m)]
        for l in range(m + 2, lmax + 1):
            P[(l, m)] = ((2 * l - 1) * ct * P[(l - 1, m)] - (l + m - 1) * P[(l - 2, m)]) / (l - m)
    out = []
    for l in range(lmax + 1):
        block = [None] * (2 * l + 1)
        block[l] = math.sqrt(2 * l + 1) * P[(l, 0)]
        for m in range(1, l + 1):
            norm = math.sqrt(2 * (2 * l + 1) * math.factorial(l - m) / math.factorial(l + m))
            block[l + m] = norm * P[(l, m)] * np.cos(m * phi)
            block[l - m] = norm * P[(l, m)] * np.sin(m * phi)
        out.extend(block)
    return np.stack(out, axis=-1)


def real_sh_hessian(vec, lmax):
    """d2Y_lm(vec/|vec|)/dvec2, shape [..., (lmax+1)^2, 3, 3], by second-order
    forward-mode differentiation (``oracle.jet``) of the same polynomial
    harmonics of the normalised vector.  Zero vectors get a zero Hessian."""
    from .jet import Jet
    v = np.asarray(vec, dtype=np.float64)
    r2 = np.sum(v * v, axis=-1)
    safe = np.where(r2 > 0, 1.0, 0.0)[..., None] * v + np.where(r2 > 0, 0.0, 1.0)[..., None] * np.array([0.0, 0.0, 1.0])
    x, y, z = Jet.variables(safe)
    inv = (x * x + y * y + z * z).sqrt().reciprocal()
    blocks = _sh_blocks(x * inv, y * inv, z * inv, lmax)
    H = np.stack([b.h for b in blocks], axis=-3)
    H[r2 == 0] = 0.0
    return H

