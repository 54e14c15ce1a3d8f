"""Real Wigner-D matrices for rotating irreps features (equivariance pins).

Test infrastructure only (see ``oracle/__init__``).

Two independent routes:

* ``wigner_d_real``: the textbook closed form of the small-d matrix
  d^l_{m'm}(beta) (a finite sum of factorial ratios), the complex
  D^l_{m'm}(alpha, beta, gamma) = e^{-i m' alpha} d^l_{m'm}(beta) e^{-i m gamma}
  for R = Rz(alpha) Ry(beta) Rz(gamma), and the change of basis of
  ``oracle.cg.real_basis_q``.  The real matrix is conj(Q) D Q^T, which is the
  form that satisfies Y(R u) = D(R) Y(u) for the harmonics of ``oracle.sh``
  (a pinned property, checked by the tests).
* ``wigner_d_fit``: the least-squares solution of Y(R u_k) = D Y(u_k) over
  random unit vectors u_k, which needs nothing but the harmonics.
"""
import math

import numpy as np

from .cg import real_basis_q
from .sh import real_sh


def rotation_zyz(alpha, beta, gamma):
    """3x3 rotation matrix Rz(alpha) @ Ry(beta) @ Rz(gamma)."""
    def rz(t):
        c, s = math.cos(t), math.sin(t)
        return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])

    def ry(t):
        c, s = math.cos(t), math.sin(t)
        return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])

    return rz(alpha) @ ry(beta) @ rz(gamma)


def euler_zyz(R):
    """Euler angles (alpha, beta, gamma) with R = Rz(alpha) Ry(beta) Rz(gamma)."""
    beta = math.acos(max(-1.0, min(1.0, R[2, 2])))
    if abs(math.sin(beta)) > 1e-12:
        alpha = math.atan2(R[1, 2], R[0, 2])
        gamma = math.atan2(R[2, 1], -R[2, 0])
    else:
        alpha = math.atan2(R[1, 0], R[0, 0]) if R[2, 2] > 0 else math.atan2(-R[1, 0], -R[0, 0])
        gamma = 0.0
    return alpha, beta, gamma


def small_d(l, beta):
    """Wigner small-d matrix d^l_{m'm}(beta), indices [m' + l, m + l]."""
    d = np.zeros((2 * l + 1, 2 * l + 1))
    c, s = math.cos(beta / 2.0), math.sin(beta / 2.0)
    f = math.factorial
    for mp in range(-l, l + 1):
        for m in range(-l, l + 1):
            pre = math.sqrt(f(l + mp) * f(l - mp) * f(l + m) * f(l - m))
            tot = 0.0
            for k in range(0, 2 * l + 1):
                a, b, cc, dd = l + m - k, k, l - k - mp, k - m + mp
                if min(a, b, cc, dd) < 0:
                    continue
                tot += ((-1) ** (k - m + mp) / (f(a) * f(b) * f(cc) * f(dd))
                        * c ** (2 * l - 2 * k + m - mp) * s ** (2 * k - m + mp))
            d[mp + l, m + l] = pre * tot
    return d


def wigner_d_complex(l, alpha, beta, gamma):
    ms = np.arange(-l, l + 1)
    return (np.exp(-1j * ms * alpha)[:, None] * small_d(l, beta)
            * np.exp(-1j * ms * gamma)[None, :])


def wigner_d_real(l, R):
    """Real (2l+1)x(2l+1) matrix of rotation R acting on a degree-l block."""
    alpha, beta, gamma = euler_zyz(R)
    D = wigner_d_complex(l, alpha, beta, gamma)
    Q = real_basis_q(l)
    Dr = Q.conj() @ D @ Q.T
    return Dr.real


def wigner_d_fit(l, R, n=64, seed=1234):
    """Least-squares D with Y_l(R u) = D Y_l(u) over n random unit vectors."""
    rng = np.random.default_rng(seed)
    u = rng.normal(size=(n, 3))
    Yu = real_sh(u, l)[:, l * l:(l + 1) ** 2]
    YRu = real_sh(u @ R.T, l)[:, l * l:(l + 1) ** 2]
    X, *_ = np.linalg.lstsq(Yu, YRu, rcond=None)
    return X.T


def block_rotation(lmax, R):
    """Block-diagonal real D for the concatenated l = 0..lmax layout."""
    n = (lmax + 1) ** 2
    D = np.zeros((n, n))
    for l in range(lmax + 1):
        D[l * l:(l + 1) ** 2, l * l:(l + 1) ** 2] = wigner_d_real(l, R)
    return D


def random_rotation(rng):
    """Haar-random rotation from a QR of a Gaussian matrix (det +1)."""
    A = rng.normal(size=(3, 3))
    Qm, Rm = np.linalg.qr(A)
    Qm = Qm * np.sign(np.diag(Rm))[None, :]
    if np.linalg.det(Qm) < 0:
        Qm[:, 0] = -Qm[:, 0]
    return Qm
