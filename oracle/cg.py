"""Clebsch-Gordan coefficients in the complex and the real basis (fp64).

Test infrastructure only (see ``oracle/__init__``).

Selection rules ("Tensor Decomposition Networks for Accelerating Machine
Learning Force Field Computations", reply to reviewer S6y1, on the low-rank
structure of the CG tensor): an entry is identically zero unless
|l1 - l2| <= l3 <= l1 + l2 and m3 = m1 + m2 (complex basis).

Conventions (the pages fix none; these are the plainest textbook readings):

* complex coefficients <l1 m1 l2 m2 | l3 m3> with the Condon-Shortley phase,
  from the Racah closed form, evaluated exactly in rational arithmetic;
* real basis: for m > 0 the real function is (Y^{-m} + (-1)^m Y^m)/sqrt(2),
  for m = 0 it is Y^0, for m < 0 it is i (Y^m - (-1)^m Y^{-m})/sqrt(2);
  index lm = l*l + (m + l), so the l = 1 block is ordered (y, z, x);
* real coefficients are the unitary (not unit-Frobenius) ones: the change of
  basis of the complex tensor.  Each path is purely real or purely
  imaginary; the real part is kept when it is nonzero, else the imaginary
  part.
"""
from fractions import Fraction
from functools import lru_cache
import math

import numpy as np


def _fact(n):
    return math.factorial(n)


@lru_cache(maxsize=None)
def complex_cg(j1, m1, j2, m2, J, M):
    """<j1 m1 j2 m2 | J M> by the Racah formula (integer angular momenta).

    The prefactors are exact rationals; the sum over k runs over every k for
    which all factorial arguments are non-negative.  Returns a Python float.
    """
    if M != m1 + m2:
        return 0.0
    if not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    pre = Fraction((2 * J + 1) * _fact(J + j1 - j2) * _fact(J - j1 + j2) * _fact(j1 + j2 - J),
                   _fact(j1 + j2 + J + 1))
    pre *= (_fact(J + M) * _fact(J - M) * _fact(j1 - m1) * _fact(j1 + m1)
            * _fact(j2 - m2) * _fact(j2 + m2))
    s = Fraction(0)
    for k in range(0, j1 + j2 + J + 2):
        args = (k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k)
        if min(args) < 0:
            continue
        den = 1
        for a in args:
            den *= _fact(a)
        s += Fraction((-1) ** k, den)
    if s == 0:
        return 0.0
    # value = sign(s) * sqrt(pre * s^2), with pre * s^2 an exact rational
    v2 = pre * s * s
    return math.copysign(math.sqrt(float(v2)), float(s))


def complex_cg_block(l1, l2, l3):
    """Dense complex CG block C[m1 + l1, m2 + l2, m3 + l3] (real numbers)."""
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for m1 in range(-l1, l1 + 1):
        for m2 in range(-l2, l2 + 1):
            m3 = m1 + m2
            if abs(m3) <= l3:
                C[m1 + l1, m2 + l2, m3 + l3] = complex_cg(l1, m1, l2, m2, l3, m3)
    return C


def real_basis_q(l):
    """Unitary Q_l with Y_real = Q_l @ Y_complex.

    Rows are indexed by the real m (offset by l), columns by the complex m.
    """
    Q = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    r = 1.0 / math.sqrt(2.0)
    for m in range(-l, l + 1):
        row = m + l
        if m > 0:
            Q[row, -m + l] = r
            Q[row, m + l] = (-1) ** m * r
        elif m == 0:
            Q[row, l] = 1.0
        else:
            Q[row, m + l] = 1j * r
            Q[row, -m + l] = -1j * (-1) ** m * r
    return Q


def real_cg_complex(l1, l2, l3):
    """The change of basis of the complex block, before the phase choice.

    C_r[a, b, c] = sum Q3[c, M] C[m1, m2, M] conj(Q1[a, m1]) conj(Q2[b, m2]).
    """
    C = complex_cg_block(l1, l2, l3)
    Q1, Q2, Q3 = real_basis_q(l1), real_basis_q(l2), real_basis_q(l3)
    return np.einsum("cM,ijM,ai,bj->abc", Q3, C, Q1.conj(), Q2.conj())


@lru_cache(maxsize=None)
def _real_cg_cached(l1, l2, l3):
    Cc = real_cg_complex(l1, l2, l3)
    if np.max(np.abs(Cc.real)) > 1e-12:
        out = Cc.real.copy()
    else:
        out = Cc.imag.copy()
    out[np.abs(out) < 1e-15] = 0.0
    out.setflags(write=False)
    return out


def real_cg(l1, l2, l3):
    """Real-basis unitary CG block [2l1+1, 2l2+1, 2l3+1] (fp64, read-only)."""
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        return np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    return _real_cg_cached(l1, l2, l3)


def paths(lmax_in, lmax_sh, lmax_out):
    """Every (l1, l2, l3) with l1 <= lmax_in, l2 <= lmax_sh and
    |l1 - l2| <= l3 <= min(l1 + l2, lmax_out), in lexicographic order."""
    out = []
    for l1 in range(lmax_in + 1):
        for l2 in range(lmax_sh + 1):
            for l3 in range(abs(l1 - l2), min(l1 + l2, lmax_out) + 1):
                out.append((l1, l2, l3))
    return out


def lm_offset(l):
    """Offset of degree l in the concatenated (l = 0..L) irreps layout."""
    return l * l
