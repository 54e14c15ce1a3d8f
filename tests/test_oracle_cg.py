"""Pins for the oracle's Clebsch-Gordan coefficients (CPU only).

Each check ties ``oracle.cg`` to something other than itself: a textbook
table, the textbook closed forms for coupling with l = 1, sympy's independent
implementation, the unitarity of the coupling, the selection rules of the
real basis, and equivariance under Wigner-D matrices built from the
harmonics.
"""
import math
import os

import numpy as np
import pytest

from oracle import cg
from oracle.wigner import block_rotation, random_rotation, wigner_d_real

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_textbook_1x1_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "cg_1x1_condon_shortley.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 19
    for m1, m2, J, M, sgn, num, den in rows:
        want = int(sgn) * math.sqrt(int(num) / int(den))
        got = cg.complex_cg(1, int(m1), 1, int(m2), int(J), int(M))
        assert got == pytest.approx(want, abs=1e-15), (m1, m2, J, M)


def _cg_j1_x_1(j1, m2, J, M):
    """Textbook closed forms of <j1 M-m2, 1 m2 | J M> (Condon-Shortley)."""
    j = j1
    if J == j + 1:
        d = {1: (j + M) * (j + M + 1) / ((2 * j + 1) * (2 * j + 2)),
             0: (j - M + 1) * (j + M + 1) / ((2 * j + 1) * (j + 1)),
             -1: (j - M) * (j - M + 1) / ((2 * j + 1) * (2 * j + 2))}[m2]
        return math.sqrt(d)
    if J == j:
        if m2 == 0:
            return M / math.sqrt(j * (j + 1))
        d = {1: (j + M) * (j - M + 1), -1: (j - M) * (j + M + 1)}[m2] / (2 * j * (j + 1))
        return -math.sqrt(d) if m2 == 1 else math.sqrt(d)
    if J == j - 1:
        d = {1: (j - M) * (j - M + 1) / (2 * j * (2 * j + 1)),
             0: (j - M) * (j + M) / (j * (2 * j + 1)),
             -1: (j + M + 1) * (j + M) / (2 * j * (2 * j + 1))}[m2]
        return -math.sqrt(d) if m2 == 0 else math.sqrt(d)
    raise ValueError


@pytest.mark.parametrize("j1", [1, 2, 3, 4])
def test_closed_form_couplings_with_l1(j1):
    for J in (j1 - 1, j1, j1 + 1):
        for M in range(-J, J + 1):
            for m2 in (-1, 0, 1):
                m1 = M - m2
                if abs(m1) > j1:
                    continue
                want = _cg_j1_x_1(j1, m2, J, M)
                assert cg.complex_cg(j1, m1, 1, m2, J, M) == pytest.approx(want, abs=1e-14)


def test_singlet_closed_form():
    for j in range(5):
        for m in range(-j, j + 1):
            want = (-1) ** (j - m) / math.sqrt(2 * j + 1)
            assert cg.complex_cg(j, m, j, -m, 0, 0) == pytest.approx(want, abs=1e-15)


def test_against_sympy():
    sym = pytest.importorskip("sympy.physics.quantum.cg")
    for j1 in range(4):
        for j2 in range(4):
            for J in range(abs(j1 - j2), j1 + j2 + 1):
                for m1 in range(-j1, j1 + 1):
                    for m2 in range(-j2, j2 + 1):
                        M = m1 + m2
                        if abs(M) > J:
                            continue
                        want = float(sym.CG(j1, m1, j2, m2, J, M).doit())
                        assert cg.complex_cg(j1, m1, j2, m2, J, M) == pytest.approx(want, abs=1e-14)


@pytest.mark.parametrize("l1,l2", [(a, b) for a in range(5) for b in range(5)])
def test_complex_orthogonality_and_completeness(l1, l2):
    blocks = [cg.complex_cg_block(l1, l2, l3) for l3 in range(abs(l1 - l2), l1 + l2 + 1)]
    for C in blocks:  # sum_{m1 m2} C[.,.,m3] C[.,.,m3'] = delta
        G = np.einsum("abc,abd->cd", C, C)
        assert np.allclose(G, np.eye(G.shape[0]), atol=1e-13)
    full = np.concatenate(blocks, axis=2)  # [d1, d2, sum(2l3+1)] = square unitary map
    S = np.einsum("abk,cdk->abcd", full, full).reshape((2 * l1 + 1) * (2 * l2 + 1), -1)
    assert np.allclose(S, np.eye(S.shape[0]), atol=1e-13)


@pytest.mark.parametrize("l1,l2", [(a, b) for a in range(5) for b in range(5)])
def test_real_orthogonality_and_completeness(l1, l2):
    blocks = [cg.real_cg(l1, l2, l3) for l3 in range(abs(l1 - l2), l1 + l2 + 1)]
    full = np.concatenate(blocks, axis=2)
    d = (2 * l1 + 1) * (2 * l2 + 1)
    M = full.reshape(d, -1)
    assert np.allclose(M.T @ M, np.eye(M.shape[1]), atol=1e-13)
    assert np.allclose(M @ M.T, np.eye(d), atol=1e-13)


def test_each_real_path_is_real_or_imaginary():
    for l1 in range(5):
        for l2 in range(5):
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                Cc = cg.real_cg_complex(l1, l2, l3)
                small = min(np.abs(Cc.real).max(), np.abs(Cc.imag).max())
                assert small < 1e-14
                # odd l1+l2+l3 is the imaginary case
                assert (np.abs(Cc.imag).max() > 1e-12) == ((l1 + l2 + l3) % 2 == 1)


def test_selection_rule_zeros():
    # complex basis: m3 != m1+m2 and triangle violations are identically zero
    for l1 in range(4):
        for l2 in range(4):
            for l3 in range(0, 8):
                for m1 in range(-l1, l1 + 1):
                    for m2 in range(-l2, l2 + 1):
                        for m3 in range(-l3, l3 + 1):
                            v = cg.complex_cg(l1, m1, l2, m2, l3, m3)
                            if m3 != m1 + m2 or not abs(l1 - l2) <= l3 <= l1 + l2:
                                assert v == 0.0
    # real basis: nonzero only if |m3| in {|m1|+|m2|, ||m1|-|m2||} and the number
    # of negative m's has the parity of l1+l2+l3 (reflection y -> -y)
    for l1 in range(5):
        for l2 in range(5):
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                C = cg.real_cg(l1, l2, l3)
                for a, b, c in zip(*np.nonzero(np.abs(C) > 1e-14)):
                    m1, m2, m3 = int(a) - l1, int(b) - l2, int(c) - l3
                    assert abs(m3) in (abs(m1) + abs(m2), abs(abs(m1) - abs(m2)))
                    assert (int(m1 < 0) + int(m2 < 0) + int(m3 < 0)) % 2 == (l1 + l2 + l3) % 2


def test_identity_paths():
    for l in range(5):
        I = np.eye(2 * l + 1)
        assert np.allclose(cg.real_cg(0, l, l)[0], I, atol=1e-15)
        assert np.allclose(cg.real_cg(l, 0, l)[:, 0, :], I, atol=1e-15)


def test_1x1_paths_are_dot_and_cross_products():
    rng = np.random.default_rng(3)
    a, b = rng.normal(size=3), rng.normal(size=3)  # stored in (y, z, x) order
    to_xyz = [2, 0, 1]
    s = np.einsum("abc,a,b->c", cg.real_cg(1, 1, 0), a, b)
    assert s[0] == pytest.approx(-np.dot(a, b) / math.sqrt(3), abs=1e-15)
    v = np.einsum("abc,a,b->c", cg.real_cg(1, 1, 1), a, b)
    cross = np.cross(a[to_xyz], b[to_xyz]) / math.sqrt(2)  # in (x, y, z)
    assert np.allclose(v[to_xyz], cross, atol=1e-15)
    # 1 x 1 -> 2 is symmetric and traceless
    C2 = cg.real_cg(1, 1, 2)
    assert np.allclose(C2, C2.transpose(1, 0, 2), atol=1e-15)
    assert np.allclose(np.einsum("aac->c", C2), 0.0, atol=1e-15)


def test_real_cg_equivariance():
    rng = np.random.default_rng(7)
    for _ in range(3):
        R = random_rotation(rng)
        for l1 in range(5):
            for l2 in range(5):
                for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                    C = cg.real_cg(l1, l2, l3)
                    x, y = rng.normal(size=2 * l1 + 1), rng.normal(size=2 * l2 + 1)
                    D1, D2, D3 = (wigner_d_real(l, R) for l in (l1, l2, l3))
                    lhs = np.einsum("abc,a,b->c", C, D1 @ x, D2 @ y)
                    rhs = D3 @ np.einsum("abc,a,b->c", C, x, y)
                    assert np.allclose(lhs, rhs, atol=1e-12)


def test_path_enumeration_counts():
    counts = {(1, 1, 1): 5, (2, 2, 2): 15, (3, 3, 3): 34, (2, 4, 2): 19}
    for L, n in counts.items():
        ps = cg.paths(*L)
        assert len(ps) == n
        assert all(abs(a - b) <= c <= a + b for a, b, c in ps)
    nnz = {(1, 1, 1): 16, (2, 2, 2): 137, (3, 3, 3): 611, (2, 4, 2): 244}
    for L, n in nnz.items():
        assert sum(int(np.count_nonzero(cg.real_cg(*p))) for p in cg.paths(*L)) == n
    assert block_rotation(2, np.eye(3)).shape == (9, 9)
