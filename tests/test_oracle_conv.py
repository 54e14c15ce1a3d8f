"""Pins for the oracle's convolution, adjoints, radial network, forces and
edge-free tensor product (CPU only)."""
import math

import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import cg, conv, graph, radial, sh, tp
from oracle.wigner import block_rotation, random_rotation


def _small_graph(seed=0, n=12, side=4.0, rc=2.5):
    rng = np.random.default_rng(seed)
    pos = (rng.random((n, 3)) * side).astype(np.float32)
    return pos, graph.neighbour_list(pos, rc)


def _inputs(nl, n, L, mult, seed=1):
    rng = np.random.default_rng(seed)
    P = len(cg.paths(*L))
    E = nl["col"].size
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult))
    w = rng.standard_normal((E, P, mult))
    g = rng.standard_normal((n, (L[2] + 1) ** 2, mult))
    return x, w, g


def _brute_force_complex(nl, x, w, L):
    """Pure-Python loops in the complex basis, with scipy's complex harmonics and
    the complex CG, mapped to the real basis at the end."""
    ss = pytest.importorskip("scipy.special")
    Lin, Lsh, Lout = L
    n, _, u = x.shape
    dst = graph.edge_dst(nl["row_ptr"])
    out = np.zeros((n, (Lout + 1) ** 2, u), dtype=np.complex128)
    for e in range(nl["col"].size):
        i, j = int(dst[e]), int(nl["col"][e])
        v = nl["edge_vec"][e].astype(np.float64)
        r = np.linalg.norm(v)
        th, ph = math.acos(v[2] / r), math.atan2(v[1], v[0])
        for p, (l1, l2, l3) in enumerate(cg.paths(*L)):
            Yc = math.sqrt(4 * math.pi) * np.array([ss.sph_harm_y(l2, m, th, ph)
                                                    for m in range(-l2, l2 + 1)])
            xc = cg.real_basis_q(l1).conj().T @ x[j, l1 * l1:(l1 + 1) ** 2, :]
            C = cg.complex_cg_block(l1, l2, l3)
            zc = np.zeros((2 * l3 + 1, u), dtype=np.complex128)
            for m1 in range(2 * l1 + 1):
                for m2 in range(2 * l2 + 1):
                    for m3 in range(2 * l3 + 1):
                        if C[m1, m2, m3] != 0.0:
                            zc[m3] += C[m1, m2, m3] * xc[m1] * Yc[m2]
            zr = cg.real_basis_q(l3) @ zc
            phase = 1.0 if (l1 + l2 + l3) % 2 == 0 else -1j  # real part, else imaginary part
            out[i, l3 * l3:(l3 + 1) ** 2, :] += phase * w[e, p][None, :] * zr
    assert np.abs(out.imag).max() < 1e-12
    return out.real


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 2, 2), (1, 2, 2), (2, 3, 1)])
def test_forward_matches_complex_basis_brute_force(L):
    pos, nl = _small_graph(n=8)
    x, w, _ = _inputs(nl, 8, L, 3)
    got = conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, *L)
    want = _brute_force_complex(nl, x, w, L)
    assert np.allclose(got, want, atol=1e-12)


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2), (3, 3, 3)])
def test_forward_equivariance(L):
    pos, nl = _small_graph(seed=2)
    x, w, _ = _inputs(nl, pos.shape[0], L, 4)
    R = random_rotation(np.random.default_rng(11))
    Din, Dout = block_rotation(L[0], R), block_rotation(L[2], R)
    out = conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, *L)
    xr = np.einsum("ab,nbu->nau", Din, x)
    ev = nl["edge_vec"].astype(np.float64) @ R.T
    out_r = conv.conv_forward(nl["row_ptr"], nl["col"], ev, xr, w, *L)
    assert np.allclose(out_r, np.einsum("ab,nbu->nau", Dout, out), atol=1e-10)


def test_scalar_path_is_weighted_segment_sum():
    pos, nl = _small_graph(seed=3)
    n = pos.shape[0]
    x, w, _ = _inputs(nl, n, (0, 0, 0), 5)
    got = conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, 0, 0, 0)
    dst = graph.edge_dst(nl["row_ptr"])
    want = np.zeros((n, 1, 5))
    for e in range(dst.size):
        want[dst[e], 0] += w[e, 0] * x[nl["col"][e], 0]
    assert np.allclose(got, want, atol=1e-13)


def test_vector_paths_are_dot_and_cross_products():
    pos, nl = _small_graph(seed=4)
    n = pos.shape[0]
    rng = np.random.default_rng(5)
    E = nl["col"].size
    x = rng.standard_normal((n, 4, 2))
    x[:, 0, :] = 0.0  # only the l = 1 block feeds the output
    ps = cg.paths(1, 1, 1)
    w = np.zeros((E, len(ps), 2))
    k110, k111 = ps.index((1, 1, 0)), ps.index((1, 1, 1))
    w[:, k110, :] = rng.standard_normal((E, 2))
    w[:, k111, :] = rng.standard_normal((E, 2))
    out = conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, 1, 1, 1)
    dst = graph.edge_dst(nl["row_ptr"])
    yzx_to_xyz = [2, 0, 1]
    want0 = np.zeros((n, 2))
    want1 = np.zeros((n, 3, 2))
    for e in range(E):
        v = nl["edge_vec"][e].astype(np.float64)
        rh = v / np.linalg.norm(v)
        xv = x[nl["col"][e], 1:4, :][yzx_to_xyz]  # (x, y, z) x channels
        want0[dst[e]] += -w[e, k110] * (rh @ xv)  # -(1/sqrt3) * sqrt3 (x . r)
        cr = np.cross(xv.T, rh).T  # x_j cross r_hat
        want1[dst[e]] += w[e, k111] * math.sqrt(3) / math.sqrt(2) * cr
    assert np.allclose(out[:, 0, :], want0, atol=1e-12)
    assert np.allclose(out[:, 1:4, :][:, yzx_to_xyz], want1, atol=1e-12)


def test_linearity():
    pos, nl = _small_graph(seed=6)
    L = (2, 2, 2)
    x, w, _ = _inputs(nl, pos.shape[0], L, 3)
    x2, w2, _ = _inputs(nl, pos.shape[0], L, 3, seed=9)
    f = lambda xx, ww: conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], xx, ww, *L)
    assert np.allclose(f(2 * x - x2, w), 2 * f(x, w) - f(x2, w), atol=1e-12)
    assert np.allclose(f(x, 3 * w + w2), 3 * f(x, w) + f(x, w2), atol=1e-12)


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2)])
def test_adjoint_identities(L):
    pos, nl = _small_graph(seed=7)
    x, w, g = _inputs(nl, pos.shape[0], L, 4)
    args = (nl["row_ptr"], nl["col"], nl["edge_vec"])
    out = conv.conv_forward(*args, x, w, *L)
    gx, gw, _ = conv.conv_backward(*args, x, w, g, *L)
    s = np.sum(g * out)
    assert np.sum(gx * x) == pytest.approx(s, rel=1e-12)
    assert np.sum(gw * w) == pytest.approx(s, rel=1e-12)


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2)])
def test_gradients_by_central_differences(L):
    pos, nl = _small_graph(seed=8, n=8)
    x, w, g = _inputs(nl, 8, L, 2)
    ev = nl["edge_vec"].astype(np.float64)
    args = (nl["row_ptr"], nl["col"])
    gx, gw, gr = conv.conv_backward(*args, ev, x, w, g, *L)
    f = lambda xx, ww, vv: np.sum(g * conv.conv_forward(*args, vv, xx, ww, *L))
    h = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(6):
        d = rng.standard_normal(ev.shape)
        fd = (f(x, w, ev + h * d) - f(x, w, ev - h * d)) / (2 * h)
        assert np.sum(gr * d) == pytest.approx(fd, rel=1e-6, abs=1e-7)
        dx = rng.standard_normal(x.shape)
        fd = (f(x + h * dx, w, ev) - f(x - h * dx, w, ev)) / (2 * h)
        assert np.sum(gx * dx) == pytest.approx(fd, rel=1e-6, abs=1e-7)
        dw = rng.standard_normal(w.shape)
        fd = (f(x, w + h * dw, ev) - f(x, w - h * dw, ev)) / (2 * h)
        assert np.sum(gw * dw) == pytest.approx(fd, rel=1e-6, abs=1e-7)


def test_radial_basis_and_derivative():
    rng = np.random.default_rng(12)
    rc = 3.0
    W1 = rng.standard_normal((8, 64)) / math.sqrt(8)
    W2 = rng.standard_normal((64, 5 * 4)) / 8.0
    # at r = mu_k the k-th Gaussian is 1 and the rest follow the closed form
    v = np.array([[0.0, 0.0, 3 * rc / 7]])
    Wv = radial.radial_forward(v, W1, W2, rc, 5, 4)
    mu = np.arange(8) * rc / 7
    phi = np.exp(-((3 * rc / 7 - mu) ** 2) / (2 * (rc / 7) ** 2))
    assert phi[3] == 1.0
    a = phi @ W1
    assert np.allclose(Wv.reshape(-1), (a / (1 + np.exp(-a))) @ W2, atol=1e-14)
    ev = rng.standard_normal((7, 3))
    gw = rng.standard_normal((7, 5, 4))
    gr = radial.radial_backward(ev, W1, W2, rc, gw)
    f = lambda vv: np.sum(gw * radial.radial_forward(vv, W1, W2, rc, 5, 4))
    h = 1e-6
    for _ in range(4):
        d = rng.standard_normal(ev.shape)
        fd = (f(ev + h * d) - f(ev - h * d)) / (2 * h)
        assert np.sum(gr * d) == pytest.approx(fd, rel=1e-6, abs=1e-8)


def _energy_and_forces(pos, nl, wl, L):
    """E = sum of l=0 outputs with the edge list fixed; forces by the adjoints."""
    row_ptr, col = nl["row_ptr"], nl["col"]
    dst = graph.edge_dst(row_ptr)

    def energy(p):
        ev = p[col] - p[dst]
        W = radial.radial_forward(ev, wl.W1, wl.W2, wl.rc, wl.n_paths, wl.mult)
        return np.sum(conv.conv_forward(row_ptr, col, ev, wl.x, W, *L)[:, 0, :])

    p = pos.astype(np.float64)
    ev = p[col] - p[dst]
    W = radial.radial_forward(ev, wl.W1, wl.W2, wl.rc, wl.n_paths, wl.mult)
    g = np.zeros((p.shape[0], (L[2] + 1) ** 2, wl.mult))
    g[:, 0, :] = 1.0
    _, gw, gr = conv.conv_backward(row_ptr, col, ev, wl.x, W, g, *L)
    gr = gr + radial.radial_backward(ev, wl.W1, wl.W2, wl.rc, gw)
    return energy, conv.edge_forces(row_ptr, col, gr, p.shape[0]), gr


def test_forces_by_central_differences_and_invariances():
    wl = synthetic.tiny()
    L = (wl.lmax_in, wl.lmax_sh, wl.lmax_out)
    nl = graph.neighbour_list(wl.pos, wl.rc)
    energy, F, gr = _energy_and_forces(wl.pos, nl, wl, L)
    p = wl.pos.astype(np.float64)
    h = 1e-6
    for a in range(0, p.shape[0], 5):
        for k in range(3):
            dp = np.zeros_like(p)
            dp[a, k] = h
            fd = (energy(p + dp) - energy(p - dp)) / (2 * h)
            assert -F[a, k] == pytest.approx(fd, rel=1e-6, abs=1e-6)
    assert np.allclose(F.sum(axis=0), 0.0, atol=1e-10)  # translation invariance
    # rotating the structure rotates the edge gradients and the forces
    R = random_rotation(np.random.default_rng(13))
    wr = synthetic.tiny()
    wr.x = np.einsum("ab,nbu->nau", block_rotation(L[0], R), wl.x.astype(np.float64))
    _, Fr, grr = _energy_and_forces(p @ R.T, nl, wr, L)
    assert np.allclose(grr, gr @ R.T, atol=1e-10)
    assert np.allclose(Fr, F @ R.T, atol=1e-10)


def test_zero_length_edge_convention():
    row_ptr = np.array([0, 1, 1], dtype=np.int32)
    col = np.array([1], dtype=np.int32)
    ev = np.zeros((1, 3), dtype=np.float32)
    rng = np.random.default_rng(14)
    x = rng.standard_normal((2, 4, 2))
    w = rng.standard_normal((1, 5, 2))
    out = conv.conv_forward(row_ptr, col, ev, x, w, 1, 1, 1)
    # Y = (1, 0, 0, 0): only the l2 = 0 paths (0,0,0) and (1,0,1) act
    ps = cg.paths(1, 1, 1)
    assert np.allclose(out[0, 0], w[0, ps.index((0, 0, 0))] * x[1, 0])
    assert np.allclose(out[0, 1:4], w[0, ps.index((1, 0, 1))] * x[1, 1:4])
    assert np.all(out[1] == 0.0)


def test_tp_equivariance_adjoints_and_single_edge_consistency():
    rng = np.random.default_rng(15)
    L = (2, 2, 2)
    B, u = 6, 3
    P = len(cg.paths(*L))
    x = rng.standard_normal((B, 9, u))
    y = rng.standard_normal((B, 9, u))
    w = rng.standard_normal((P, u))
    g = rng.standard_normal((B, 9, u))
    z = tp.tp_forward(x, y, w, *L)
    R = random_rotation(rng)
    D = block_rotation(2, R)
    rot = lambda a: np.einsum("ab,nbu->nau", D, a)
    assert np.allclose(tp.tp_forward(rot(x), rot(y), w, *L), rot(z), atol=1e-12)
    gx, gy, gw = tp.tp_backward(x, y, w, g, *L)
    s = np.sum(g * z)
    assert np.sum(gx * x) == pytest.approx(s, rel=1e-12)
    assert np.sum(gy * y) == pytest.approx(s, rel=1e-12)
    assert np.sum(gw * w) == pytest.approx(s, rel=1e-12)
    # with y the harmonics of a vector, one pair is a one-edge convolution
    v = rng.standard_normal((1, 3))
    yv = np.repeat(sh.real_sh(v, 2)[:, :, None], u, axis=2)
    zt = tp.tp_forward(x[:1], yv, w, *L)
    zc = conv.conv_forward(np.array([0, 1]), np.array([0]), v, x[:1], w[None], *L)
    assert np.allclose(zt, zc, atol=1e-13)
