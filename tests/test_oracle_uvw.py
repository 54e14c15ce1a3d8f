"""Pins of the oracle's fully connected ("uvw") convolution: the identity
mixing reduces it to the channelwise convolution, a pure-Python brute force
over edges, nonzeros and channels (real CG from the Racah formula, harmonics
from the independent Legendre-recurrence route), equivariance under rotations, and
linearity in the mixing matrices; the backward against the channelwise
backward (identity mixing) and against central differences of the forward."""
import numpy as np
import pytest

from oracle import cg as ocg
from oracle import conv
from oracle import graph
from oracle import sh as osh
from oracle.wigner import block_rotation, random_rotation


def _problem(seed, L, u=3, v=2, n=8):
    rng = np.random.default_rng(seed)
    pos = rng.random((n, 3)) * 4.0
    nl = graph.neighbour_list(pos, 3.0)
    E, P = nl["col"].size, len(ocg.paths(*L))
    x = rng.standard_normal((n, (L[0] + 1) ** 2, u))
    w = rng.standard_normal((E, P, u))
    mix = rng.standard_normal((P, u, v))
    return nl, x, w, mix


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 2, 2), (2, 4, 2)])
def test_identity_mixing_is_the_channelwise_convolution(L):
    nl, x, w, _ = _problem(1, L, u=4)
    P = w.shape[1]
    eye = np.stack([np.eye(4)] * P)
    a = conv.conv_uvw_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, eye, *L)
    b = conv.conv_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, *L)
    assert np.abs(a - b).max() <= 1e-13 * np.abs(b).max()


def test_brute_force_loops():
    L = (1, 2, 1)
    nl, x, w, mix = _problem(2, L, u=2, v=3, n=6)
    rp, col, ev = nl["row_ptr"], nl["col"], nl["edge_vec"].astype(np.float64)
    dst = graph.edge_dst(rp)
    Y = osh.real_sh_legendre(ev, L[1])  # the independent harmonics route
    n, no = x.shape[0], (L[2] + 1) ** 2
    want = np.zeros((n, no, 3))
    for p, (l1, l2, l3) in enumerate(ocg.paths(*L)):
        C = ocg.real_cg(l1, l2, l3)
        for e in range(col.size):
            for a in range(2 * l1 + 1):
                for b in range(2 * l2 + 1):
                    for c in range(2 * l3 + 1):
                        if C[a, b, c] == 0.0:
                            continue
                        for uu in range(2):
                            t = C[a, b, c] * w[e, p, uu] * x[col[e], l1 * l1 + a, uu] * Y[e, l2 * l2 + b]
                            for vv in range(3):
                                want[dst[e], l3 * l3 + c, vv] += t * mix[p, uu, vv]
    got = conv.conv_uvw_forward(rp, col, ev, x, w, mix, *L)
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2)])
def test_equivariance(L):
    nl, x, w, mix = _problem(3, L)
    R = random_rotation(np.random.default_rng(12))
    Din, Dout = block_rotation(L[0], R), block_rotation(L[2], R)
    out = conv.conv_uvw_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, mix, *L)
    xr = np.einsum("ab,nbu->nau", Din, x)
    ev = nl["edge_vec"].astype(np.float64) @ R.T
    out_r = conv.conv_uvw_forward(nl["row_ptr"], nl["col"], ev, xr, w, mix, *L)
    assert np.abs(out_r - np.einsum("ab,nbv->nav", Dout, out)).max() <= 1e-10 * np.abs(out).max()


def test_linear_in_the_mixing():
    L = (2, 2, 2)
    nl, x, w, mix = _problem(4, L)
    mix2 = np.random.default_rng(5).standard_normal(mix.shape)
    f = lambda m: conv.conv_uvw_forward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, m, *L)
    assert np.abs(f(mix + 2.0 * mix2) - f(mix) - 2.0 * f(mix2)).max() <= 1e-12 * np.abs(f(mix)).max()


def test_backward_with_identity_mixing_is_channelwise_backward():
    L = (2, 2, 2)
    nl, x, w, _ = _problem(6, L, u=3)
    P = w.shape[1]
    g = np.random.default_rng(7).standard_normal((x.shape[0], 9, 3))
    eye = np.stack([np.eye(3)] * P)
    gx, gw, gm, gr = conv.conv_uvw_backward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, eye, g, *L)
    rx, rw, rr = conv.conv_backward(nl["row_ptr"], nl["col"], nl["edge_vec"], x, w, g, *L)
    for a, b in ((gx, rx), (gw, rw), (gr, rr)):
        assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2)])
def test_backward_matches_differences_of_forward(L):
    nl, x, w, mix = _problem(8, L)
    g = np.random.default_rng(9).standard_normal((x.shape[0], (L[2] + 1) ** 2, mix.shape[2]))
    rp, col = nl["row_ptr"], nl["col"]
    ev = nl["edge_vec"].astype(np.float64)
    grads = conv.conv_uvw_backward(rp, col, ev, x, w, mix, g, *L)
    f = lambda x_, w_, m_, e_: float(np.sum(g * conv.conv_uvw_forward(rp, col, e_, x_, w_, m_, *L)))
    rng = np.random.default_rng(10)
    h = 1e-6
    base = dict(x_=x, w_=w, m_=mix, e_=ev)
    for key, grad in zip(("x_", "w_", "m_", "e_"), grads):
        d = rng.standard_normal(base[key].shape)
        plus, minus = dict(base), dict(base)
        plus[key] = base[key] + h * d
        minus[key] = base[key] - h * d
        fd = (f(**plus) - f(**minus)) / (2 * h)
        an = float(np.sum(grad * d))
        assert abs(fd - an) <= 1e-7 * np.linalg.norm(grad) * np.linalg.norm(d), (key, fd, an)
