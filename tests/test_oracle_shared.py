"""Pins of the oracle's shared-weight convolution (one weight row per edge
for every path): a brute-force loop over edges, paths and nonzeros with the
Legendre-route harmonics, and the backward against central differences of
the forward."""
import numpy as np
import pytest

from oracle import cg as ocg
from oracle import conv
from oracle import graph
from oracle import sh as osh


def _problem(seed, L, u=3, n=8):
    rng = np.random.default_rng(seed)
    nl = graph.neighbour_list(rng.random((n, 3)) * 4.0, 3.0)
    E = nl["col"].size
    x = rng.standard_normal((n, (L[0] + 1) ** 2, u))
    w = rng.standard_normal((E, u))
    g = rng.standard_normal((n, (L[2] + 1) ** 2, u))
    return nl, x, w, g


def test_brute_force():
    L = (1, 2, 1)
    nl, x, w, _ = _problem(1, L, u=2, n=6)
    rp, col, ev = nl["row_ptr"], nl["col"], nl["edge_vec"].astype(np.float64)
    dst = graph.edge_dst(rp)
    Y = osh.real_sh_legendre(ev, L[1])
    want = np.zeros((x.shape[0], 4, 2))
    for (l1, l2, l3) in ocg.paths(*L):
        C = ocg.real_cg(l1, l2, l3)
        for e in range(col.size):
            for a, b, c in zip(*np.nonzero(C)):
                want[dst[e], l3 * l3 + c] += C[a, b, c] * w[e] * x[col[e], l1 * l1 + a] * Y[e, l2 * l2 + b]
    got = conv.conv_forward_shared(rp, col, ev, x, w, *L)
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


@pytest.mark.parametrize("L", [(1, 1, 1), (2, 4, 2)])
def test_backward_matches_differences(L):
    nl, x, w, g = _problem(2, L)
    rp, col = nl["row_ptr"], nl["col"]
    ev = nl["edge_vec"].astype(np.float64)
    grads = conv.conv_backward_shared(rp, col, ev, x, w, g, *L)
    f = lambda x_, w_, e_: float(np.sum(g * conv.conv_forward_shared(rp, col, e_, x_, w_, *L)))
    rng = np.random.default_rng(3)
    h = 1e-6
    base = dict(x_=x, w_=w, e_=ev)
    for key, grad in zip(("x_", "w_", "e_"), grads):
        d = rng.standard_normal(base[key].shape)
        plus, minus = dict(base), dict(base)
        plus[key] = base[key] + h * d
        minus[key] = base[key] - h * d
        fd = (f(**plus) - f(**minus)) / (2 * h)
        an = float(np.sum(grad * d))
        assert abs(fd - an) <= 1e-7 * np.linalg.norm(grad) * np.linalg.norm(d), (key, fd, an)
