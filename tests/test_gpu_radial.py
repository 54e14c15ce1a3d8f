"""GPU parity of the radial weight network against the oracle: forward weights
and the backward's edge-vector gradient (added in place to a nonzero
grad_edge_vec) for output widths that do and do not fill the 128-wide output
tiles, edge counts around the 128-edge tiles (ragged tails, a single edge, many
tiles per persistent block), zero-length edges and an empty edge set."""
import numpy as np
import pytest

from oracle import cg as ocg
from oracle import radial as oradial
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu

RC = 5.0


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _inputs(seed, E, N):
    rng = np.random.default_rng(seed)
    d = rng.standard_normal((E, 3))
    d /= np.maximum(np.linalg.norm(d, axis=1, keepdims=True), 1e-12)
    ev = (d * rng.uniform(0.3, RC, (E, 1))).astype(np.float32)
    W1 = (rng.standard_normal((8, 64)) / np.sqrt(8)).astype(np.float32)
    W2 = (rng.standard_normal((64, N)) / 8.0).astype(np.float32)
    gw = rng.standard_normal((E, N)).astype(np.float32)
    g0 = rng.standard_normal((E, 3)).astype(np.float32)
    return ev, W1, W2, gw, g0


@pytest.mark.parametrize("L,mult,E", [((0, 0, 0), 4, 1), ((0, 0, 0), 4, 300), ((1, 1, 1), 8, 127),
                                      ((1, 2, 1), 32, 129), ((2, 4, 2), 8, 1000), ((2, 4, 2), 128, 700),
                                      ((3, 3, 3), 64, 257), ((2, 2, 2), 96, 4000)])
def test_matches_oracle(api, L, mult, E):
    plan = api.Plan(*L, mult)
    P = len(ocg.paths(*L))
    N = P * mult
    ev, W1, W2, gw, g0 = _inputs(7 * E + mult, E, N)
    Wg = plan.radial_forward(cuda(ev), RC, cuda(W1), cuda(W2))
    ref = oradial.radial_forward(ev, W1, W2, RC, P, mult)
    assert Wg.shape == (E, P, mult)
    assert rel_err(host(Wg), ref) <= FWD_TOL
    gev = cuda(g0)
    plan.radial_backward(cuda(ev), RC, cuda(W1), cuda(W2), cuda(gw), gev)
    want = g0.astype(np.float64) + oradial.radial_backward(ev, W1, W2, RC, gw.reshape(E, P, mult))
    assert rel_err(host(gev), want) <= GRAD_TOL


def test_zero_length_edges(api):
    L, mult = (1, 1, 1), 8
    plan = api.Plan(*L, mult)
    P = len(ocg.paths(*L))
    E = 130
    ev, W1, W2, gw, g0 = _inputs(3, E, P * mult)
    ev[::7] = 0.0
    Wg = plan.radial_forward(cuda(ev), RC, cuda(W1), cuda(W2))
    assert rel_err(host(Wg), oradial.radial_forward(ev, W1, W2, RC, P, mult)) <= FWD_TOL
    gev = cuda(g0)
    plan.radial_backward(cuda(ev), RC, cuda(W1), cuda(W2), cuda(gw), gev)
    got = host(gev)
    assert np.array_equal(got[::7], g0[::7])  # nothing added along an undefined direction
    want = g0.astype(np.float64) + oradial.radial_backward(ev, W1, W2, RC, gw)
    assert rel_err(got, want) <= GRAD_TOL


def test_no_edges(api):
    plan = api.Plan(1, 1, 1, 8)
    P = plan.n_paths
    ev = np.zeros((0, 3), np.float32)
    W1 = np.ones((8, 64), np.float32)
    W2 = np.ones((64, P * 8), np.float32)
    Wg = plan.radial_forward(cuda(ev), RC, cuda(W1), cuda(W2))
    assert Wg.shape == (0, P, 8)
    gev = cuda(np.zeros((0, 3), np.float32))
    plan.radial_backward(cuda(ev), RC, cuda(W1), cuda(W2), cuda(np.zeros((0, P * 8), np.float32)), gev)
