"""GPU parity: harmonics and neighbour lists against the oracle."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import graph as ograph
from oracle import sh as osh
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _vectors():
    rng = np.random.default_rng(20)
    v = rng.standard_normal((1000, 3)).astype(np.float32)
    axes = np.array([[1, 0, 0], [0, 1, 0], [0, 0, 1], [-1, 0, 0], [0, -1, 0], [0, 0, -1],
                     [3, 4, 0], [0, 0, 2.5], [1e-3, 0, 0], [0, 0, 0]], dtype=np.float32)
    return np.concatenate([v, axes, 40.0 * v[:50]])


@pytest.mark.parametrize("lmax", [0, 1, 2, 3, 4])
def test_harmonics_and_jacobian(api, lmax):
    v = _vectors()
    Y, dY = api.spherical_harmonics(lmax, cuda(v), with_grad=True)
    Yo = osh.real_sh(v.astype(np.float64), lmax)
    Jo = osh.real_sh_jacobian(v.astype(np.float64), lmax)
    assert rel_err(host(Y), Yo) < FWD_TOL
    # the Jacobian scales as 1/|r|; compare per edge against each edge's scale
    J = host(dY)
    for k in range(v.shape[0]):
        s = np.max(np.abs(Jo[k]))
        assert np.max(np.abs(J[k] - Jo[k])) <= GRAD_TOL * max(s, 1e-30) + 1e-30
    Y2 = api.spherical_harmonics(lmax, cuda(v))  # value-only path (rsqrt) vs the dual-number path
    assert rel_err(host(Y2), Yo) < FWD_TOL


def _compare_graph(g, o):
    E = o["col"].size
    assert g.n_edges == E
    assert np.array_equal(host(g.row_ptr), o["row_ptr"])
    assert np.array_equal(host(g.col), o["col"])
    assert np.array_equal(host(g.edge_vec).view(np.uint32), o["edge_vec"].view(np.uint32))
    assert np.array_equal(host(g.csc_ptr), o["csc_ptr"])
    assert np.array_equal(host(g.csc_edge), o["csc_edge"])
    assert np.array_equal(host(g.csc_dst), o["csc_dst"])


@pytest.mark.parametrize("name", ["tiny", "bulk", "molecules", "bulk_large"])
def test_neighbour_list_bit_exact(api, name):
    w = synthetic.WORKLOADS[name]()
    gp = None
    if w.graph_size is not None:
        gp = cuda(np.arange(0, w.n_nodes + 1, w.graph_size, dtype=np.int32))
    g = api.build_graph(cuda(w.pos), w.rc, box=w.box, graph_ptr=gp)
    o = ograph.neighbour_list(w.pos, w.rc, w.box, w.graph_id)
    _compare_graph(g, o)


def test_neighbour_list_small_capacity_rebuilds(api):
    w = synthetic.tiny()
    g = api.build_graph(cuda(w.pos), w.rc, max_edges=10)
    _compare_graph(g, ograph.neighbour_list(w.pos, w.rc))


def test_neighbour_list_edge_cases(api):
    # exactly-at-cutoff pair excluded, coincident atoms included, isolated atom, ties in rint
    pos = np.array([[0, 0, 0], [3, 0, 0], [0, 2.5, 0], [0, 2.5, 0], [9, 9, 9]], dtype=np.float32)
    g = api.build_graph(cuda(pos), 3.0)
    _compare_graph(g, ograph.neighbour_list(pos, 3.0))
    pos = np.array([[0, 0, 0], [2, 0, 0], [0.5, 5, 5], [9.6, 5, 5]], dtype=np.float32)
    g = api.build_graph(cuda(pos), 2.0, box=4.0 * 2.5)
    _compare_graph(g, ograph.neighbour_list(pos, 2.0, box=10.0))
    one = np.zeros((1, 3), dtype=np.float32)
    g = api.build_graph(cuda(one), 1.0)
    assert g.n_edges == 0 and np.array_equal(host(g.row_ptr), [0, 0])


def test_csr_transpose_of_asymmetric_graph(api):
    rng = np.random.default_rng(21)
    n = 300
    deg = rng.integers(0, 40, size=n)
    rows = [np.sort(rng.choice(n, size=d, replace=False)).astype(np.int32) for d in deg]
    row_ptr = np.zeros(n + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(deg)
    col = np.concatenate(rows).astype(np.int32)
    cp, ce, cd = api.csr_transpose(n, cuda(row_ptr), cuda(col))
    o = ograph.csr_to_csc(row_ptr, col, n)
    assert np.array_equal(host(cp), o["csc_ptr"])
    assert np.array_equal(host(ce), o["csc_edge"])
    assert np.array_equal(host(cd), o["csc_dst"])


def test_graph_check_flags(api):
    row_ptr = np.array([0, 2, 1, 3], dtype=np.int32)
    col = np.array([1, 5, 0], dtype=np.int32)
    ev = np.array([[0, 0, 0], [1, 0, 0], [np.nan, 0, 0]], dtype=np.float32)
    flags = api.graph_check(3, cuda(row_ptr), cuda(col), cuda(ev))
    assert flags == (1 | 2 | 4 | 8)
    w = synthetic.tiny()
    g = api.build_graph(cuda(w.pos), w.rc)
    assert api.graph_check(w.n_nodes, g.row_ptr, g.col, g.edge_vec) == 0
