"""GPU parity: convolution forward/backward, radial network and forces
against the fp64 oracle, at the tiny, bulk and molecules workloads (full
size) and on edge cases (empty rows, isolated nodes, a single node, zero-length
edges, every supported multiplicity class)."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import cg as ocg
from oracle import conv as oconv
from oracle import graph as ograph
from oracle import radial as oradial
from tests.gpu_common import FWD_TOL, GRAD_TOL, THREADS, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _graph_pair(api, w):
    gp = None
    if w.graph_size is not None:
        gp = cuda(np.arange(0, w.n_nodes + 1, w.graph_size, dtype=np.int32))
    g = api.build_graph(cuda(w.pos), w.rc, box=w.box, graph_ptr=gp)
    o = ograph.neighbour_list(w.pos, w.rc, w.box, w.graph_id)
    assert g.n_edges == o["col"].size
    assert np.array_equal(host(g.col), o["col"])
    return g, o


def _random_w(o, P, mult, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((o["col"].size, P, mult)).astype(np.float32)


@pytest.mark.parametrize("name", ["tiny", "bulk", "molecules"])
def test_conv_forward_backward_random_weights(api, name):
    w = synthetic.WORKLOADS[name]()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    g, o = _graph_pair(api, w)
    W = _random_w(o, w.n_paths, w.mult, 100)
    plan = api.Plan(*L, w.mult)
    out = plan.conv_forward(g, cuda(w.x), cuda(W))
    ref = oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], w.x, W, *L, threads=THREADS)
    assert rel_err(host(out), ref) < FWD_TOL
    gx, gw, gr = plan.conv_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out))
    rx, rw, rr = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], w.x, W, w.grad_out, *L,
                                     threads=THREADS)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
    assert rel_err(host(gr), rr) < GRAD_TOL


@pytest.mark.parametrize("name", ["tiny", "molecules"])
def test_pipeline_with_radial_network_and_forces(api, name):
    """Graph -> radial weights -> conv forward -> backward (energy = sum of the
    l = 0 outputs, or the workload's output gradient) -> radial backward -> forces."""
    w = synthetic.WORKLOADS[name]()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    g, o = _graph_pair(api, w)
    plan = api.Plan(*L, w.mult)
    W1, W2 = cuda(w.W1), cuda(w.W2)
    Wg = plan.radial_forward(g.edge_vec, w.rc, W1, W2)
    Wo = oradial.radial_forward(o["edge_vec"], w.W1, w.W2, w.rc, w.n_paths, w.mult)
    assert rel_err(host(Wg), Wo) < FWD_TOL
    out = plan.conv_forward(g, cuda(w.x), Wg)
    ref = oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], w.x, Wo, *L, threads=THREADS)
    assert rel_err(host(out), ref) < FWD_TOL
    gx, gw, gr = plan.conv_backward(g, cuda(w.x), Wg, cuda(w.grad_out))
    rx, rw, rr = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], w.x, Wo, w.grad_out, *L,
                                     threads=THREADS)
    rr = rr + oradial.radial_backward(o["edge_vec"], w.W1, w.W2, w.rc, rw)
    plan.radial_backward(g.edge_vec, w.rc, W1, W2, gw, gr)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
    assert rel_err(host(gr), rr) < GRAD_TOL
    F = api.forces(g, gr)
    Fo = oconv.edge_forces(o["row_ptr"], o["col"], rr, w.n_nodes)
    assert rel_err(host(F), Fo) < GRAD_TOL
    assert np.abs(host(F).astype(np.float64).sum(axis=0)).max() < 1e-3 * np.abs(Fo).max()


@pytest.mark.parametrize("L,mult", [((0, 0, 0), 4), ((1, 1, 1), 8), ((1, 1, 1), 16), ((1, 2, 1), 32),
                                    ((2, 2, 2), 64), ((2, 2, 2), 96), ((2, 4, 2), 128), ((2, 4, 2), 256),
                                    ((3, 3, 3), 64), ((3, 3, 3), 128),
                                    # interaction, embedding and read-out shapes of the wider policy
                                    ((2, 3, 2), 64), ((1, 4, 1), 32), ((3, 4, 3), 32), ((3, 4, 3), 128),
                                    ((2, 0, 2), 16), ((0, 4, 3), 64), ((0, 1, 1), 8), ((3, 2, 0), 32),
                                    ((1, 4, 0), 128)])
def test_shapes_and_multiplicities(api, L, mult):
    rng = np.random.default_rng(30 + mult)
    n = 37  # ragged: not a multiple of any tile
    pos = (rng.random((n, 3)) * 6.0).astype(np.float32)
    o = ograph.neighbour_list(pos, 3.0)
    g = api.build_graph(cuda(pos), 3.0)
    P = len(ocg.paths(*L))
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult)).astype(np.float32)
    W = rng.standard_normal((o["col"].size, P, mult)).astype(np.float32)
    go = rng.standard_normal((n, (L[2] + 1) ** 2, mult)).astype(np.float32)
    plan = api.Plan(*L, mult)
    assert plan.n_paths == P and plan.paths == ocg.paths(*L)
    out = plan.conv_forward(g, cuda(x), cuda(W))
    assert rel_err(host(out), oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], x, W, *L)) < FWD_TOL
    gx, gw, gr = plan.conv_backward(g, cuda(x), cuda(W), cuda(go))
    rx, rw, rr = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], x, W, go, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
    assert rel_err(host(gr), rr) < GRAD_TOL


def test_high_degree_rows_span_several_batches(api):
    # one hub node with 150 neighbours plus leaves: rows longer than any edge batch
    rng = np.random.default_rng(31)
    n = 151
    row_ptr = np.zeros(n + 1, dtype=np.int32)
    row_ptr[1:] = np.concatenate([[150], 150 + np.arange(1, n)])
    col = np.concatenate([np.arange(1, n), np.zeros(n - 1)]).astype(np.int32)
    ev = rng.standard_normal((col.size, 3)).astype(np.float32)
    L, mult = (2, 4, 2), 128
    P = len(ocg.paths(*L))
    x = rng.standard_normal((n, 9, mult)).astype(np.float32)
    W = rng.standard_normal((col.size, P, mult)).astype(np.float32)
    go = rng.standard_normal((n, 9, mult)).astype(np.float32)
    cp, ce, cd = api.csr_transpose(n, cuda(row_ptr), cuda(col))
    g = api.Graph(n, col.size, cuda(row_ptr), cuda(col), cuda(ev), cp, ce, cd)
    plan = api.Plan(*L, mult)
    out = plan.conv_forward(g, cuda(x), cuda(W))
    assert rel_err(host(out), oconv.conv_forward(row_ptr, col, ev, x, W, *L)) < FWD_TOL
    gx, gw, gr = plan.conv_backward(g, cuda(x), cuda(W), cuda(go))
    rx, rw, rr = oconv.conv_backward(row_ptr, col, ev, x, W, go, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
    assert rel_err(host(gr), rr) < GRAD_TOL


def test_empty_isolated_single_and_zero_length(api):
    L, mult = (1, 1, 1), 8
    plan = api.Plan(*L, mult)
    rng = np.random.default_rng(32)
    # no edges at all: outputs and gradients are zero
    n = 5
    row_ptr = np.zeros(n + 1, dtype=np.int32)
    empty_i = np.zeros(0, dtype=np.int32)
    g = api.Graph(n, 0, cuda(row_ptr), cuda(empty_i), cuda(np.zeros((0, 3), np.float32)), cuda(row_ptr),
                  cuda(empty_i), cuda(empty_i))
    x = rng.standard_normal((n, 4, mult)).astype(np.float32)
    out = plan.conv_forward(g, cuda(x), cuda(np.zeros((0, 5, mult), np.float32)))
    assert np.all(host(out) == 0.0)
    gx, gw, gr = plan.conv_backward(g, cuda(x), cuda(np.zeros((0, 5, mult), np.float32)), cuda(x))
    assert np.all(host(gx) == 0.0)
    # zero-length edge (coincident atoms) and an isolated node
    row_ptr = np.array([0, 1, 2, 2], dtype=np.int32)
    col = np.array([1, 0], dtype=np.int32)
    ev = np.array([[0, 0, 0], [0, 0, 0]], dtype=np.float32)
    n = 3
    x = rng.standard_normal((n, 4, mult)).astype(np.float32)
    W = rng.standard_normal((2, 5, mult)).astype(np.float32)
    go = rng.standard_normal((n, 4, mult)).astype(np.float32)
    cp, ce, cd = api.csr_transpose(n, cuda(row_ptr), cuda(col))
    g = api.Graph(n, 2, cuda(row_ptr), cuda(col), cuda(ev), cp, ce, cd)
    out = plan.conv_forward(g, cuda(x), cuda(W))
    assert rel_err(host(out), oconv.conv_forward(row_ptr, col, ev, x, W, *L)) < FWD_TOL
    gx, gw, gr = plan.conv_backward(g, cuda(x), cuda(W), cuda(go))
    rx, rw, rr = oconv.conv_backward(row_ptr, col, ev, x, W, go, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL and rel_err(host(gw), rw) < GRAD_TOL
    assert np.all(host(gr) == 0.0) and np.all(rr == 0.0)


def test_optional_gradients_and_errors(api):
    from equivariant_mlip_tensor_b200 import CGTPError
    w = synthetic.tiny()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    g, o = _graph_pair(api, w)
    W = _random_w(o, w.n_paths, w.mult, 101)
    plan = api.Plan(*L, w.mult)
    full = plan.conv_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out))
    only_x = plan.conv_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out), want_w=False, want_r=False)
    only_r = plan.conv_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out), want_x=False, want_w=False)
    assert np.array_equal(host(only_x[0]), host(full[0]))
    assert np.array_equal(host(only_r[2]), host(full[2]))
    with pytest.raises(CGTPError) as ei:  # workspace too small
        plan.conv_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out), workspace=cuda(np.zeros(4, np.float32)))
    assert ei.value.status == 7
    with pytest.raises(CGTPError) as ei:
        api.Plan(2, 3, 1, 128)  # outside the compiled shapes
    assert ei.value.status == 2
    with pytest.raises(CGTPError) as ei:
        api.Plan(2, 3, 2, 128, mode="uvw")  # a shape the fully connected mode is not built for
    assert ei.value.status == 2
    # an entry point given a plan of another mode
    from equivariant_mlip_tensor_b200._lib import lib
    import ctypes
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    z = cuda(np.zeros((2, 4, w.mult), np.float32))
    assert lib().cgtp_tp_forward(plan.handle("conv"), 2, p(z), p(z), p(z), p(z), None) == 1
    assert lib().cgtp_conv_forward(plan.handle("pair"), g.n_nodes, g.n_edges, p(g.row_ptr), p(g.col),
                                   p(g.edge_vec), p(cuda(w.x)), p(cuda(W)), p(cuda(w.x)), None) == 1
    with pytest.raises(CGTPError) as ei:
        api.Plan(1, 1, 1, 6)
    assert ei.value.status == 1


def test_checked_mode_reports_and_stops_invalid_graphs(api):
    """Checked plans validate each call's graph on the device first; an index
    out of range is reported by cgtp_plan_check and the kernels do no work
    (the planted index is one past the last node, so even an unguarded read
    would stay inside the caller's allocation)."""
    w = synthetic.tiny()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    g, o = _graph_pair(api, w)
    W = _random_w(o, w.n_paths, w.mult, 102)
    plan = api.Plan(*L, w.mult)
    plan.set_checked(True)
    x, Wd, go = cuda(w.x), cuda(W), cuda(w.grad_out)
    out = plan.conv_forward(g, x, Wd)
    gx, gw, gr = plan.conv_backward(g, x, Wd, go)
    assert plan.check() == 0
    assert rel_err(host(out), oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], w.x, W, *L)) < FWD_TOL
    rx, rw, rr = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], w.x, W, w.grad_out, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL and rel_err(host(gw), rw) < GRAD_TOL
    bad_col = g.col.clone()
    bad_col[3] = w.n_nodes
    gb = api.Graph(g.n_nodes, g.n_edges, g.row_ptr, bad_col, g.edge_vec, g.csc_ptr, g.csc_edge, g.csc_dst)
    plan.conv_forward(gb, x, Wd)
    assert plan.check() & 2
    bad_dst = g.csc_dst.clone()
    bad_dst[0] = w.n_nodes
    gb = api.Graph(g.n_nodes, g.n_edges, g.row_ptr, g.col, g.edge_vec, g.csc_ptr, g.csc_edge, bad_dst)
    plan.conv_backward(gb, x, Wd, go)
    assert plan.check() & 32
    bad_ptr = g.csc_ptr.clone()
    bad_ptr[-1] = g.n_edges + 1
    gb = api.Graph(g.n_nodes, g.n_edges, g.row_ptr, g.col, g.edge_vec, bad_ptr, g.csc_edge, g.csc_dst)
    plan.conv_backward(gb, x, Wd, go)
    assert plan.check() & 16
    # the flags were cleared and a valid call computes as before
    out2 = plan.conv_forward(g, x, Wd)
    assert plan.check() == 0 and np.array_equal(host(out2), host(out))
    plan.set_checked(False)
    out3 = plan.conv_forward(g, x, Wd)
    assert np.array_equal(host(out3), host(out))
