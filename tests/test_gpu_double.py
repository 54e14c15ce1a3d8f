"""GPU parity of the double backward (adjoint of the convolution backward)
against the oracle: every shape, each cotangent alone and all together, the
nullable outputs, an edge-free graph, and sampled outputs at the molecules
workload (97 480 edges, L = (2,4,2), mult 128)."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import cg as ocg
from oracle import conv as oconv
from oracle import graph as ograph
from tests.gpu_common import GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _case(api, L, mult, seed, n=37):
    rng = np.random.default_rng(seed)
    pos = (rng.random((n, 3)) * 6.0).astype(np.float32)
    o = ograph.neighbour_list(pos, 3.0)
    g = api.build_graph(cuda(pos), 3.0)
    E, P = o["col"].size, len(ocg.paths(*L))
    ni, no = (L[0] + 1) ** 2, (L[2] + 1) ** 2
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    d = dict(o=o, g=g, x=f(n, ni, mult), W=f(E, P, mult), go=f(n, no, mult),
             ggx=f(n, ni, mult), ggw=f(E, P, mult), ggr=f(E, 3))
    return d


def _check(api, plan, d, L, cots):
    o = d["o"]
    ref = oconv.conv_double_backward(o["row_ptr"], o["col"], o["edge_vec"], d["x"], d["W"], d["go"],
                                     d["ggx"] if "x" in cots else None, d["ggw"] if "w" in cots else None,
                                     d["ggr"] if "r" in cots else None, *L)
    got = plan.conv_double_backward(d["g"], cuda(d["x"]), cuda(d["W"]), cuda(d["go"]),
                                    gg_x=cuda(d["ggx"]) if "x" in cots else None,
                                    gg_w=cuda(d["ggw"]) if "w" in cots else None,
                                    gg_edge_vec=cuda(d["ggr"]) if "r" in cots else None)
    for name, a, b in zip(("d_x", "d_w", "d_grad_out", "d_edge_vec"), got, ref):
        if not np.any(b):
            assert not np.any(host(a)), name
        else:
            assert rel_err(host(a), b) <= GRAD_TOL, (name, rel_err(host(a), b))


@pytest.mark.parametrize("L,mult", [((1, 1, 1), 8), ((2, 2, 2), 64), ((2, 4, 2), 128), ((3, 3, 3), 32),
                                    ((3, 3, 3), 128), ((2, 3, 2), 32), ((0, 2, 2), 16), ((3, 4, 3), 32)])
def test_all_cotangents(api, L, mult):
    d = _case(api, L, mult, 40 + mult)
    _check(api, api.Plan(*L, mult), d, L, "xwr")


@pytest.mark.parametrize("cots", ["x", "w", "r", "xw", "xr", "wr", ""])
def test_each_cotangent_combination(api, cots):
    L, mult = (2, 4, 2), 16
    d = _case(api, L, mult, 50 + len(cots))
    _check(api, api.Plan(*L, mult), d, L, cots)


def test_nullable_outputs_match_full_call(api):
    L, mult = (2, 2, 2), 32
    d = _case(api, L, mult, 61)
    plan = api.Plan(*L, mult)
    args = (d["g"], cuda(d["x"]), cuda(d["W"]), cuda(d["go"]))
    kw = dict(gg_x=cuda(d["ggx"]), gg_w=cuda(d["ggw"]), gg_edge_vec=cuda(d["ggr"]))
    full = plan.conv_double_backward(*args, **kw)
    flags = ("want_x", "want_w", "want_grad_out", "want_r")
    for k in range(4):
        only = plan.conv_double_backward(*args, **kw, **{f: (f == flags[k]) for f in flags})
        assert all(only[m] is None for m in range(4) if m != k)
        assert np.array_equal(host(only[k]), host(full[k]))


def test_graph_without_edges(api):
    L, mult = (1, 1, 1), 8
    n = 5
    pos = np.arange(3 * n, dtype=np.float32).reshape(n, 3) * 10.0  # nothing within the cutoff
    g = api.build_graph(cuda(pos), 1.0)
    assert g.n_edges == 0
    plan = api.Plan(*L, mult)
    x = cuda(np.ones((n, 4, mult), np.float32))
    go = cuda(np.ones((n, 4, mult), np.float32))
    w = cuda(np.zeros((0, plan.n_paths, mult), np.float32))
    dx, dw, dg, dr = plan.conv_double_backward(g, x, w, go, gg_x=x)
    assert not np.any(host(dx)) and not np.any(host(dg))
    assert dw.shape[0] == 0 and dr.shape[0] == 0


def _subgraph(o, edges):
    """CSR over all nodes holding only the given edges (in CSR order)."""
    edges = np.sort(edges)
    dst = ograph.edge_dst(o["row_ptr"])[edges]
    n = o["row_ptr"].size - 1
    rp = np.zeros(n + 1, dtype=np.int64)
    np.add.at(rp, dst + 1, 1)
    return np.cumsum(rp), o["col"][edges], o["edge_vec"][edges], edges


def test_molecules_sampled(api):
    import torch
    w = synthetic.molecules()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n = w.n_nodes
    gp = cuda(np.arange(0, n + 1, w.graph_size, dtype=np.int32))
    g = api.build_graph(cuda(w.pos), w.rc, graph_ptr=gp)
    plan = api.Plan(*L, w.mult)
    o = ograph.neighbour_list(w.pos, w.rc, None, w.graph_id)
    E = o["col"].size
    assert g.n_edges == E
    rng = np.random.default_rng(70)
    W = rng.standard_normal((E, plan.n_paths, w.mult)).astype(np.float32)
    ggx = rng.standard_normal(w.x.shape).astype(np.float32)
    ggw = rng.standard_normal(W.shape).astype(np.float32)
    ggr = rng.standard_normal((E, 3)).astype(np.float32)
    dx, dw, dg, dr = plan.conv_double_backward(g, cuda(w.x), cuda(W), cuda(w.grad_out), gg_x=cuda(ggx),
                                               gg_w=cuda(ggw), gg_edge_vec=cuda(ggr))
    torch.cuda.synchronize()
    # per-edge outputs of sampled edges: only those edges' data enter them
    edges = rng.choice(E, size=64, replace=False)
    rp, col, ev, es = _subgraph(o, edges)
    _, rw, _, rr = oconv.conv_double_backward(rp, col, ev, w.x, W[es], w.grad_out, ggx, ggw[es], ggr[es], *L)
    assert rel_err(host(dw[es.tolist()]), rw) <= GRAD_TOL
    assert rel_err(host(dr[es.tolist()]), rr) <= GRAD_TOL
    # rows of d_grad_out (all edges into sampled destinations) and of d_x (all
    # edges out of sampled sources)
    nodes = np.sort(rng.choice(n, size=12, replace=False))
    dst = ograph.edge_dst(o["row_ptr"])
    into = np.nonzero(np.isin(dst, nodes))[0]
    rp, col, ev, es = _subgraph(o, into)
    _, _, rg, _ = oconv.conv_double_backward(rp, col, ev, w.x, W[es], w.grad_out, ggx, ggw[es], ggr[es], *L)
    assert rel_err(host(dg[nodes.tolist()]), rg[nodes]) <= GRAD_TOL
    outof = np.nonzero(np.isin(o["col"], nodes))[0]
    rp, col, ev, es = _subgraph(o, outof)
    rx, _, _, _ = oconv.conv_double_backward(rp, col, ev, w.x, W[es], w.grad_out, ggx, ggw[es], ggr[es], *L)
    assert rel_err(host(dx[nodes.tolist()]), rx[nodes]) <= GRAD_TOL
