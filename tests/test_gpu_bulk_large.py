"""GPU parity at the large periodic workload (20,000 atoms, ~1.05M edges,
L = 3, mult 128): the whole path runs at full size on the GPU; the oracle
checks the full neighbour list bit for bit and a sample of outputs it can
compute one by one (output rows, weight gradients of sampled edges, feature
gradients of sampled sources, edge-vector gradients and forces)."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import conv as oconv
from oracle import graph as ograph
from oracle import radial as oradial
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def run():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api
    w = synthetic.bulk_large()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    g = api.build_graph(cuda(w.pos), w.rc, box=w.box, max_edges=1_200_000)
    plan = api.Plan(*L, w.mult)
    W1, W2 = cuda(w.W1), cuda(w.W2)
    Wg = plan.radial_forward(g.edge_vec, w.rc, W1, W2)
    x = cuda(w.x)
    out = plan.conv_forward(g, x, Wg)
    gx, gw, gr = plan.conv_backward(g, x, Wg, cuda(w.grad_out))
    plan.radial_backward(g.edge_vec, w.rc, W1, W2, gw, gr)
    F = api.forces(g, gr)
    torch.cuda.synchronize()
    o = ograph.neighbour_list(w.pos, w.rc, w.box)
    rng = np.random.default_rng(77)
    nodes = np.sort(rng.choice(w.n_nodes, size=24, replace=False))
    nodes = np.unique(np.concatenate([nodes, [0, w.n_nodes - 1]]))
    res = dict(w=w, L=L, g=g, o=o, nodes=nodes, out=out, gx=gx, gw=gw, gr=gr, F=F, Wg=Wg)
    yield res
    del res, Wg, gw, out, gx, gr, F
    torch.cuda.empty_cache()


def test_graph_bit_exact(run):
    g, o = run["g"], run["o"]
    assert g.n_edges == o["col"].size
    assert np.array_equal(host(g.row_ptr), o["row_ptr"])
    assert np.array_equal(host(g.col), o["col"])
    assert np.array_equal(host(g.edge_vec).view(np.uint32), o["edge_vec"].view(np.uint32))
    assert np.array_equal(host(g.csc_edge), o["csc_edge"])
    assert np.array_equal(host(g.csc_dst), o["csc_dst"])


def _edge_grads(w, L, o, edges):
    """Oracle gradients of the sampled edges: weights, and edge vectors
    including the radial network's contribution."""
    dst = ograph.edge_dst(o["row_ptr"])
    ev = o["edge_vec"][edges]
    Wo = oradial.radial_forward(ev, w.W1, w.W2, w.rc, w.n_paths, w.mult)
    mx, gw, gr = oconv.edge_backward(o["col"][edges], dst[edges], ev, w.x, Wo, w.grad_out, *L)
    gr = gr + oradial.radial_backward(ev, w.W1, w.W2, w.rc, gw)
    return mx, gw, gr


def test_forward_rows(run):
    w, L, o, nodes = run["w"], run["L"], run["o"], run["nodes"]
    rp = o["row_ptr"].astype(np.int64)
    Wrows = {}
    ref = []
    for i in nodes:
        s, e = rp[i], rp[i + 1]
        ev = o["edge_vec"][s:e]
        Wo = oradial.radial_forward(ev, w.W1, w.W2, w.rc, w.n_paths, w.mult)
        m = oconv.edge_messages(o["col"][s:e], ev, w.x, Wo, *L)
        ref.append(m.sum(axis=0))
    got = host(run["out"][nodes.tolist()])
    assert rel_err(got, np.stack(ref)) < FWD_TOL


def test_weight_and_edge_gradients_of_sampled_edges(run):
    w, L, o = run["w"], run["L"], run["o"]
    rng = np.random.default_rng(78)
    E = o["col"].size
    edges = np.unique(np.concatenate([rng.choice(E, size=400, replace=False), [0, E - 1]]))
    _, gw, gr = _edge_grads(w, L, o, edges)
    assert rel_err(host(run["gw"][edges.tolist()]), gw) < GRAD_TOL
    assert rel_err(host(run["gr"][edges.tolist()]), gr) < GRAD_TOL


def test_feature_gradients_and_forces_of_sampled_nodes(run):
    w, L, o, nodes = run["w"], run["L"], run["o"], run["nodes"]
    cp, ce = o["csc_ptr"].astype(np.int64), o["csc_edge"]
    rp = o["row_ptr"].astype(np.int64)
    gx_ref, F_ref = [], []
    for j in nodes:
        out_edges = ce[cp[j]:cp[j + 1]]          # edges leaving j (j is the source)
        in_edges = np.arange(rp[j], rp[j + 1])   # edges arriving at j
        mx, _, gr_out = _edge_grads(w, L, o, out_edges)
        gx_ref.append(mx.sum(axis=0))
        _, _, gr_in = _edge_grads(w, L, o, in_edges)
        F_ref.append(gr_in.sum(axis=0) - gr_out.sum(axis=0))
    assert rel_err(host(run["gx"][nodes.tolist()]), np.stack(gx_ref)) < GRAD_TOL
    assert rel_err(host(run["F"][nodes.tolist()]), np.stack(F_ref)) < GRAD_TOL
