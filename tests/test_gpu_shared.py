"""GPU parity of the convolution with weights shared by every path (path
stride 0) against the oracle: several shapes and multiplicities with a
ragged node count, and sampled rows and edges at the molecules workload."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import conv as oconv
from oracle import graph as ograph
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


@pytest.mark.parametrize("L,mult", [((1, 1, 1), 8), ((2, 2, 2), 64), ((2, 4, 2), 128), ((3, 3, 3), 32),
                                    ((3, 3, 3), 128)])
def test_matches_oracle(api, L, mult):
    rng = np.random.default_rng(110 + mult)
    n = 37
    pos = (rng.random((n, 3)) * 6.0).astype(np.float32)
    o = ograph.neighbour_list(pos, 3.0)
    g = api.build_graph(cuda(pos), 3.0)
    E = o["col"].size
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult)).astype(np.float32)
    w = rng.standard_normal((E, mult)).astype(np.float32)
    go = rng.standard_normal((n, (L[2] + 1) ** 2, mult)).astype(np.float32)
    plan = api.Plan(*L, mult)
    out = plan.conv_forward_shared(g, cuda(x), cuda(w))
    assert rel_err(host(out), oconv.conv_forward_shared(o["row_ptr"], o["col"], o["edge_vec"], x, w, *L)) <= FWD_TOL
    gx, gw, gr = plan.conv_backward_shared(g, cuda(x), cuda(w), cuda(go))
    rx, rw, rr = oconv.conv_backward_shared(o["row_ptr"], o["col"], o["edge_vec"], x, w, go, *L)
    for name, a, b in (("grad_x", gx, rx), ("grad_w", gw, rw), ("grad_r", gr, rr)):
        assert rel_err(host(a), b) <= GRAD_TOL, (name, rel_err(host(a), b))


def test_molecules_sampled(api):
    w = synthetic.molecules()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n = w.n_nodes
    g = api.build_graph(cuda(w.pos), w.rc, graph_ptr=cuda(np.arange(0, n + 1, w.graph_size, dtype=np.int32)))
    o = ograph.neighbour_list(w.pos, w.rc, None, w.graph_id)
    plan = api.Plan(*L, w.mult)
    rng = np.random.default_rng(120)
    E = o["col"].size
    ws = rng.standard_normal((E, w.mult)).astype(np.float32)
    out = plan.conv_forward_shared(g, cuda(w.x), cuda(ws))
    gx, gw, gr = plan.conv_backward_shared(g, cuda(w.x), cuda(ws), cuda(w.grad_out))
    rp = o["row_ptr"]
    dst_all = ograph.edge_dst(rp)

    def sub(edges):
        edges = np.sort(edges)
        sp = np.zeros(n + 1, dtype=np.int64)
        np.add.at(sp, dst_all[edges] + 1, 1)
        return np.cumsum(sp), o["col"][edges], o["edge_vec"][edges], edges

    nodes = np.sort(rng.choice(n, size=12, replace=False))
    srp, scol, sev, es = sub(np.nonzero(np.isin(dst_all, nodes))[0])
    ref = oconv.conv_forward_shared(srp, scol, sev, w.x, ws[es], *L)
    assert rel_err(host(out[nodes.tolist()]), ref[nodes]) <= FWD_TOL
    srp, scol, sev, es = sub(rng.choice(E, size=48, replace=False))
    _, rw, rr = oconv.conv_backward_shared(srp, scol, sev, w.x, ws[es], w.grad_out, *L)
    assert rel_err(host(gw[es.tolist()]), rw) <= GRAD_TOL
    assert rel_err(host(gr[es.tolist()]), rr) <= GRAD_TOL
    srp, scol, sev, es = sub(np.nonzero(np.isin(o["col"], nodes))[0])
    rx, _, _ = oconv.conv_backward_shared(srp, scol, sev, w.x, ws[es], w.grad_out, *L)
    assert rel_err(host(gx[nodes.tolist()]), rx[nodes]) <= GRAD_TOL
