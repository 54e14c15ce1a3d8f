"""GPU parity of the fully connected ("uvw") convolution against the oracle:
forward at several shapes and output multiplicities, identity mixing against
the channelwise convolution, sampled rows at the molecules workload, an
edge-free graph and the host-side errors; backward (grad_x, grad_w, grad_mix,
grad_edge_vec) at four shapes and with each output alone."""
import ctypes

import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import cg as ocg
from oracle import conv as oconv
from oracle import graph as ograph
from tests.gpu_common import FWD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def _case(api, L, mult, mult_out, seed, n=37):
    rng = np.random.default_rng(seed)
    pos = (rng.random((n, 3)) * 6.0).astype(np.float32)
    o = ograph.neighbour_list(pos, 3.0)
    g = api.build_graph(cuda(pos), 3.0)
    E, P = o["col"].size, len(ocg.paths(*L))
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult)).astype(np.float32)
    W = rng.standard_normal((E, P, mult)).astype(np.float32)
    mix = (rng.standard_normal((P, mult, mult_out)) / np.sqrt(mult)).astype(np.float32)
    return o, g, x, W, mix


@pytest.mark.parametrize("L,mult,mult_out", [((1, 1, 1), 8, 4), ((1, 1, 1), 8, 12), ((2, 2, 2), 32, 16),
                                             ((2, 4, 2), 128, 128), ((2, 4, 2), 64, 96), ((3, 3, 3), 64, 32)])
def test_matches_oracle(api, L, mult, mult_out):
    o, g, x, W, mix = _case(api, L, mult, mult_out, 80 + mult + mult_out)
    plan = api.Plan(*L, mult)
    out = plan.uvw_forward(g, cuda(x), cuda(W), cuda(mix))
    ref = oconv.conv_uvw_forward(o["row_ptr"], o["col"], o["edge_vec"], x, W, mix, *L)
    assert out.shape == ref.shape
    assert rel_err(host(out), ref) <= FWD_TOL


def test_identity_mixing_is_channelwise_convolution(api):
    L, mult = (2, 4, 2), 32
    o, g, x, W, _ = _case(api, L, mult, mult, 90)
    plan = api.Plan(*L, mult)
    eye = np.stack([np.eye(mult, dtype=np.float32)] * plan.n_paths)
    a = plan.uvw_forward(g, cuda(x), cuda(W), cuda(eye))
    b = plan.conv_forward(g, cuda(x), cuda(W))
    ref = oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], x, W, *L)
    assert rel_err(host(a), ref) <= FWD_TOL
    assert rel_err(host(a), host(b).astype(np.float64)) <= FWD_TOL


def test_molecules_sampled_rows(api):
    w = synthetic.molecules()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n = w.n_nodes
    g = api.build_graph(cuda(w.pos), w.rc, graph_ptr=cuda(np.arange(0, n + 1, w.graph_size, dtype=np.int32)))
    o = ograph.neighbour_list(w.pos, w.rc, None, w.graph_id)
    plan = api.Plan(*L, w.mult)
    rng = np.random.default_rng(91)
    W = rng.standard_normal((o["col"].size, plan.n_paths, w.mult)).astype(np.float32)
    mix = (rng.standard_normal((plan.n_paths, w.mult, 128)) / np.sqrt(w.mult)).astype(np.float32)
    out = plan.uvw_forward(g, cuda(w.x), cuda(W), cuda(mix))
    nodes = np.sort(rng.choice(n, size=16, replace=False))
    rp = o["row_ptr"]
    edges = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in nodes])
    dst = ograph.edge_dst(rp)[edges]
    sub = np.zeros(n + 1, dtype=np.int64)
    np.add.at(sub, dst + 1, 1)
    ref = oconv.conv_uvw_forward(np.cumsum(sub), o["col"][edges], o["edge_vec"][edges], w.x, W[edges], mix, *L)
    assert rel_err(host(out[nodes.tolist()]), ref[nodes]) <= FWD_TOL


def test_graph_without_edges(api):
    L, mult = (1, 1, 1), 8
    n = 4
    pos = np.arange(3 * n, dtype=np.float32).reshape(n, 3) * 10.0
    g = api.build_graph(cuda(pos), 1.0)
    assert g.n_edges == 0
    plan = api.Plan(*L, mult)
    mix = cuda(np.ones((plan.n_paths, mult, 8), np.float32))
    w = cuda(np.zeros((0, plan.n_paths, mult), np.float32))
    out = plan.uvw_forward(g, cuda(np.ones((n, 4, mult), np.float32)), w, mix)
    assert not np.any(host(out))


def test_host_errors(api):
    import torch
    from equivariant_mlip_tensor_b200._lib import lib
    L, mult = (1, 1, 1), 8
    o, g, x, W, mix = _case(api, L, mult, 8, 92)
    plan = api.Plan(*L, mult)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    xd, Wd, md = cuda(x), cuda(W), cuda(mix)
    out = torch.empty((g.n_nodes, 4, 8), device="cuda")
    nb = plan.uvw_forward_workspace_bytes(g.n_nodes, 8)
    ws = torch.empty(nb // 4 + 64, device="cuda")
    args = (plan.handle("uvw"), g.n_nodes, g.n_edges, p(g.row_ptr), p(g.col), p(g.edge_vec), p(xd), p(Wd), p(md))
    f = lib().cgtp_uvw_forward
    assert f(*args, 6, p(out), p(ws), nb, None) == 2                # mult_out not a multiple of 4
    assert f(*args, 8, p(out), p(ws), nb - 256, None) == 7          # workspace too small
    assert f(*args, 8, p(out), None, 0, None) == 7                  # no workspace
    assert f(*args, 8, p(out), p(ws), nb, None) == 0


@pytest.mark.parametrize("L,mult,mult_out", [((1, 1, 1), 8, 12), ((2, 2, 2), 32, 16), ((2, 4, 2), 128, 128),
                                             ((3, 3, 3), 64, 32)])
def test_backward_matches_oracle(api, L, mult, mult_out):
    from tests.gpu_common import GRAD_TOL
    o, g, x, W, mix = _case(api, L, mult, mult_out, 95 + mult)
    rng = np.random.default_rng(96)
    go = rng.standard_normal((x.shape[0], (L[2] + 1) ** 2, mult_out)).astype(np.float32)
    plan = api.Plan(*L, mult)
    got = plan.uvw_backward(g, cuda(x), cuda(W), cuda(mix), cuda(go))
    ref = oconv.conv_uvw_backward(o["row_ptr"], o["col"], o["edge_vec"], x, W, mix, go, *L)
    for name, a, b in zip(("grad_x", "grad_w", "grad_mix", "grad_edge_vec"), got, ref):
        assert rel_err(host(a), b) <= GRAD_TOL, (name, rel_err(host(a), b))


def test_backward_nullable_outputs(api):
    L, mult, mult_out = (2, 2, 2), 16, 8
    o, g, x, W, mix = _case(api, L, mult, mult_out, 97)
    go = np.random.default_rng(98).standard_normal((x.shape[0], 9, mult_out)).astype(np.float32)
    plan = api.Plan(*L, mult)
    args = (g, cuda(x), cuda(W), cuda(mix), cuda(go))
    full = plan.uvw_backward(*args)
    flags = ("want_x", "want_w", "want_mix", "want_r")
    for k in range(4):
        only = plan.uvw_backward(*args, **{f: (f == flags[k]) for f in flags})
        assert all(only[m] is None for m in range(4) if m != k)
        # the chunk plan (and so the summation order of grad_x) depends on
        # whether grad_edge_vec is requested: equal to rounding, not bitwise
        assert rel_err(host(only[k]), host(full[k]).astype(np.float64)) <= 1e-6


def test_backward_molecules_sampled(api):
    """Full-size backward: per-edge gradients of sampled edges and grad_x rows
    of sampled sources against the oracle on the sub-graphs that determine them."""
    from tests.gpu_common import GRAD_TOL
    w = synthetic.molecules()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n = w.n_nodes
    g = api.build_graph(cuda(w.pos), w.rc, graph_ptr=cuda(np.arange(0, n + 1, w.graph_size, dtype=np.int32)))
    o = ograph.neighbour_list(w.pos, w.rc, None, w.graph_id)
    plan = api.Plan(*L, w.mult)
    rng = np.random.default_rng(99)
    E = o["col"].size
    W = rng.standard_normal((E, plan.n_paths, w.mult)).astype(np.float32)
    mix = (rng.standard_normal((plan.n_paths, w.mult, 64)) / np.sqrt(w.mult)).astype(np.float32)
    go = rng.standard_normal((n, 9, 64)).astype(np.float32)
    gx, gw, gm, gr = plan.uvw_backward(g, cuda(w.x), cuda(W), cuda(mix), cuda(go))
    rp = o["row_ptr"]
    dst_all = ograph.edge_dst(rp)

    def sub(edges):
        edges = np.sort(edges)
        sp = np.zeros(n + 1, dtype=np.int64)
        np.add.at(sp, dst_all[edges] + 1, 1)
        return np.cumsum(sp), o["col"][edges], o["edge_vec"][edges], edges

    edges = rng.choice(E, size=48, replace=False)
    srp, scol, sev, es = sub(edges)
    _, rw, _, rr = oconv.conv_uvw_backward(srp, scol, sev, w.x, W[es], mix, go, *L)
    assert rel_err(host(gw[es.tolist()]), rw) <= GRAD_TOL
    assert rel_err(host(gr[es.tolist()]), rr) <= GRAD_TOL
    nodes = np.sort(rng.choice(n, size=8, replace=False))
    srp, scol, sev, es = sub(np.nonzero(np.isin(o["col"], nodes))[0])
    rx, _, _, _ = oconv.conv_uvw_backward(srp, scol, sev, w.x, W[es], mix, go, *L)
    assert rel_err(host(gx[nodes.tolist()]), rx[nodes]) <= GRAD_TOL
