"""GPU parity at the large periodic workload (20,000 atoms, ~1.05M edges,
L = 3, mult 128), whole tensors: the whole path runs at full size on the GPU;
the oracle checks the full neighbour list bit for bit and then recomputes
every output row, every feature gradient, every weight gradient (18 GB,
streamed from the device in chunks of whole source rows), every edge-vector
gradient and every force, in fp64 on the host's cores, and the measure
max|gpu - oracle| / max|oracle| is taken over each whole tensor."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import conv as oconv
from oracle import graph as ograph
from oracle import radial as oradial
from tests.gpu_common import FWD_TOL, GRAD_TOL, THREADS, cuda, host

pytestmark = pytest.mark.gpu

CHUNK_EDGES = 4096  # edges per oracle work item (whole rows)


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
    del Wg
    o = ograph.neighbour_list(w.pos, w.rc, w.box)
    res = dict(w=w, L=L, g=g, o=o, out=host(out), gx=host(gx), gw=gw, gr=host(gr), F=host(F))
    yield res
    del res, gw, out, gx, gr, F
    torch.cuda.empty_cache()


def _row_chunks(ptr, target):
    """Consecutive node ranges [a, b) of about `target` edges each (whole rows)."""
    ptr = np.asarray(ptr, dtype=np.int64)
    n = ptr.size - 1
    cuts = np.searchsorted(ptr, np.arange(0, ptr[-1], target), side="right") - 1
    cuts = np.unique(np.concatenate([[0], cuts, [n]]))
    return [(int(a), int(b)) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]


def _segment_sums(vals, starts, n_rows, n_vals):
    """Row sums of consecutive segments (rows with no entries are zero)."""
    out = np.zeros((n_rows,) + vals.shape[1:])
    deg = np.diff(np.concatenate([starts, [n_vals]]))
    nz = deg > 0
    if n_vals:
        out[nz] = np.add.reduceat(vals, starts[nz], axis=0)
    return out


def _bounded_map(fn, items, workers):
    """fn over items on a thread pool, results in order, at most 2 x workers
    in flight (each result holds a chunk of weight gradients)."""
    with ThreadPoolExecutor(max_workers=workers) as ex:
        pending = []
        for it in items:
            pending.append(ex.submit(fn, *it))
            if len(pending) >= 2 * workers:
                yield pending.pop(0).result()
        for f in pending:
            yield f.result()


class _Err:
    """max|got - want| and max|want| accumulated over chunks of one tensor."""

    def __init__(self):
        self.d = self.s = 0.0

    def add(self, got, want):
        got = np.asarray(got, dtype=np.float64)
        self.d = max(self.d, float(np.max(np.abs(got - want), initial=0.0)))
        self.s = max(self.s, float(np.max(np.abs(want), initial=0.0)))

    def rel(self):
        return self.d / self.s if self.s > 0 else self.d


@pytest.fixture(scope="module")
def whole(run):
    """Oracle over the whole graph, compared chunk by chunk with the GPU."""
    import torch
    from threadpoolctl import threadpool_limits
    w, L, o = run["w"], run["L"], run["o"]
    rp, col, ev = o["row_ptr"].astype(np.int64), o["col"].astype(np.int64), o["edge_vec"]
    cp, ce, cd = o["csc_ptr"].astype(np.int64), o["csc_edge"].astype(np.int64), o["csc_dst"].astype(np.int64)
    n, E = w.n_nodes, col.size
    workers = max(1, THREADS)

    def fwd(a, b):
        e0, e1 = rp[a], rp[b]
        Wc = oradial.radial_forward(ev[e0:e1], w.W1, w.W2, w.rc, w.n_paths, w.mult)
        m = oconv.edge_messages(col[e0:e1], ev[e0:e1], w.x, Wc, *L)
        return a, b, _segment_sums(m, rp[a:b] - e0, b - a, e1 - e0)

    def bwd(a, b):
        k0, k1 = cp[a], cp[b]
        edges = ce[k0:k1]
        evk = ev[edges]
        Wc = oradial.radial_forward(evk, w.W1, w.W2, w.rc, w.n_paths, w.mult)
        mx, gw, gr = oconv.edge_backward(col[edges], cd[k0:k1], evk, w.x, Wc, w.grad_out, *L)
        gr = gr + oradial.radial_backward(evk, w.W1, w.W2, w.rc, gw)
        return a, b, edges, _segment_sums(mx, cp[a:b] - k0, b - a, k1 - k0), gw, gr

    errs = {k: _Err() for k in ("out", "gx", "gw", "gr", "F")}
    gr_ref = np.zeros((E, 3))
    with threadpool_limits(1):
        for a, b, ref in _bounded_map(fwd, _row_chunks(rp, CHUNK_EDGES), workers):
            errs["out"].add(run["out"][a:b], ref)
        for a, b, edges, gx_ref, gw_ref, gr_chunk in _bounded_map(bwd, _row_chunks(cp, CHUNK_EDGES), workers):
            errs["gx"].add(run["gx"][a:b], gx_ref)
            idx = torch.as_tensor(edges, device=run["gw"].device)
            errs["gw"].add(host(run["gw"].index_select(0, idx)), gw_ref)
            gr_ref[edges] = gr_chunk
    errs["gr"].add(run["gr"], gr_ref)
    errs["F"].add(run["F"], oconv.edge_forces(rp, col, gr_ref, n))
    return {k: e.rel() for k, e in errs.items()}


def test_graph_bit_exact(run):
    g, o = run["g"], run["o"]
    assert g.n_edges == o["col"].size
    assert np.array_equal(host(g.row_ptr), o["row_ptr"])
    assert np.array_equal(host(g.col), o["col"])
    assert np.array_equal(host(g.edge_vec).view(np.uint32), o["edge_vec"].view(np.uint32))
    assert np.array_equal(host(g.csc_edge), o["csc_edge"])
    assert np.array_equal(host(g.csc_dst), o["csc_dst"])


def test_forward_whole_tensor(whole):
    assert whole["out"] < FWD_TOL, whole


def test_feature_and_weight_gradients_whole_tensors(whole):
    assert whole["gx"] < GRAD_TOL, whole
    assert whole["gw"] < GRAD_TOL, whole


def test_edge_vector_gradients_and_forces_whole_tensors(whole):
    assert whole["gr"] < GRAD_TOL, whole
    assert whole["F"] < GRAD_TOL, whole


def test_chunking_helpers_cover_every_row_once():
    assert _row_chunks(np.array([0, 0, 0, 5]), 2)[0][0] == 0  # leading empty rows are covered
    ptr = np.array([0, 3, 3, 3, 10, 11, 11, 20])
    chunks = _row_chunks(ptr, 4)
    assert chunks[0][0] == 0 and chunks[-1][1] == 7
    assert all(b0 == a1 for (_, b0), (a1, _) in zip(chunks[:-1], chunks[1:]))
    vals = np.arange(20.0)[:, None]
    sums = _segment_sums(vals, ptr[:-1], 7, 20)
    assert np.array_equal(sums[:, 0], [0 + 1 + 2, 0, 0, sum(range(3, 10)), 10, 0, sum(range(11, 20))])
