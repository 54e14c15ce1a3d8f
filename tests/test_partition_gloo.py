"""Domain decomposition of one graph over several ranks, on CPU.

The partition and its halo exchanges (equivariant_mlip_tensor_b200.partition)
run as 2 and 3 gloo processes; each rank's compute is the fp64 oracle here
(a test-side backend with the calls the library's kernels serve on GPUs).
The owned rows of the forward, the feature gradients and forces of the owned
nodes, and the weight and edge-vector gradients of the local edges must equal
the single-rank oracle's over the whole graph.  Host-side index bookkeeping
(edge-balanced bounds, local numbering) is checked directly.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from equivariant_mlip_tensor_b200 import partition as part

TOL = 1e-12  # both sides fp64: only the summation order differs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleKernels:
    """The compute calls of a rank, evaluated by the oracle on CPU tensors."""

    def __init__(self, L):
        import torch
        self.L, self.device = L, torch.device("cpu")

    def graph(self, g, edge_vec_local):
        return {"g": g, "ev": np.asarray(edge_vec_local)}

    def empty(self, shape):
        import torch
        return torch.empty(shape, dtype=torch.float64)

    def zeros(self, shape):
        import torch
        return torch.zeros(shape, dtype=torch.float64)

    def gather_rows(self, idx, src):
        return src[idx.long()].contiguous()

    def scatter_add_rows(self, idx, src, dst):
        dst[idx.long()] += src
        return dst

    def conv_forward(self, graph, n_own, x_ext, w):
        import torch
        from oracle import conv as oconv
        g = graph["g"]
        return torch.from_numpy(oconv.conv_forward(g.row_ptr[:n_own + 1], g.col, graph["ev"], x_ext.numpy(),
                                                   w.numpy(), *self.L))

    def conv_backward(self, graph, x_ext, w, grad_out_ext):
        import torch
        from oracle import conv as oconv
        g = graph["g"]
        gx, gw, gr = oconv.conv_backward(g.row_ptr, g.col, graph["ev"], x_ext.numpy(), w.numpy(),
                                         grad_out_ext.numpy(), *self.L)
        return torch.from_numpy(gx), torch.from_numpy(gw), torch.from_numpy(gr)

    def forces(self, graph, grad_edge_vec):
        import torch
        from oracle import conv as oconv
        g = graph["g"]
        return torch.from_numpy(oconv.edge_forces(g.row_ptr, g.col, grad_edge_vec.numpy(), g.n_ext))


def _problem(seed, n, mult, L):
    """A periodic bulk graph and seeded features, weights and output gradient."""
    from oracle import graph as ograph
    rng = np.random.default_rng(seed)
    box = 9.0
    pos = (rng.random((n, 3)) * box).astype(np.float32)
    o = ograph.neighbour_list(pos, 3.5, box)
    P = sum(1 for l1 in range(L[0] + 1) for l2 in range(L[1] + 1)
            for l3 in range(abs(l1 - l2), min(l1 + l2, L[2]) + 1))
    E = o["col"].size
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult))
    w = rng.standard_normal((E, P, mult))
    g = rng.standard_normal((n, (L[2] + 1) ** 2, mult))
    return o, x, w, g


def _rank_main(rank, world, port, seed, n, mult, L, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        o, x, w, g = _problem(seed, n, mult, L)
        bounds = part.edge_balanced_bounds(o["row_ptr"], world)
        n0, n1 = int(bounds[rank]), int(bounds[rank + 1])
        e0, e1 = int(o["row_ptr"][n0]), int(o["row_ptr"][n1])
        dd = part.DomainDecomposition(o["row_ptr"], o["col"], o["edge_vec"][e0:e1], world, rank,
                                      OracleKernels(L), part.TorchComm(world, rank))
        xo = torch.from_numpy(x[n0:n1].copy())
        wl = torch.from_numpy(w[e0:e1].copy())
        y, x_ext = dd.forward(xo, wl)
        gx, gw, gr, F = dd.backward(x_ext, wl, torch.from_numpy(g[n0:n1].copy()))
        out.put((rank, n0, n1, e0, e1, int(dd.g.halo.size), y.numpy(), gx.numpy(), gw.numpy(), gr.numpy(),
                 F.numpy()))
    finally:
        dist.destroy_process_group()


def _rel(a, b):
    s = np.max(np.abs(b)) if b.size else 0.0
    return np.max(np.abs(a - b)) / s if s > 0 else np.max(np.abs(a - b), initial=0.0)


@pytest.mark.parametrize("world, L", [(2, (1, 1, 1)), (3, (2, 2, 2))])
def test_partitioned_step_equals_the_whole_graph(world, L):
    from oracle import conv as oconv
    seed, n, mult = 7, 150, 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, seed, n, mult, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    o, x, w, g = _problem(seed, n, mult, L)
    y_ref = oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], x, w, *L)
    gx_ref, gw_ref, gr_ref = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], x, w, g, *L)
    F_ref = oconv.edge_forces(o["row_ptr"], o["col"], gr_ref, n)
    covered = np.zeros(n, dtype=int)
    assert sum(r[5] for r in res) > 0  # the ranks do exchange halo rows
    for (_, n0, n1, e0, e1, _, y, gx, gw, gr, F) in res:
        covered[n0:n1] += 1
        assert _rel(y, y_ref[n0:n1]) < TOL
        assert _rel(gx, gx_ref[n0:n1]) < TOL
        assert _rel(gw, gw_ref[e0:e1]) < TOL
        assert _rel(gr, gr_ref[e0:e1]) < TOL
        assert _rel(F, F_ref[n0:n1]) < TOL
    assert np.all(covered == 1)  # the ranges tile the nodes


def test_edge_balanced_bounds_and_local_numbering():
    rng = np.random.default_rng(3)
    deg = rng.integers(0, 9, size=101)
    deg[40:45] = 0  # empty rows, also at a boundary
    row_ptr = np.concatenate([[0], np.cumsum(deg)])
    E = int(row_ptr[-1])
    col = rng.integers(0, 101, size=E)
    for world in (1, 2, 3, 5, 8):
        b = part.edge_balanced_bounds(row_ptr, world)
        assert b[0] == 0 and b[-1] == 101 and np.all(np.diff(b) >= 0)
        loads = row_ptr[b[1:]] - row_ptr[b[:-1]]
        assert loads.sum() == E and loads.max() - loads.min() <= 2 * deg.max() + E // world // 10 + 1
        for r in range(world):
            lg = part.local_graph(row_ptr, col, b, r)
            n0, n1 = int(b[r]), int(b[r + 1])
            src = col[lg.e0:lg.e1]
            # the extended numbering maps back to the global sources
            glob = np.where(lg.col < lg.n_own, lg.col + n0, lg.halo[np.clip(lg.col - lg.n_own, 0, None)]
                            if lg.halo.size else -1)
            assert np.array_equal(glob, src)
            assert np.all((lg.halo < n0) | (lg.halo >= n1)) and np.all(np.diff(lg.halo) > 0)
            assert lg.recv_counts.sum() == lg.halo.size and lg.recv_counts[r] == 0
            assert lg.row_ptr.size == lg.n_ext + 1 and lg.row_ptr[-1] == lg.e1 - lg.e0
