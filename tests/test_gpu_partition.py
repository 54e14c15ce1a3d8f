"""The domain decomposition with the library's kernels on one GPU.

Ranks are host threads, each with its own CUDA stream, that exchange their
halo rows through a thread barrier and device copies (no kernel waits on
another rank); each rank runs the partitioned forward, backward and forces
through the library (row gather / scatter-add, convolution, forces), and its
owned rows and local edges must match the fp64 oracle over the whole graph.
"""
import threading

import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import partition as part
from tests.gpu_common import FWD_TOL, GRAD_TOL, rel_err

pytestmark = pytest.mark.gpu


class ThreadComm:
    """all_to_all among threads of one process: each rank publishes its
    input split by destination, waits for every rank, then copies its own
    pieces in rank order."""

    def __init__(self, world, rank, shared):
        self.world, self.rank, self.sh = world, rank, shared

    def all_to_all(self, out, inp, out_counts, in_counts):
        import torch
        torch.cuda.current_stream().synchronize()
        offs = np.concatenate([[0], np.cumsum(np.asarray(in_counts, dtype=np.int64))])
        self.sh["slots"][self.rank] = [inp[int(offs[r]):int(offs[r + 1])] for r in range(self.world)]
        self.sh["barrier"].wait()
        o = 0
        for r in range(self.world):
            piece = self.sh["slots"][r][self.rank]
            k = piece.shape[0]
            if k:
                out[o:o + k].copy_(piece)
            o += k
        torch.cuda.current_stream().synchronize()
        self.sh["barrier"].wait()
        return out


def _problem(seed, n, mult, L):
    from oracle import graph as ograph
    rng = np.random.default_rng(seed)
    box = 12.0
    pos = (rng.random((n, 3)) * box).astype(np.float32)
    o = ograph.neighbour_list(pos, 4.0, box)
    P = sum(1 for l1 in range(L[0] + 1) for l2 in range(L[1] + 1)
            for l3 in range(abs(l1 - l2), min(l1 + l2, L[2]) + 1))
    E = o["col"].size
    x = rng.standard_normal((n, (L[0] + 1) ** 2, mult)).astype(np.float32)
    w = (rng.standard_normal((E, P, mult)) / np.sqrt(P)).astype(np.float32)
    g = rng.standard_normal((n, (L[2] + 1) ** 2, mult)).astype(np.float32)
    return o, x, w, g


@pytest.mark.parametrize("world", [2, 3])
def test_partitioned_step_on_the_gpu_equals_the_oracle(world):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api
    from oracle import conv as oconv
    L, mult, n = (2, 2, 2), 32, 600
    o, x, w, g = _problem(11, n, mult, L)
    dev = torch.device("cuda", 0)
    plan = api.Plan(*L, mult)
    bounds = part.edge_balanced_bounds(o["row_ptr"], world)
    shared = {"barrier": threading.Barrier(world), "slots": [None] * world}
    results, errors = [None] * world, []

    def rank_main(rank):
        try:
            torch.cuda.set_device(dev)
            with torch.cuda.stream(torch.cuda.Stream(dev)):
                n0, n1 = int(bounds[rank]), int(bounds[rank + 1])
                e0, e1 = int(o["row_ptr"][n0]), int(o["row_ptr"][n1])
                ev = torch.from_numpy(o["edge_vec"][e0:e1].copy()).to(dev)
                dd = part.DomainDecomposition(o["row_ptr"], o["col"], ev, world, rank,
                                              part.LibraryKernels(plan, dev), ThreadComm(world, rank, shared),
                                              bounds=bounds)
                xo = torch.from_numpy(x[n0:n1].copy()).to(dev)
                wl = torch.from_numpy(w[e0:e1].copy()).to(dev)
                y, x_ext = dd.forward(xo, wl)
                gx, gw, gr, F = dd.backward(x_ext, wl, torch.from_numpy(g[n0:n1].copy()).to(dev))
                torch.cuda.current_stream().synchronize()
                results[rank] = (n0, n1, e0, e1, dd.g.halo.size, *(t.cpu().numpy() for t in (y, gx, gw, gr, F)))
        except BaseException as exc:  # noqa: BLE001 - reported below
            errors.append(exc)
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    y_ref = oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], x, w, *L)
    gx_ref, gw_ref, gr_ref = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], x, w, g, *L)
    F_ref = oconv.edge_forces(o["row_ptr"], o["col"], gr_ref, n)
    assert sum(r[4] for r in results) > 0  # halo rows were exchanged
    for (n0, n1, e0, e1, _, y, gx, gw, gr, F) in results:
        assert rel_err(y, y_ref[n0:n1]) <= FWD_TOL
        assert rel_err(gx, gx_ref[n0:n1]) <= GRAD_TOL
        assert rel_err(gw, gw_ref[e0:e1]) <= GRAD_TOL
        assert rel_err(gr, gr_ref[e0:e1]) <= GRAD_TOL
        assert rel_err(F, F_ref[n0:n1]) <= GRAD_TOL
