"""Domain decomposition of one graph over several GPUs (one process per GPU).

For a graph too large for one GPU, or one step that several GPUs should
share, the destination nodes are cut into contiguous ranges with about the
same number of edges (CSR rows) per rank.  A rank owns the rows of its range:
their edges, weights and weight gradients stay local, so the dominant bytes
(W, grad_W) never move.  The one exchange a convolution needs is the feature
rows of the sources that lie in another rank's range (the halo):

  forward   x of the halo sources arrive from their owners (all-to-all),
            then the node-centric forward runs over the owned rows;
  backward  the source-centric backward runs over the local edges grouped by
            source (a CSC over the owned and halo nodes), so each rank forms
            grad_x for its own sources and partial grad_x for its halo
            sources; the halo partials go back to their owners (all-to-all)
            and are added there; the per-atom forces, whose source part is
            likewise partial on the halo, take the same reverse exchange.

The pages name scalability across GPUs as a goal without a method ("LunaTP:
Enabling Efficient and Scalable Tensor Product for Equivariant MLIPs",
abstract); this partition is our design.  The exchange uses
torch.distributed.all_to_all_single, which runs over NCCL (NVLink) on GPUs and
over gloo on CPU tensors; packing and unpacking the rows are the library's
gather / scatter-add kernels on GPUs.  No exchange buffer crosses to a peer
GPU except through the collective, so no kernel reads another GPU's memory.

Compute goes through a ``kernels`` object with the calls of
``LibraryKernels`` below (the library's kernels); the partition logic itself
is host-side index bookkeeping.
"""
from dataclasses import dataclass

import numpy as np


def edge_balanced_bounds(row_ptr, world):
    """Node boundaries b[0] = 0 <= ... <= b[world] = N of contiguous ranges
    whose edge counts differ by at most the largest row: b[r] is the first
    node whose row starts at or after r * E / world."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n, E = row_ptr.size - 1, int(row_ptr[-1])
    b = np.empty(world + 1, dtype=np.int64)
    b[0], b[world] = 0, n
    for r in range(1, world):
        b[r] = min(n, int(np.searchsorted(row_ptr[:n], (r * E) // world, side="left")))
    return np.maximum.accumulate(b)


@dataclass
class LocalGraph:
    """A rank's part of the graph, in its extended node numbering: owned
    nodes 0..n_own-1 (global n0..n1-1), then the halo sources n_own..n_ext-1
    (sorted by global index, hence grouped by owner)."""
    n0: int
    n1: int
    e0: int
    e1: int
    n_own: int
    n_ext: int
    halo: np.ndarray        # [H] global ids of the halo sources
    recv_counts: np.ndarray  # [world] halo rows owned by each rank
    row_ptr: np.ndarray     # [n_ext + 1] local CSR (rows past n_own empty)
    col: np.ndarray         # [E_loc] sources in the extended numbering


def local_graph(row_ptr, col, bounds, rank):
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    n0, n1 = int(bounds[rank]), int(bounds[rank + 1])
    e0, e1 = int(row_ptr[n0]), int(row_ptr[n1])
    src = col[e0:e1]
    halo = np.unique(src[(src < n0) | (src >= n1)])
    owner = np.searchsorted(bounds, halo, side="right") - 1
    world = bounds.size - 1
    recv_counts = np.bincount(owner, minlength=world).astype(np.int64)
    n_own = n1 - n0
    ext = np.where((src >= n0) & (src < n1), src - n0, n_own + np.searchsorted(halo, src))
    n_ext = n_own + halo.size
    rp = np.concatenate([row_ptr[n0:n1 + 1] - e0, np.full(halo.size, e1 - e0, dtype=np.int64)])
    return LocalGraph(n0, n1, e0, e1, n_own, n_ext, halo, recv_counts, rp, ext.astype(np.int64))


class TorchComm:
    """all_to_all over torch.distributed (NCCL for CUDA tensors, gloo for CPU
    ones); rows split along dim 0."""

    def __init__(self, world, rank):
        import torch.distributed as dist
        self.world, self.rank, self._dist = world, rank, dist

    def all_to_all(self, out, inp, out_counts, in_counts):
        if self.world == 1:
            if inp.numel():
                out.copy_(inp)
            return out
        self._dist.all_to_all_single(out, inp, output_split_sizes=[int(c) for c in out_counts],
                                     input_split_sizes=[int(c) for c in in_counts])
        return out


class DomainDecomposition:
    """One rank's view of the partitioned graph and its halo exchanges.

    row_ptr, col: the whole graph's CSR (host arrays, the same on every rank);
    edge_vec: the local edges' vectors (rows e0..e1 of the whole graph's) on
    the compute device; kernels: the compute calls (``LibraryKernels``);
    comm: the exchange (``TorchComm``).  Construction exchanges the halo
    requests once (two all-to-alls), so every rank must construct it in the
    same order."""

    def __init__(self, row_ptr, col, edge_vec_local, world, rank, kernels, comm, bounds=None):
        import torch
        self.world, self.rank, self.k, self.comm = world, rank, kernels, comm
        self.bounds = edge_balanced_bounds(row_ptr, world) if bounds is None else np.asarray(bounds)
        g = self.g = local_graph(row_ptr, col, self.bounds, rank)
        dev = kernels.device
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)
        # who wants which of my rows: counts, then the global ids themselves
        send_counts = torch.zeros(world, dtype=torch.int64, device=dev)
        comm.all_to_all(send_counts, torch.as_tensor(g.recv_counts, device=send_counts.device),
                        np.ones(world, dtype=np.int64), np.ones(world, dtype=np.int64))
        self.send_counts = send_counts.cpu().numpy().astype(np.int64)
        self.recv_counts = g.recv_counts
        req = torch.empty(int(self.send_counts.sum()), dtype=torch.int64, device=send_counts.device)
        comm.all_to_all(req, torch.as_tensor(g.halo, dtype=torch.int64, device=send_counts.device),
                        self.send_counts, self.recv_counts)
        send_ids = req.cpu().numpy() - g.n0
        assert np.all((send_ids >= 0) & (send_ids < g.n_own)), "halo request outside the owned range"
        self.send_idx = i32(send_ids)                       # owned rows to send, grouped by peer
        self.send_off = np.concatenate([[0], np.cumsum(self.send_counts)])
        self.graph = kernels.graph(g, edge_vec_local)       # local CSR (+ CSC over the extended nodes)

    # -------------------------------------------------------------- exchanges
    def halo_forward(self, x_own, x_ext):
        """x_ext[:n_own] = x_own; x_ext[n_own:] = the halo rows from their owners."""
        g = self.g
        x_ext[:g.n_own].copy_(x_own)
        send = self.k.gather_rows(self.send_idx, x_own)
        self.comm.all_to_all(x_ext[g.n_own:], send, self.recv_counts, self.send_counts)
        return x_ext

    def halo_reverse_add(self, own, ext_rows):
        """own[j] += the halo partials of j that other ranks computed
        (ext_rows: this rank's partials of its halo rows, in halo order)."""
        import torch
        back = torch.empty((int(self.send_counts.sum()),) + tuple(own.shape[1:]), dtype=own.dtype,
                           device=own.device)
        self.comm.all_to_all(back, ext_rows, self.send_counts, self.recv_counts)
        for r in range(self.world):  # a node appears at most once in each peer's segment
            a, b = int(self.send_off[r]), int(self.send_off[r + 1])
            if b > a:
                self.k.scatter_add_rows(self.send_idx[a:b], back[a:b], own)
        return own

    # -------------------------------------------------------------- the path
    def forward(self, x_own, w_local, x_ext=None):
        """out rows of the owned nodes; x_ext (optional) receives the
        extended features for the backward."""
        g = self.g
        if x_ext is None:
            x_ext = self.k.empty((g.n_ext,) + tuple(x_own.shape[1:]))
        self.halo_forward(x_own, x_ext)
        return self.k.conv_forward(self.graph, g.n_own, x_ext, w_local), x_ext

    def backward(self, x_ext, w_local, grad_out_own):
        """(grad_x of the owned nodes, grad_w of the local edges, grad_edge_vec
        of the local edges, forces of the owned nodes)."""
        g = self.g
        go_ext = self.k.zeros((g.n_ext,) + tuple(grad_out_own.shape[1:]))
        go_ext[:g.n_own].copy_(grad_out_own)  # only owned destinations are read
        gx_ext, gw, gr = self.k.conv_backward(self.graph, x_ext, w_local, go_ext)
        gx = gx_ext[:g.n_own].clone()
        self.halo_reverse_add(gx, gx_ext[g.n_own:].contiguous())
        F_ext = self.k.forces(self.graph, gr)
        F = F_ext[:g.n_own].clone()
        self.halo_reverse_add(F, F_ext[g.n_own:].contiguous())
        return gx, gw, gr, F


class LibraryKernels:
    """The compute of a rank through the library (CUDA tensors)."""

    def __init__(self, plan, device):
        self.plan, self.device = plan, device

    def graph(self, g, edge_vec_local):
        import torch
        from . import api
        i32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=self.device)
        row_ptr, col = i32(g.row_ptr), i32(g.col)
        csc_ptr, ce, cd = api.csr_transpose(g.n_ext, row_ptr, col)
        return api.Graph(g.n_ext, int(col.numel()), row_ptr, col, edge_vec_local, csc_ptr, ce, cd)

    def empty(self, shape):
        import torch
        return torch.empty(shape, dtype=torch.float32, device=self.device)

    def zeros(self, shape):
        import torch
        return torch.zeros(shape, dtype=torch.float32, device=self.device)

    def gather_rows(self, idx, src):
        from . import api
        return api.gather_rows(idx, src.contiguous())

    def scatter_add_rows(self, idx, src, dst):
        from . import api
        return api.scatter_add_rows(idx, src.contiguous(), dst)

    def conv_forward(self, graph, n_own, x_ext, w):
        """Output rows of the n_own owned nodes (the local CSR's first rows)."""
        from . import api
        fwd = api.Graph(n_own, graph.n_edges, graph.row_ptr[:n_own + 1], graph.col, graph.edge_vec,
                        graph.csc_ptr, graph.csc_edge, graph.csc_dst)
        return self.plan.conv_forward(fwd, x_ext, w)

    def conv_backward(self, graph, x_ext, w, grad_out_ext):
        return self.plan.conv_backward(graph, x_ext, w, grad_out_ext)

    def forces(self, graph, grad_edge_vec):
        from . import api
        return api.forces(graph, grad_edge_vec)
