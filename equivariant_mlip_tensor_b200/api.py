"""Python binding of libcgtp.so over torch CUDA tensors.

Argument marshalling only: every step runs in the library's kernels; torch
supplies device memory and the current stream.  Tensors must be CUDA,
contiguous, fp32 (features, weights, vectors) or int32 (indices), in the
layouts of include/cgtp.h.
"""
import ctypes
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from ._lib import call, lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(t, dtype, name):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def n_paths(lmax_in, lmax_sh, lmax_out):
    return sum(1 for l1 in range(lmax_in + 1) for l2 in range(lmax_sh + 1)
               for l3 in range(abs(l1 - l2), min(l1 + l2, lmax_out) + 1))


# plan modes of the C ABI (cgtp_mode)
MODES = {"conv": 0, "pair": 1, "conv_shared": 2, "uvw": 3}


def supported(lmax_in, lmax_sh, lmax_out, mode="conv"):
    return bool(lib().cgtp_supported(lmax_in, lmax_sh, lmax_out, MODES[mode]))


def cg_block(l1, l2, l3):
    """Dense real CG block of one path from the library's host generator (no GPU)."""
    import numpy as np
    out = np.zeros((2 * l1 + 1) * (2 * l2 + 1) * (2 * l3 + 1), dtype=np.float64)
    call("cgtp_cg_block", l1, l2, l3, out.ctypes.data_as(ctypes.c_void_p))
    return out.reshape(2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1)


@dataclass
class Graph:
    n_nodes: int
    n_edges: int
    row_ptr: torch.Tensor   # [N+1] int32
    col: torch.Tensor       # [E] int32, source of each edge
    edge_vec: torch.Tensor  # [E][3] fp32, pos_src - pos_dst
    csc_ptr: torch.Tensor   # [N+1] int32
    csc_edge: torch.Tensor  # [E] int32
    csc_dst: torch.Tensor   # [E] int32


def build_graph(pos, rc, box=None, graph_ptr=None, max_edges=None, n_edges_out=None):
    """Neighbour list on the device.  Reads the edge count back once (4 bytes);
    if it exceeds the capacity, rebuilds with exactly enough room."""
    _check(pos, torch.float32, "pos")
    _check(graph_ptr, torch.int32, "graph_ptr")
    n = pos.shape[0]
    dev = pos.device
    if max_edges is None:
        max_edges = max(64, 64 * n)
    while True:
        row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
        csc_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
        col = torch.empty(max(max_edges, 1), dtype=torch.int32, device=dev)
        ev = torch.empty((max(max_edges, 1), 3), dtype=torch.float32, device=dev)
        ce = torch.empty(max(max_edges, 1), dtype=torch.int32, device=dev)
        cd = torch.empty(max(max_edges, 1), dtype=torch.int32, device=dev)
        ne = n_edges_out if n_edges_out is not None else torch.empty(1, dtype=torch.int32, device=dev)
        call("cgtp_graph_build", _ptr(pos), n, ctypes.c_float(0.0 if box is None else float(box)),
             ctypes.c_float(float(rc)), _ptr(graph_ptr), 0 if graph_ptr is None else graph_ptr.numel() - 1,
             _ptr(row_ptr), _ptr(col), _ptr(ev), _ptr(csc_ptr), _ptr(ce), _ptr(cd), max_edges, _ptr(ne),
             _stream())
        E = int(ne.item())
        if E <= max_edges:
            return Graph(n, E, row_ptr, col[:E], ev[:E], csc_ptr, ce[:E], cd[:E])
        max_edges = E


def csr_transpose(n, row_ptr, col):
    """(csc_ptr, csc_edge, csc_dst) of an arbitrary CSR graph."""
    _check(row_ptr, torch.int32, "row_ptr")
    _check(col, torch.int32, "col")
    E = col.numel()
    dev = row_ptr.device
    csc_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
    ce = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
    cd = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
    ws = torch.empty(max(n, 1), dtype=torch.int32, device=dev)
    call("cgtp_csr_transpose", n, E, _ptr(row_ptr), _ptr(col), _ptr(csc_ptr), _ptr(ce), _ptr(cd), _ptr(ws),
         ws.numel() * 4, _stream())
    return csc_ptr, ce[:E], cd[:E]


def graph_check(n, row_ptr, col, edge_vec):
    """Device-side validation flags (see cgtp_graph_check)."""
    flags = torch.empty(1, dtype=torch.int32, device=row_ptr.device)
    call("cgtp_graph_check", n, col.numel(), _ptr(row_ptr), _ptr(col), _ptr(edge_vec), _ptr(flags), _stream())
    return int(flags.item())


def spherical_harmonics(lmax_sh, edge_vec, with_grad=False):
    _check(edge_vec, torch.float32, "edge_vec")
    E = edge_vec.shape[0]
    NS = (lmax_sh + 1) ** 2
    Y = torch.empty((E, NS), dtype=torch.float32, device=edge_vec.device)
    dY = torch.empty((E, NS, 3), dtype=torch.float32, device=edge_vec.device) if with_grad else None
    call("cgtp_spherical_harmonics", lmax_sh, E, _ptr(edge_vec), _ptr(Y), _ptr(dY), _stream())
    return (Y, dY) if with_grad else Y


def forces(graph, grad_edge_vec, out=None):
    _check(grad_edge_vec, torch.float32, "grad_edge_vec")
    if out is None:
        out = torch.empty((graph.n_nodes, 3), dtype=torch.float32, device=grad_edge_vec.device)
    call("cgtp_forces", graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.csc_ptr),
         _ptr(graph.csc_edge), _ptr(grad_edge_vec), _ptr(out), _stream())
    return out


def gather_rows(idx, src, out=None):
    """out[k] = src[idx[k]] (rows of src's trailing shape)."""
    _check(idx, torch.int32, "idx")
    _check(src, torch.float32, "src")
    n, rf = idx.numel(), int(np.prod(src.shape[1:]))
    if out is None:
        out = torch.empty((n,) + tuple(src.shape[1:]), dtype=torch.float32, device=src.device)
    call("cgtp_gather_rows", n, rf, _ptr(idx), _ptr(src), _ptr(out), _stream())
    return out


def scatter_add_rows(idx, src, dst):
    """dst[idx[k]] += src[k] (idx without repeats); returns dst."""
    _check(idx, torch.int32, "idx")
    _check(src, torch.float32, "src")
    _check(dst, torch.float32, "dst")
    n = idx.numel()
    rf = int(np.prod(dst.shape[1:])) if dst.dim() > 1 else 1
    call("cgtp_scatter_add_rows", n, rf, _ptr(idx), _ptr(src), _ptr(dst), _stream())
    return dst


class Plan:
    """Paths and CG coefficients of one irreps shape (lmax_in, lmax_sh, lmax_out, mult).

    The C library takes one plan per mode (what the plan computes: "conv", the
    channelwise convolution; "pair", the edge-free product and its CP
    surrogate; "conv_shared", the convolution with one weight row per edge
    for every path; "uvw", the fully connected convolution).  This object
    holds the plan of ``mode`` and creates the plan of another mode of the
    same shape the first time one of that mode's methods is called."""

    def __init__(self, lmax_in, lmax_sh, lmax_out, mult, mode="conv"):
        self.lmax_in, self.lmax_sh, self.lmax_out, self.mult = lmax_in, lmax_sh, lmax_out, mult
        self.mode = mode
        self._handles = {}
        self._checked = False
        h = self.handle(mode)
        n = ctypes.c_int()
        nnz = ctypes.c_int()
        call("cgtp_plan_info", h, ctypes.byref(n), None, ctypes.byref(nnz))
        buf = (ctypes.c_int * (3 * n.value))()
        call("cgtp_plan_info", h, ctypes.byref(n), ctypes.cast(buf, ctypes.c_void_p), ctypes.byref(nnz))
        self.n_paths = n.value
        self.n_cg_nonzero = nnz.value
        self.paths = [tuple(buf[3 * k:3 * k + 3]) for k in range(n.value)]
        self.ni, self.ns, self.no = (lmax_in + 1) ** 2, (lmax_sh + 1) ** 2, (lmax_out + 1) ** 2

    def handle(self, mode=None):
        """The C plan (cgtp_plan) of ``mode`` (default: this plan's own)."""
        mode = self.mode if mode is None else mode
        h = self._handles.get(mode)
        if h is None:
            h = ctypes.c_void_p()
            call("cgtp_plan_create", self.lmax_in, self.lmax_sh, self.lmax_out, self.mult, MODES[mode],
                 ctypes.byref(h))
            self._handles[mode] = h
            if self._checked:
                call("cgtp_plan_set_checked", h, 1)
        return h

    @property
    def _h(self):
        return self.handle()

    def set_checked(self, on=True):
        """Checked mode for every plan of this object (see cgtp_plan_set_checked)."""
        self._checked = bool(on)
        for h in self._handles.values():
            call("cgtp_plan_set_checked", h, 1 if on else 0)

    def check(self):
        """Flags recorded by checked-mode calls (0 = every graph was valid);
        synchronises the device and clears them."""
        flags = 0
        for h in self._handles.values():
            f = ctypes.c_int()
            st = lib().cgtp_plan_check(h, ctypes.byref(f))
            if st not in (0, 3):  # CGTP_OK, CGTP_ERR_BAD_GRAPH
                call("cgtp_plan_check", h, None)  # raises with the status
            flags |= f.value
        return flags

    def __del__(self):
        for h in getattr(self, "_handles", {}).values():
            if h is not None and h.value:
                try:
                    lib().cgtp_plan_destroy(h)
                except Exception:
                    pass
        self._handles = {}

    # ------------------------------------------------------------ convolution
    def conv_forward(self, graph, x, w, out=None):
        _check(x, torch.float32, "x")
        _check(w, torch.float32, "w")
        if out is None:
            out = torch.empty((graph.n_nodes, self.no, self.mult), dtype=torch.float32, device=x.device)
        call("cgtp_conv_forward", self.handle("conv"), graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.col),
             _ptr(graph.edge_vec), _ptr(x), _ptr(w), _ptr(out), _stream())
        return out

    def conv_backward_workspace_bytes(self, n_edges):
        b = ctypes.c_size_t()
        call("cgtp_conv_backward_workspace_size", self.handle("conv"), n_edges, ctypes.byref(b))
        return b.value

    def conv_backward(self, graph, x, w, grad_out, want_x=True, want_w=True, want_r=True,
                      grad_x=None, grad_w=None, grad_edge_vec=None, workspace=None):
        _check(x, torch.float32, "x")
        _check(w, torch.float32, "w")
        _check(grad_out, torch.float32, "grad_out")
        dev = x.device
        E = graph.n_edges
        if want_x and grad_x is None:
            grad_x = torch.empty((graph.n_nodes, self.ni, self.mult), dtype=torch.float32, device=dev)
        if want_w and grad_w is None:
            grad_w = torch.empty((E, self.n_paths, self.mult), dtype=torch.float32, device=dev)
        if want_r and grad_edge_vec is None:
            grad_edge_vec = torch.empty((E, 3), dtype=torch.float32, device=dev)
        ws_bytes = 0
        if want_r:
            ws_bytes = self.conv_backward_workspace_bytes(E)
            if workspace is None:
                workspace = torch.empty(max(ws_bytes // 4, 64), dtype=torch.float32, device=dev)
        call("cgtp_conv_backward", self.handle("conv"), graph.n_nodes, E, _ptr(graph.csc_ptr), _ptr(graph.csc_edge),
             _ptr(graph.csc_dst), _ptr(graph.edge_vec), _ptr(x), _ptr(w), _ptr(grad_out),
             _ptr(grad_x if want_x else None), _ptr(grad_w if want_w else None),
             _ptr(grad_edge_vec if want_r else None), _ptr(workspace if want_r else None),
             workspace.numel() * 4 if (want_r and workspace is not None) else 0, _stream())
        return (grad_x if want_x else None, grad_w if want_w else None, grad_edge_vec if want_r else None)

    def conv_double_backward_workspace_bytes(self, n_edges):
        b = ctypes.c_size_t()
        call("cgtp_conv_double_backward_workspace_size", self.handle("conv"), n_edges, ctypes.byref(b))
        return b.value

    def conv_double_backward(self, graph, x, w, grad_out, gg_x=None, gg_w=None, gg_edge_vec=None,
                             want_x=True, want_w=True, want_grad_out=True, want_r=True, workspace=None):
        """Adjoint of conv_backward: gradients of <gg_x, grad_x> + <gg_w, grad_w>
        + <gg_edge_vec, grad_edge_vec> with respect to (x, w, grad_out, edge_vec)."""
        for t, nm in ((x, "x"), (w, "w"), (grad_out, "grad_out")):
            _check(t, torch.float32, nm)
        for t, nm in ((gg_x, "gg_x"), (gg_w, "gg_w"), (gg_edge_vec, "gg_edge_vec")):
            if t is not None:
                _check(t, torch.float32, nm)
        dev = x.device
        E = graph.n_edges
        d_x = torch.empty_like(x) if want_x else None
        d_w = torch.empty((E, self.n_paths, self.mult), dtype=torch.float32, device=dev) if want_w else None
        d_g = torch.empty_like(grad_out) if want_grad_out else None
        d_r = torch.empty((E, 3), dtype=torch.float32, device=dev) if want_r else None
        nb = 0
        if want_r or gg_edge_vec is not None:
            nb = self.conv_double_backward_workspace_bytes(E)
            if workspace is None:
                workspace = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=dev)
        call("cgtp_conv_double_backward", self.handle("conv"), graph.n_nodes, E, _ptr(graph.row_ptr), _ptr(graph.col),
             _ptr(graph.csc_ptr), _ptr(graph.csc_edge), _ptr(graph.csc_dst), _ptr(graph.edge_vec), _ptr(x),
             _ptr(w), _ptr(grad_out), _ptr(gg_x), _ptr(gg_w), _ptr(gg_edge_vec), _ptr(d_x), _ptr(d_w), _ptr(d_g),
             _ptr(d_r), _ptr(workspace if nb else None), workspace.numel() * 4 if (nb and workspace is not None) else 0,
             _stream())
        return d_x, d_w, d_g, d_r

    def uvw_forward_workspace_bytes(self, n_nodes, mult_out):
        b = ctypes.c_size_t()
        call("cgtp_uvw_forward_workspace_size", self.handle("uvw"), n_nodes, mult_out, ctypes.byref(b))
        return b.value

    def uvw_forward(self, graph, x, w, mix, out=None, workspace=None):
        """Fully connected convolution: per-path messages mixed by mix [P][mult][mult_out]."""
        for t, nm in ((x, "x"), (w, "w"), (mix, "mix")):
            _check(t, torch.float32, nm)
        mult_out = mix.shape[2]
        if out is None:
            out = torch.empty((graph.n_nodes, self.no, mult_out), dtype=torch.float32, device=x.device)
        nb = self.uvw_forward_workspace_bytes(graph.n_nodes, mult_out)
        if workspace is None:
            workspace = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=x.device)
        call("cgtp_uvw_forward", self.handle("uvw"), graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.col),
             _ptr(graph.edge_vec), _ptr(x), _ptr(w), _ptr(mix), mult_out, _ptr(out), _ptr(workspace),
             workspace.numel() * 4, _stream())
        return out

    def uvw_backward_workspace_bytes(self, n_nodes, n_edges, mult_out):
        b = ctypes.c_size_t()
        call("cgtp_uvw_backward_workspace_size", self.handle("uvw"), n_nodes, n_edges, mult_out, ctypes.byref(b))
        return b.value

    def uvw_backward(self, graph, x, w, mix, grad_out, want_x=True, want_w=True, want_mix=True, want_r=True,
                     workspace=None):
        """Adjoint of uvw_forward: (grad_x, grad_w, grad_mix, grad_edge_vec)."""
        for t, nm in ((x, "x"), (w, "w"), (mix, "mix"), (grad_out, "grad_out")):
            _check(t, torch.float32, nm)
        dev = x.device
        E, mult_out = graph.n_edges, mix.shape[2]
        gx = torch.empty_like(x) if want_x else None
        gw = torch.empty((E, self.n_paths, self.mult), dtype=torch.float32, device=dev) if want_w else None
        gm = torch.empty_like(mix) if want_mix else None
        gr = torch.empty((E, 3), dtype=torch.float32, device=dev) if want_r else None
        nb = self.uvw_backward_workspace_bytes(graph.n_nodes, E, mult_out)
        if workspace is None:
            workspace = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=dev)
        call("cgtp_uvw_backward", self.handle("uvw"), graph.n_nodes, E, _ptr(graph.row_ptr), _ptr(graph.col),
             _ptr(graph.csc_ptr), _ptr(graph.csc_edge), _ptr(graph.csc_dst), _ptr(graph.edge_vec), _ptr(x), _ptr(w),
             _ptr(mix), mult_out, _ptr(grad_out), _ptr(gx), _ptr(gw), _ptr(gm), _ptr(gr), _ptr(workspace),
             workspace.numel() * 4, _stream())
        return gx, gw, gm, gr

    def conv_forward_shared(self, graph, x, w, out=None):
        """Convolution with one weight row per edge for every path: w [E][mult]."""
        _check(x, torch.float32, "x")
        _check(w, torch.float32, "w")
        if out is None:
            out = torch.empty((graph.n_nodes, self.no, self.mult), dtype=torch.float32, device=x.device)
        call("cgtp_conv_forward", self.handle("conv_shared"), graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr),
             _ptr(graph.col), _ptr(graph.edge_vec), _ptr(x), _ptr(w), _ptr(out), _stream())
        return out

    def conv_backward_shared(self, graph, x, w, grad_out, want_x=True, want_w=True, want_r=True, workspace=None):
        """Adjoint of conv_forward_shared: (grad_x, grad_w [E][mult], grad_edge_vec)."""
        for t, nm in ((x, "x"), (w, "w"), (grad_out, "grad_out")):
            _check(t, torch.float32, nm)
        dev, E = x.device, graph.n_edges
        gx = torch.empty_like(x) if want_x else None
        gw = torch.empty((E, self.mult), dtype=torch.float32, device=dev) if want_w else None
        gr = torch.empty((E, 3), dtype=torch.float32, device=dev) if want_r else None
        nb = 0
        if want_r:
            b = ctypes.c_size_t()
            call("cgtp_conv_backward_workspace_size", self.handle("conv_shared"), E, ctypes.byref(b))
            nb = b.value
        if want_r and workspace is None:
            workspace = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=dev)
        call("cgtp_conv_backward", self.handle("conv_shared"), graph.n_nodes, E, _ptr(graph.csc_ptr),
             _ptr(graph.csc_edge), _ptr(graph.csc_dst), _ptr(graph.edge_vec), _ptr(x), _ptr(w), _ptr(grad_out),
             _ptr(gx), _ptr(gw), _ptr(gr), _ptr(workspace if want_r else None),
             workspace.numel() * 4 if (want_r and workspace is not None) else 0, _stream())
        return gx, gw, gr

    # ------------------------------------------------------------ radial network
    def _radial_mode(self):
        return self.mode if self.mode in ("conv", "conv_shared", "uvw") else "conv"

    def radial_forward(self, edge_vec, rc, W1, W2, out=None):
        """Per-edge weights of the plan's mode: [E][n_paths][mult], or [E][mult]
        for "conv_shared"."""
        _check(edge_vec, torch.float32, "edge_vec")
        _check(W1, torch.float32, "W1")
        _check(W2, torch.float32, "W2")
        E = edge_vec.shape[0]
        if out is None:
            shape = (E, self.mult) if self._radial_mode() == "conv_shared" else (E, self.n_paths, self.mult)
            out = torch.empty(shape, dtype=torch.float32, device=edge_vec.device)
        call("cgtp_radial_forward", self.handle(self._radial_mode()), E, _ptr(edge_vec), ctypes.c_float(float(rc)), _ptr(W1), _ptr(W2),
             _ptr(out), _stream())
        return out

    def radial_backward(self, edge_vec, rc, W1, W2, grad_w, grad_edge_vec):
        """Adds dL/d edge_vec through the weights into grad_edge_vec (in place)."""
        _check(grad_w, torch.float32, "grad_w")
        _check(grad_edge_vec, torch.float32, "grad_edge_vec")
        call("cgtp_radial_backward", self.handle(self._radial_mode()), edge_vec.shape[0], _ptr(edge_vec), ctypes.c_float(float(rc)),
             _ptr(W1), _ptr(W2), _ptr(grad_w), _ptr(grad_edge_vec), _stream())
        return grad_edge_vec

    # ------------------------------------------------------------ edge-free product
    def tp_forward(self, x, y, w, out=None):
        for t, nm in ((x, "x"), (y, "y"), (w, "w")):
            _check(t, torch.float32, nm)
        B = x.shape[0]
        if out is None:
            out = torch.empty((B, self.no, self.mult), dtype=torch.float32, device=x.device)
        call("cgtp_tp_forward", self.handle("pair"), B, _ptr(x), _ptr(y), _ptr(w), _ptr(out), _stream())
        return out

    def tp_backward(self, x, y, w, grad_z, want_x=True, want_y=True, want_w=True):
        B = x.shape[0]
        dev = x.device
        gx = torch.empty_like(x) if want_x else None
        gy = torch.empty_like(y) if want_y else None
        gw = torch.empty_like(w) if want_w else None
        ws = None
        nb = 0
        if want_w:
            b = ctypes.c_size_t()
            call("cgtp_tp_backward_workspace_size", self.handle("pair"), B, ctypes.byref(b))
            nb = b.value
            ws = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=dev)
        call("cgtp_tp_backward", self.handle("pair"), B, _ptr(x), _ptr(y), _ptr(w), _ptr(grad_z), _ptr(gx), _ptr(gy),
             _ptr(gw), _ptr(ws), nb, _stream())
        return gx, gy, gw

    # ------------------------------------------------------------ CP-decomposed product
    def cp_forward(self, A, B, C, x, y, out=None):
        """z = A (B^T x (*) C^T y) per (pair, channel); A [d3][R], B [d1][R], C [d2][R]."""
        for t, nm in ((A, "A"), (B, "B"), (C, "C"), (x, "x"), (y, "y")):
            _check(t, torch.float32, nm)
        R, batch = A.shape[1], x.shape[0]
        if out is None:
            out = torch.empty((batch, (self.lmax_out + 1) ** 2, self.mult), dtype=torch.float32, device=x.device)
        call("cgtp_cp_forward", self.handle("pair"), R, batch, _ptr(A), _ptr(B), _ptr(C), _ptr(x), _ptr(y), _ptr(out),
             _stream())
        return out

    def cp_backward_workspace_bytes(self, rank, batch):
        b = ctypes.c_size_t()
        call("cgtp_cp_backward_workspace_size", self.handle("pair"), rank, batch, ctypes.byref(b))
        return b.value

    def cp_backward(self, A, B, C, x, y, grad_z, want_x=True, want_y=True, want_factors=True):
        """(grad_x, grad_y, grad_A, grad_B, grad_C); the unrequested ones are None."""
        for t, nm in ((A, "A"), (B, "B"), (C, "C"), (x, "x"), (y, "y"), (grad_z, "grad_z")):
            _check(t, torch.float32, nm)
        R, batch = A.shape[1], x.shape[0]
        gx = torch.empty_like(x) if want_x else None
        gy = torch.empty_like(y) if want_y else None
        gA, gB, gC = (torch.empty_like(v) if want_factors else None for v in (A, B, C))
        ws, nb = None, 0
        if want_factors:
            nb = self.cp_backward_workspace_bytes(R, batch)
            ws = torch.empty(max(nb // 4, 64), dtype=torch.float32, device=x.device)
        call("cgtp_cp_backward", self.handle("pair"), R, batch, _ptr(A), _ptr(B), _ptr(C), _ptr(x), _ptr(y), _ptr(grad_z),
             _ptr(gx), _ptr(gy), _ptr(gA), _ptr(gB), _ptr(gC), _ptr(ws), nb, _stream())
        return gx, gy, gA, gB, gC
