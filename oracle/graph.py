"""Brute-force all-pairs neighbour list, CSR by destination, CSC by source.

Test infrastructure only (see ``oracle/__init__``).

The convolution runs over directed edges j -> i for every pair within the
cutoff ("LunaTP: Enabling Efficient and Scalable Tensor Product for
Equivariant MLIPs", abstract: node-centric CGTP convolutions; the pair loops
of "AccelNet" (pith.science review), direct path).  The bit-exact contract:

* positions are fp32 and are upcast to fp64 before any arithmetic;
* d = p_j - p_i per axis in fp64;
* periodic box of side L (fp32, upcast): d <- d - L * rint(d / L), each
  operation rounded separately, rint rounding halves to even;
* the pair is an edge when ((dx*dx + dy*dy) + dz*dz) < rc*rc, each product
  and sum rounded separately in fp64 (no fused multiply-add), with
  rc*rc formed in fp64 from the fp32 cutoff; i != j;
* with graph ids, only pairs of the same graph are candidates;
* edges are ordered by destination i ascending, then source j ascending
  (CSR rows by destination); the edge vector is (float32) d, i.e. it points
  from the centre i to the neighbour j.

The CSC view lists, for each source j, the edges leaving j in ascending
destination order: csc_ptr[j]..csc_ptr[j+1] index into csc_edge (the CSR edge
number) and csc_dst (its destination).
"""
import numpy as np


def pair_displacements(pos, box=None):
    """fp64 d[i, j] = p_j - p_i with the minimum-image shift, shape [N, N, 3]."""
    p = np.asarray(pos, dtype=np.float32).astype(np.float64)
    d = p[None, :, :] - p[:, None, :]
    if box is not None:
        L = np.float64(np.float32(box))
        q = d / L
        d = d - L * np.rint(q)
    return d


def neighbour_list(pos, rc, box=None, graph_id=None, rows=None):
    """All-pairs neighbour list.

    Returns dict with row_ptr [N+1] int32, col [E] int32 (source j of each
    edge), edge_vec [E, 3] float32, and the CSC arrays csc_ptr [N+1],
    csc_edge [E], csc_dst [E] (int32).  ``rows`` (optional) restricts the
    computation to those destination rows and returns only per-row lists
    (used to sample huge graphs): then the result is {i: (cols, vecs)}.
    """
    p = np.asarray(pos, dtype=np.float32).astype(np.float64)
    n = p.shape[0]
    rc64 = np.float64(np.float32(rc))
    rc2 = rc64 * rc64
    L = None if box is None else np.float64(np.float32(box))
    if L is not None and not rc64 < L / 2:
        raise ValueError("minimum image needs rc < box / 2")
    gid = None if graph_id is None else np.asarray(graph_id)

    def row(i):
        d = p - p[i]
        if L is not None:
            d = d - L * np.rint(d / L)
        r2 = (d[:, 0] * d[:, 0] + d[:, 1] * d[:, 1]) + d[:, 2] * d[:, 2]
        mask = r2 < rc2
        mask[i] = False
        if gid is not None:
            mask &= gid == gid[i]
        js = np.nonzero(mask)[0]
        return js.astype(np.int32), d[js].astype(np.float32)

    if rows is not None:
        return {int(i): row(int(i)) for i in rows}

    cols, vecs, counts = [], [], np.zeros(n, dtype=np.int64)
    for i in range(n):
        js, dv = row(i)
        cols.append(js)
        vecs.append(dv)
        counts[i] = js.size
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col = np.concatenate(cols) if n else np.zeros(0, np.int32)
    edge_vec = np.concatenate(vecs) if n else np.zeros((0, 3), np.float32)
    out = dict(row_ptr=row_ptr.astype(np.int32), col=col.astype(np.int32),
               edge_vec=edge_vec.astype(np.float32).reshape(-1, 3))
    out.update(csr_to_csc(out["row_ptr"], out["col"], n))
    return out


def edge_dst(row_ptr):
    """Destination (CSR row) of every edge."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    return np.repeat(np.arange(row_ptr.size - 1), np.diff(row_ptr)).astype(np.int32)


def csr_to_csc(row_ptr, col, n_nodes):
    """CSC by source: edges grouped by col ascending, each group by dst ascending."""
    col = np.asarray(col, dtype=np.int64)
    dst = edge_dst(row_ptr).astype(np.int64)
    order = np.lexsort((dst, col))  # primary key col, secondary dst
    counts = np.bincount(col, minlength=n_nodes) if col.size else np.zeros(n_nodes, np.int64)
    csc_ptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.cumsum(counts, out=csc_ptr[1:])
    return dict(csc_ptr=csc_ptr.astype(np.int32), csc_edge=order.astype(np.int32),
                csc_dst=dst[order].astype(np.int32))


def neighbour_list_all_pairs_matrix(pos, rc, box=None, graph_id=None):
    """Second, fully vectorised route (dense N x N mask) for cross-checking the
    row loop on small inputs: returns (dst, src) pairs in CSR order."""
    d = pair_displacements(pos, box)
    rc64 = np.float64(np.float32(rc))
    r2 = (d[..., 0] * d[..., 0] + d[..., 1] * d[..., 1]) + d[..., 2] * d[..., 2]
    mask = r2 < rc64 * rc64
    np.fill_diagonal(mask, False)
    if graph_id is not None:
        g = np.asarray(graph_id)
        mask &= g[:, None] == g[None, :]
    i, j = np.nonzero(mask)  # row-major: i ascending, then j ascending
    return i.astype(np.int32), j.astype(np.int32), d[i, j].astype(np.float32)
