"""The CGTP convolution, its adjoints and the per-atom forces (fp64).

Test infrastructure only (see ``oracle/__init__``).

Definition ("LunaTP: Enabling Efficient and Scalable Tensor Product for
Equivariant MLIPs", abstract: CGTP convolutions; selection rules from "Tensor
Decomposition Networks ...", reply to reviewer S6y1).  For every edge
e = (j -> i) with edge vector r_e, real harmonics Y_e = Y(r_e/|r_e|) and
weights W_e[p][u]:

    out[i][l3, m3][u] = sum_{e in row i} sum_{p=(l1,l2,l3)} W_e[p][u]
                        sum_{m1,m2} C^p[m1,m2,m3] x[j][l1,m1][u] Y_e[l2,m2]

Readings where the pages are silent: no normalisation constants (no
1/sqrt(degree), no path normalisation); paths that share l3 are summed into
one output block; feature layout [node][l*l + m + l][u].

This module evaluates the sum literally: every path, every nonzero
(m1, m2, m3), every edge, vectorised only over channels and edge chunks.  It
does not factor the per-edge matrix sum_m2 C Y out of the channel loop.

Backward (the bilinear adjoints of the same sum, cf. the closed-form
gradients of a bilinear tensor product in the reply to reviewer S6y1):

    grad_x[j][l1,m1][u] = sum_{e: src=j} sum_p W_e[p][u] sum_{m2,m3} C Y_e[l2,m2] g[i][l3,m3][u]
    grad_W[e][p][u]     = sum_{m1,m2,m3} C x[j][l1,m1][u] Y_e[l2,m2] g[i][l3,m3][u]
    grad_Y[e][l2,m2]    = sum_p sum_{m1,m3} C sum_u W_e[p][u] x[j][l1,m1][u] g[i][l3,m3][u]
    grad_r[e]           = (dY_e/dr_e)^T grad_Y[e]

Forces: with r_e = pos_j - pos_i, dE/dpos_j += grad_r[e] and
dE/dpos_i -= grad_r[e]; the force is F = -dE/dpos.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .cg import paths, real_cg
from .graph import edge_dst
from .sh import real_sh, real_sh_hessian, real_sh_jacobian


def path_nonzeros(lmax_in, lmax_sh, lmax_out):
    """[(p, row_in, row_sh, row_out, C)] for every nonzero real CG entry,
    rows being offsets into the concatenated l = 0..L layouts."""
    out = []
    for p, (l1, l2, l3) in enumerate(paths(lmax_in, lmax_sh, lmax_out)):
        C = real_cg(l1, l2, l3)
        for a, b, c in zip(*np.nonzero(C)):
            out.append((p, l1 * l1 + int(a), l2 * l2 + int(b), l3 * l3 + int(c), float(C[a, b, c])))
    return out


def _chunks(n, size):
    return [(s, min(n, s + size)) for s in range(0, n, size)]


def _map_chunks(fn, n, chunk, threads):
    parts = _chunks(n, chunk)
    if threads <= 1 or len(parts) <= 1:
        return [fn(s, e) for s, e in parts]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda se: fn(*se), parts))


def edge_messages(src, edge_vec, x, w, lmax_in, lmax_sh, lmax_out):
    """m[e][l3,m3][u]: the contribution of edge e to its destination row."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    E, u = w.shape[0], x.shape[2]
    Y = real_sh(edge_vec, lmax_sh)
    xs = x[src]
    m = np.zeros((E, (lmax_out + 1) ** 2, u))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        m[:, ro, :] += c * w[:, p, :] * xs[:, ri, :] * Y[:, rs][:, None]
    return m


def conv_forward(row_ptr, col, edge_vec, x, w, lmax_in, lmax_sh, lmax_out,
                 threads=1, chunk=4096):
    """out [N][(lmax_out+1)^2][u] in fp64."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    x = np.asarray(x, dtype=np.float64)
    n, u = row_ptr.size - 1, x.shape[2]
    dst = edge_dst(row_ptr)

    def part(s, e):
        o = np.zeros((n, (lmax_out + 1) ** 2, u))
        m = edge_messages(col[s:e], np.asarray(edge_vec)[s:e], x, np.asarray(w)[s:e],
                          lmax_in, lmax_sh, lmax_out)
        np.add.at(o, dst[s:e], m)
        return o

    out = np.zeros((n, (lmax_out + 1) ** 2, u))
    for o in _map_chunks(part, col.size, chunk, threads):
        out += o
    return out


def conv_forward_rows(row_ptr, col, edge_vec, x, w, lmax_in, lmax_sh, lmax_out, rows):
    """Output rows ``rows`` only (for sampling graphs too large to evaluate)."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    res = []
    for i in rows:
        s, e = row_ptr[i], row_ptr[i + 1]
        m = edge_messages(np.asarray(col)[s:e], np.asarray(edge_vec)[s:e], x,
                          np.asarray(w)[s:e], lmax_in, lmax_sh, lmax_out)
        res.append(m.sum(axis=0))
    return np.stack(res) if res else np.zeros((0, (lmax_out + 1) ** 2, np.asarray(x).shape[2]))


def edge_backward(src, dst, edge_vec, x, w, g, lmax_in, lmax_sh, lmax_out):
    """Per-edge adjoints: (msg_x [E][(lmax_in+1)^2][u], grad_w [E][P][u], grad_r [E][3])."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    E, P, u = w.shape
    Y = real_sh(edge_vec, lmax_sh)
    J = real_sh_jacobian(edge_vec, lmax_sh)
    xs, gd = x[src], g[dst]
    mx = np.zeros((E, (lmax_in + 1) ** 2, u))
    gw = np.zeros((E, P, u))
    gY = np.zeros((E, (lmax_sh + 1) ** 2))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        mx[:, ri, :] += c * w[:, p, :] * Y[:, rs][:, None] * gd[:, ro, :]
        gw[:, p, :] += c * xs[:, ri, :] * Y[:, rs][:, None] * gd[:, ro, :]
        gY[:, rs] += c * np.sum(w[:, p, :] * xs[:, ri, :] * gd[:, ro, :], axis=1)
    gr = np.einsum("eb,ebk->ek", gY, J)
    return mx, gw, gr


def conv_backward(row_ptr, col, edge_vec, x, w, grad_out, lmax_in, lmax_sh, lmax_out,
                  threads=1, chunk=4096):
    """(grad_x [N][(lmax_in+1)^2][u], grad_w [E][P][u], grad_edge_vec [E][3]) in fp64."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w)
    n, u = row_ptr.size - 1, x.shape[2]
    E, P = col.size, w.shape[1]
    dst = edge_dst(row_ptr)
    grad_w = np.zeros((E, P, u))
    grad_r = np.zeros((E, 3))

    def part(s, e):
        gx = np.zeros((n, (lmax_in + 1) ** 2, u))
        mx, gw, gr = edge_backward(col[s:e], dst[s:e], np.asarray(edge_vec)[s:e], x, w[s:e],
                                   grad_out, lmax_in, lmax_sh, lmax_out)
        np.add.at(gx, col[s:e], mx)
        grad_w[s:e] = gw
        grad_r[s:e] = gr
        return gx

    grad_x = np.zeros((n, (lmax_in + 1) ** 2, u))
    for gx in _map_chunks(part, E, chunk, threads):
        grad_x += gx
    return grad_x, grad_w, grad_r


def edge_forces(row_ptr, col, grad_edge_vec, n_nodes):
    """F = -dE/dpos from dE/dr_e, with r_e = pos_src - pos_dst."""
    col = np.asarray(col, dtype=np.int64)
    dst = edge_dst(row_ptr).astype(np.int64)
    gr = np.asarray(grad_edge_vec, dtype=np.float64)
    dEdpos = np.zeros((n_nodes, 3))
    np.add.at(dEdpos, col, gr)
    np.add.at(dEdpos, dst, -gr)
    return -dEdpos


def conv_double_backward(row_ptr, col, edge_vec, x, w, grad_out, gg_x, gg_w, gg_r,
                         lmax_in, lmax_sh, lmax_out):
    """Adjoint of the backward: the gradients of

        L = <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r>

    (grad_x, grad_w, grad_r = conv_backward(x, w, grad_out, edge_vec)) with
    respect to x, w, grad_out and the edge vectors, for cotangents gg_x
    [N][(lmax_in+1)^2][u], gg_w [E][P][u] and gg_r [E][3] (any may be None).
    This is the second derivative that force training needs ("LunaTP ...",
    abstract: higher-order derivative computation).

    Written out per nonzero (p, m1, m2, m3) of each edge e = (j -> i), with
    uY[e] = (dY_e/dr_e) gg_r[e] (the directional derivative of the harmonics)
    and gY[e] the harmonic gradient of the backward, L is

        sum_e sum_nz C sum_u g[i,m3,u] (gg_x[j,m1,u] W[e,p,u] Y[e,m2]
                                        + gg_w[e,p,u] x[j,m1,u] Y[e,m2]
                                        + uY[e,m2] W[e,p,u] x[j,m1,u])

    so that, term by term,
        dL/dg[i,m3,u] = sum_e sum_nz C (gg_x W Y + gg_w x Y + uY W x)
        dL/dx[j,m1,u] = sum_e sum_nz C g (gg_w Y + uY W)
        dL/dW[e,p,u]  = sum_nz(p) C g (gg_x Y + uY x)
        dL/dr_e       = (dY/dr)^T [sum_nz C sum_u g (gg_x W + gg_w x)]
                        + sum_m2 gY[e,m2] (d2Y[e,m2]/dr2) gg_r[e].
    Returns (d_x, d_w, d_grad_out, d_edge_vec) in fp64.
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    src = np.asarray(col, dtype=np.int64)
    dst = edge_dst(row_ptr).astype(np.int64)
    ev = np.asarray(edge_vec, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    n, u = row_ptr.size - 1, x.shape[2]
    E, P = src.size, w.shape[1]
    ns = (lmax_sh + 1) ** 2
    ggx = np.zeros_like(x) if gg_x is None else np.asarray(gg_x, dtype=np.float64)
    ggw = np.zeros_like(w) if gg_w is None else np.asarray(gg_w, dtype=np.float64)
    ggr = np.zeros((E, 3)) if gg_r is None else np.asarray(gg_r, dtype=np.float64)
    Y = real_sh(ev, lmax_sh)
    J = real_sh_jacobian(ev, lmax_sh)
    H = real_sh_hessian(ev, lmax_sh)
    uY = np.einsum("ebk,ek->eb", J, ggr)
    xs, gd, ggxs = x[src], g[dst], ggx[src]
    d_g_edge = np.zeros((E, g.shape[1], u))
    d_x_edge = np.zeros((E, x.shape[1], u))
    d_w = np.zeros((E, P, u))
    dY_expl = np.zeros((E, ns))
    gY = np.zeros((E, ns))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        Yc, uc = Y[:, rs][:, None], uY[:, rs][:, None]
        Wp, ggwp = w[:, p, :], ggw[:, p, :]
        d_g_edge[:, ro, :] += c * (ggxs[:, ri, :] * Wp * Yc + ggwp * xs[:, ri, :] * Yc + uc * Wp * xs[:, ri, :])
        d_x_edge[:, ri, :] += c * gd[:, ro, :] * (ggwp * Yc + uc * Wp)
        d_w[:, p, :] += c * gd[:, ro, :] * (ggxs[:, ri, :] * Yc + uc * xs[:, ri, :])
        dY_expl[:, rs] += c * np.sum(gd[:, ro, :] * (ggxs[:, ri, :] * Wp + ggwp * xs[:, ri, :]), axis=1)
        gY[:, rs] += c * np.sum(Wp * xs[:, ri, :] * gd[:, ro, :], axis=1)
    d_g = np.zeros_like(g)
    np.add.at(d_g, dst, d_g_edge)
    d_x = np.zeros_like(x)
    np.add.at(d_x, src, d_x_edge)
    d_r = np.einsum("eb,ebk->ek", dY_expl, J) + np.einsum("eb,ebjk,ek->ej", gY, H, ggr)
    return d_x, d_w, d_g, d_r


def conv_uvw_forward(row_ptr, col, edge_vec, x, w, mix, lmax_in, lmax_sh, lmax_out):
    """Fully connected ("uvw") convolution: the per-path messages of the
    channelwise convolution, summed over each row but kept per path, then
    mixed across channels by a dense matrix per path ("Tensor Decomposition
    Networks ...", reply to reviewer cmnz: the fully connected CG tensor
    product of Equiformer):

        t[i][p][m3][u]   = sum_{e in row i} W_e[p][u] sum_{m1,m2} C^p x[j][l1,m1][u] Y_e[l2,m2]
        out[i][l3,m3][v] = sum_{p: l3(p) = l3} sum_u t[i][p][m3][u] mix[p][u][v]

    mix is [P][u][v]; out is [N][(lmax_out+1)^2][v] in fp64.  With every
    mix[p] the identity this is conv_forward.
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    src = np.asarray(col, dtype=np.int64)
    dst = edge_dst(row_ptr).astype(np.int64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    mix = np.asarray(mix, dtype=np.float64)
    n, u = row_ptr.size - 1, x.shape[2]
    P, v = mix.shape[0], mix.shape[2]
    Y = real_sh(edge_vec, lmax_sh)
    xs = x[src]
    pl = paths(lmax_in, lmax_sh, lmax_out)
    t = np.zeros((n, P, (lmax_out + 1) ** 2, u))  # rows of l3(p) used only
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        msg = c * w[:, p, :] * xs[:, ri, :] * Y[:, rs][:, None]
        np.add.at(t[:, p, ro, :], dst, msg)
    out = np.zeros((n, (lmax_out + 1) ** 2, v))
    for p, (l1, l2, l3) in enumerate(pl):
        rows = slice(l3 * l3, (l3 + 1) * (l3 + 1))
        out[:, rows, :] += np.einsum("imu,uv->imv", t[:, p, rows, :], mix[p])
    return out


def conv_uvw_backward(row_ptr, col, edge_vec, x, w, mix, grad_out, lmax_in, lmax_sh, lmax_out):
    """Adjoint of conv_uvw_forward for the output gradient g = grad_out
    [N][(lmax_out+1)^2][v]: (grad_x, grad_w, grad_mix, grad_edge_vec) in fp64.

        gt[i][p][m3][u]  = sum_v g[i][l3,m3][v] mix[p][u][v]
        grad_mix[p][u][v] = sum_i sum_m3 t[i][p][m3][u] g[i][l3,m3][v]
    and the channelwise backward with one output gradient per path:
        grad_x[j][l1,m1][u] = sum_{e: src=j} sum_p W_e[p][u] sum C Y_e gt[i][p][m3][u]
        grad_W[e][p][u]     = sum C x[j][l1,m1][u] Y_e gt[i][p][m3][u]
        grad_Y[e][l2,m2]    = sum_p sum C sum_u W_e[p][u] x[j][l1,m1][u] gt[i][p][m3][u]
        grad_r[e]           = (dY_e/dr_e)^T grad_Y[e]
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    src = np.asarray(col, dtype=np.int64)
    dst = edge_dst(row_ptr).astype(np.int64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    mix = np.asarray(mix, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    n, u = row_ptr.size - 1, x.shape[2]
    E, P = src.size, w.shape[1]
    Y = real_sh(edge_vec, lmax_sh)
    J = real_sh_jacobian(edge_vec, lmax_sh)
    xs = x[src]
    pl = paths(lmax_in, lmax_sh, lmax_out)
    no = (lmax_out + 1) ** 2
    t = np.zeros((n, P, no, u))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        np.add.at(t[:, p, ro, :], dst, c * w[:, p, :] * xs[:, ri, :] * Y[:, rs][:, None])
    gt = np.zeros((n, P, no, u))
    grad_mix = np.zeros_like(mix)
    for p, (l1, l2, l3) in enumerate(pl):
        rows = slice(l3 * l3, (l3 + 1) * (l3 + 1))
        gt[:, p, rows, :] = np.einsum("imv,uv->imu", g[:, rows, :], mix[p])
        grad_mix[p] = np.einsum("imu,imv->uv", t[:, p, rows, :], g[:, rows, :])
    gd = gt[dst]  # [E][P][no][u]
    mx = np.zeros((E, x.shape[1], u))
    grad_w = np.zeros((E, P, u))
    gY = np.zeros((E, Y.shape[1]))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        mx[:, ri, :] += c * w[:, p, :] * Y[:, rs][:, None] * gd[:, p, ro, :]
        grad_w[:, p, :] += c * xs[:, ri, :] * Y[:, rs][:, None] * gd[:, p, ro, :]
        gY[:, rs] += c * np.sum(w[:, p, :] * xs[:, ri, :] * gd[:, p, ro, :], axis=1)
    grad_x = np.zeros_like(x)
    np.add.at(grad_x, src, mx)
    grad_r = np.einsum("eb,ebk->ek", gY, J)
    return grad_x, grad_w, grad_mix, grad_r


def conv_forward_shared(row_ptr, col, edge_vec, x, w_shared, lmax_in, lmax_sh, lmax_out):
    """Convolution whose weights are shared by every path (path stride 0:
    W_e[p][u] = w_shared[e][u]; "Tensor Decomposition Networks ...", reply to
    reviewer oXft: path-weight sharing): conv_forward with the one row repeated
    for every path."""
    w_shared = np.asarray(w_shared, dtype=np.float64)
    P = len(paths(lmax_in, lmax_sh, lmax_out))
    return conv_forward(row_ptr, col, edge_vec, x, np.repeat(w_shared[:, None, :], P, axis=1),
                        lmax_in, lmax_sh, lmax_out)


def conv_backward_shared(row_ptr, col, edge_vec, x, w_shared, grad_out, lmax_in, lmax_sh, lmax_out):
    """Adjoint of conv_forward_shared: (grad_x, grad_w_shared [E][u], grad_edge_vec);
    the shared row's gradient is the sum over paths of the per-path ones."""
    w_shared = np.asarray(w_shared, dtype=np.float64)
    P = len(paths(lmax_in, lmax_sh, lmax_out))
    gx, gw, gr = conv_backward(row_ptr, col, edge_vec, x, np.repeat(w_shared[:, None, :], P, axis=1), grad_out,
                               lmax_in, lmax_sh, lmax_out)
    return gx, gw.sum(axis=1), gr

