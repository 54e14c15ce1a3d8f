"""Edge-free channelwise CG tensor product of batched pairs, and its adjoints.

Test infrastructure only (see ``oracle/__init__``).

"Tensor Decomposition Networks ...", reply to reviewer S6y1: the exact CG
tensor product of two irreps inputs x and y (the map the CP factors
approximate), timed at batch 1000 and multiplicity 128.  Channelwise form,
with one weight per path and channel (a scalar per path is the special case
of a weight constant over channels):

    z[b][l3,m3][u] = sum_{p=(l1,l2,l3)} w[p][u] sum_{m1,m2} C^p[m1,m2,m3]
                     x[b][l1,m1][u] y[b][l2,m2][u]

Adjoints (the closed-form gradients of a bilinear map, as written in the same
reply for the CP form): grad_x and grad_y contract grad_z with the other
operand; grad_w sums over the batch.
"""
import numpy as np

from .conv import path_nonzeros


def tp_forward(x, y, w, lmax_in, lmax_sh, lmax_out):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, _, u = x.shape
    z = np.zeros((B, (lmax_out + 1) ** 2, u))
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        z[:, ro, :] += c * w[p][None, :] * x[:, ri, :] * y[:, rs, :]
    return z


def tp_backward(x, y, w, grad_z, lmax_in, lmax_sh, lmax_out):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(grad_z, dtype=np.float64)
    gx = np.zeros_like(x)
    gy = np.zeros_like(y)
    gw = np.zeros_like(w)
    for p, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        gx[:, ri, :] += c * w[p][None, :] * y[:, rs, :] * g[:, ro, :]
        gy[:, rs, :] += c * w[p][None, :] * x[:, ri, :] * g[:, ro, :]
        gw[p] += c * np.sum(x[:, ri, :] * y[:, rs, :] * g[:, ro, :], axis=0)
    return gx, gy, gw
