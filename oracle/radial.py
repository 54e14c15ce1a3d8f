"""Radial network that makes the per-edge, per-path, per-channel weights (fp64).

Test infrastructure only (see ``oracle/__init__``).

The convolution scales each path by per-edge, per-path, per-channel radial
weights ("LunaTP ...", abstract: CGTP convolutions; the synthetic workloads
draw them from a small network of the edge length).  Readings, since the
pages print no network:

* 8 Gaussian basis functions on [0, rc]: centres mu_k = k rc / 7
  (k = 0..7), width sigma = rc / 7, phi_k(r) = exp(-(r - mu_k)^2 / (2 sigma^2));
* a = phi @ W1 with W1 [8][64], h = SiLU(a) = a / (1 + exp(-a));
* W_e[p][u] = (h @ W2)[p * mult + u] with W2 [64][P * mult];
* no biases, no cutoff envelope;
* r = |r_e| evaluated in fp64 from the fp32 edge vector.

The backward maps grad_W to dL/d r_e through the chain
dL/dr = sum_k (grad_W @ W2^T)_k SiLU'(a_k) (W1 @ dphi/dr)_k, and
dL/d r_e = dL/dr * r_e / |r_e| (zero for a zero-length edge).
"""
import numpy as np

N_BASIS = 8
HIDDEN = 64


def _basis(r, rc):
    mu = np.arange(N_BASIS) * (rc / (N_BASIS - 1))
    sigma = rc / (N_BASIS - 1)
    diff = r[:, None] - mu[None, :]
    phi = np.exp(-diff * diff / (2.0 * sigma * sigma))
    dphi = -diff / (sigma * sigma) * phi
    return phi, dphi


def _silu(a):
    s = 1.0 / (1.0 + np.exp(-a))
    return a * s, s * (1.0 + a * (1.0 - s))


def radial_forward(edge_vec, W1, W2, rc, n_paths, mult):
    """W [E][n_paths][mult] in fp64."""
    v = np.asarray(edge_vec, dtype=np.float64)
    r = np.sqrt(np.sum(v * v, axis=1))
    phi, _ = _basis(r, float(np.float32(rc)))
    a = phi @ np.asarray(W1, dtype=np.float64)
    h, _ = _silu(a)
    return (h @ np.asarray(W2, dtype=np.float64)).reshape(-1, n_paths, mult)


def radial_backward(edge_vec, W1, W2, rc, grad_w):
    """dL/d r_e [E][3] contributed through the weights, in fp64."""
    v = np.asarray(edge_vec, dtype=np.float64)
    r = np.sqrt(np.sum(v * v, axis=1))
    phi, dphi = _basis(r, float(np.float32(rc)))
    W1 = np.asarray(W1, dtype=np.float64)
    W2 = np.asarray(W2, dtype=np.float64)
    a = phi @ W1
    _, dsilu = _silu(a)
    gh = np.asarray(grad_w, dtype=np.float64).reshape(r.size, -1) @ W2.T
    dr = np.sum(gh * dsilu * (dphi @ W1), axis=1)
    safe = np.where(r > 0, r, 1.0)
    out = dr[:, None] * v / safe[:, None]
    out[r == 0] = 0.0
    return out
