"""CP-decomposed CG tensor product: the low-rank surrogate of the exact
channelwise product, its adjoints, and the fit of its factors (fp64).

Test infrastructure only (see ``oracle/__init__``).

"Tensor Decomposition Networks for Accelerating Machine Learning Force Field
Computations", reply to reviewer S6y1 (complexity of the backward): with
factor matrices A [d3][R], B [d1][R], C [d2][R] the map of inputs
x [d1], y [d2] is

    z = A (B^T x (*) C^T y)                   ((*) = elementwise product)

and, for an output gradient g_z, the input gradients are

    g_x = (g_z^T A (*) C^T y) B^T,   g_y = (g_z^T A (*) B^T x) C^T.

Same reply, on Figure 3: the factors are fitted once, before training, by
minimising the Frobenius norm between the exact and the approximate product
on batches of standard-normal inputs.  The reply to reviewer S6y1 on the
low-rank structure bounds the rank of the CG tensor by (L+1)^4.

The same reply (on Figure 3) reports the surrogate's SO(3)-equivariance error
against its rank; ``equivariance_error`` measures it for given factors.

Readings (the pages fix none of these):

* R-cp1: the exact map is the plan's channelwise CG product with unit path
  weights, d1 = (L_in+1)^2, d2 = (L_sh+1)^2, d3 = (L_out+1)^2, i.e. the tensor
  M[k][i][j] = sum over paths of the real CG coefficient that couples input
  row i and harmonic row j into output row k.  The factors are shared by every
  pair of a batch and every channel:
  z[b][:, u] = A (B^T x[b][:, u] (*) C^T y[b][:, u]).
* R-cp2: the factor gradients (the reply says they must be computed for
  training but prints no formula) follow from the same trilinear form, summed
  over pairs and channels: with s = B^T x, t = C^T y, q = A^T g_z,
  g_A = sum g_z (s (*) t)^T,  g_B = sum x (q (*) t)^T,  g_C = sum y (q (*) s)^T.
* R-cp3: the fit is alternating least squares on batches: each factor in
  turn takes the exact least-squares solution on a fresh batch of N(0,1)
  inputs (the loss is linear in each factor when the other two are fixed).
  Under N(0,1) inputs the expected batch loss per pair is ||M - M~||_F^2, so
  the same objective is reported as the relative Frobenius error.
"""
import numpy as np

from .cg import paths
from .conv import path_nonzeros
from .tp import tp_forward
from .wigner import block_rotation, random_rotation


def dims(lmax_in, lmax_sh, lmax_out):
    return (lmax_in + 1) ** 2, (lmax_sh + 1) ** 2, (lmax_out + 1) ** 2


def exact_tensor(lmax_in, lmax_sh, lmax_out):
    """M [d3][d1][d2]: the unit-weight CG product as a dense tensor (R-cp1)."""
    d1, d2, d3 = dims(lmax_in, lmax_sh, lmax_out)
    M = np.zeros((d3, d1, d2))
    for _, ri, rs, ro, c in path_nonzeros(lmax_in, lmax_sh, lmax_out):
        M[ro, ri, rs] += c
    return M


def cp_tensor(A, B, C):
    """The tensor of the CP map: sum_r A[:, r] (x) B[:, r] (x) C[:, r]."""
    return np.einsum("kr,ir,jr->kij", A, B, C)


def rel_error(A, B, C, lmax_in, lmax_sh, lmax_out):
    """||M - M~||_F / ||M||_F."""
    M = exact_tensor(lmax_in, lmax_sh, lmax_out)
    return float(np.linalg.norm(M - cp_tensor(A, B, C)) / np.linalg.norm(M))


def cp_forward(A, B, C, x, y):
    """z [batch][d3][u] from x [batch][d1][u], y [batch][d2][u]."""
    A, B, C = (np.asarray(v, dtype=np.float64) for v in (A, B, C))
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    s = np.einsum("ir,biu->bru", B, x)
    t = np.einsum("jr,bju->bru", C, y)
    return np.einsum("kr,bru->bku", A, s * t)


def cp_backward(A, B, C, x, y, grad_z):
    """(g_x, g_y, g_A, g_B, g_C) for the output gradient grad_z."""
    A, B, C = (np.asarray(v, dtype=np.float64) for v in (A, B, C))
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    g = np.asarray(grad_z, dtype=np.float64)
    s = np.einsum("ir,biu->bru", B, x)
    t = np.einsum("jr,bju->bru", C, y)
    q = np.einsum("kr,bku->bru", A, g)
    gx = np.einsum("ir,bru->biu", B, q * t)
    gy = np.einsum("jr,bru->bju", C, q * s)
    gA = np.einsum("bku,bru->kr", g, s * t)
    gB = np.einsum("biu,bru->ir", x, q * t)
    gC = np.einsum("bju,bru->jr", y, q * s)
    return gx, gy, gA, gB, gC


def _exact_pairs(X, Y, lmax_in, lmax_sh, lmax_out):
    """The exact product of single-channel pairs, through the oracle's edge-free
    tensor product with unit path weights."""
    w = np.ones((len(paths(lmax_in, lmax_sh, lmax_out)), 1))
    return tp_forward(X[:, :, None], Y[:, :, None], w, lmax_in, lmax_sh, lmax_out)[:, :, 0]


def fit_als(lmax_in, lmax_sh, lmax_out, rank, rng, n_iter=25, batch=None):
    """Factors (A, B, C) fitted by alternating least squares on batches of
    standard-normal pairs (R-cp3)."""
    d1, d2, d3 = dims(lmax_in, lmax_sh, lmax_out)
    if batch is None:
        batch = 4 * rank * max(d1, d2) + 64
    A = rng.standard_normal((d3, rank)) / np.sqrt(rank)
    B = rng.standard_normal((d1, rank))
    C = rng.standard_normal((d2, rank))
    for _ in range(n_iter):
        X = rng.standard_normal((batch, d1))
        Y = rng.standard_normal((batch, d2))
        Z = _exact_pairs(X, Y, lmax_in, lmax_sh, lmax_out)  # [n][d3]
        # A: Z ~ P A^T with P = (X B) (*) (Y C)
        P = (X @ B) * (Y @ C)
        A = np.linalg.lstsq(P, Z, rcond=None)[0].T
        # B: Z[n, k] = sum_{i, r} X[n, i] A[k, r] (Y C)[n, r] B[i, r]
        D = np.einsum("ni,kr,nr->nkir", X, A, Y @ C).reshape(batch * d3, d1 * rank)
        B = np.linalg.lstsq(D, Z.reshape(-1), rcond=None)[0].reshape(d1, rank)
        # C: Z[n, k] = sum_{j, r} Y[n, j] A[k, r] (X B)[n, r] C[j, r]
        D = np.einsum("nj,kr,nr->nkjr", Y, A, X @ B).reshape(batch * d3, d2 * rank)
        C = np.linalg.lstsq(D, Z.reshape(-1), rcond=None)[0].reshape(d2, rank)
    return A, B, C


def batch_loss(A, B, C, lmax_in, lmax_sh, lmax_out, rng, batch):
    """Mean over a batch of N(0,1) pairs of ||exact(x, y) - CP(x, y)||^2."""
    d1, d2, _ = dims(lmax_in, lmax_sh, lmax_out)
    X = rng.standard_normal((batch, d1))
    Y = rng.standard_normal((batch, d2))
    Z = _exact_pairs(X, Y, lmax_in, lmax_sh, lmax_out)
    Zc = cp_forward(A, B, C, X[:, :, None], Y[:, :, None])[:, :, 0]
    return float(np.mean(np.sum((Z - Zc) ** 2, axis=1)))


def equivariance_error(A, B, C, lmax_in, lmax_sh, lmax_out, rng, n_rot=8, batch=64):
    """Relative SO(3)-equivariance error of the CP map: for Haar-random rotations
    R with block Wigner-D matrices D_in, D_sh, D_out,
    ||CP(D_in x, D_sh y) - D_out CP(x, y)|| / ||CP(x, y)|| over N(0,1) pairs
    (zero for any exactly equivariant map, such as the exact CG product)."""
    d1, d2, _ = dims(lmax_in, lmax_sh, lmax_out)
    num = den = 0.0
    for _ in range(n_rot):
        R = random_rotation(rng)
        D1, D2, D3 = (block_rotation(l, R) for l in (lmax_in, lmax_sh, lmax_out))
        x = rng.standard_normal((batch, d1, 1))
        y = rng.standard_normal((batch, d2, 1))
        z = cp_forward(A, B, C, x, y)
        zr = cp_forward(A, B, C, np.einsum("ab,nbu->nau", D1, x), np.einsum("ab,nbu->nau", D2, y))
        num += float(np.sum((zr - np.einsum("ab,nbu->nau", D3, z)) ** 2))
        den += float(np.sum(z ** 2))
    return float(np.sqrt(num / den))
