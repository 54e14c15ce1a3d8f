"""Seeded synthetic workloads for the CGTP convolution.

This module only draws random inputs (positions, features, network weights,
output gradients) with the shapes and structure of the five standard
workloads; it contains none of the convolution's arithmetic and is shared by
the tests, the benchmark and the smoke check.  Every draw uses
``numpy.random.default_rng(seed)`` in a fixed order: positions, features,
weights, output gradient.

Workloads (positions in Angstrom, all arrays fp32):

* ``tiny``      32 atoms uniform in a 5 A cube, no periodicity, cutoff 3 A,
                8 channels of l = 0, 1; harmonics l <= 1; outputs l <= 1;
                radial network 8 Gaussians -> 64 SiLU -> paths x 8.
* ``tp_batch``  1000 independent (x, y) pairs, 128 channels of l = 0..2 each;
                outputs l <= 2; per-path, per-channel weights ~ N(0, 1/P).
* ``bulk``      1000 atoms uniform in a periodic cube at 0.1 atoms/A^3
                (side 21.544 A), cutoff 5 A; 64 channels of l = 0..2;
                harmonics l <= 2; outputs l <= 2.
* ``bulk_large`` 20000 atoms at the same density (side 58.480 A), cutoff 5 A;
                128 channels of l = 0..3; harmonics l <= 3; outputs l <= 3;
                energy = sum of the l = 0 outputs.
* ``molecules`` 256 graphs of 30 atoms, each uniform in an 8 A cube with
                sequential rejection of candidates closer than 0.9 A to an
                accepted atom of the same graph, cutoff 5 A, one CSR over the
                whole batch; 128 channels of l = 0..2; harmonics l <= 4;
                outputs l <= 2; energy = sum of the l = 0 outputs.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

N_BASIS = 8
HIDDEN = 64


@dataclass
class ConvWorkload:
    name: str
    seed: int
    lmax_in: int
    lmax_sh: int
    lmax_out: int
    mult: int
    n_paths: int
    rc: float
    box: Optional[float]
    pos: np.ndarray                 # [N][3] fp32
    graph_id: Optional[np.ndarray]  # [N] int32 or None
    x: np.ndarray                   # [N][(lmax_in+1)^2][mult] fp32
    W1: np.ndarray                  # [8][64] fp32
    W2: np.ndarray                  # [64][n_paths*mult] fp32
    grad_out: np.ndarray            # [N][(lmax_out+1)^2][mult] fp32
    energy_grad: bool               # grad_out is the gradient of sum of l=0 outputs
    graph_size: Optional[int] = None
    meta: dict = field(default_factory=dict)

    @property
    def n_nodes(self):
        return self.pos.shape[0]


@dataclass
class TPWorkload:
    name: str
    seed: int
    lmax_in: int
    lmax_sh: int
    lmax_out: int
    mult: int
    n_paths: int
    x: np.ndarray       # [B][(lmax_in+1)^2][mult]
    y: np.ndarray       # [B][(lmax_sh+1)^2][mult]
    w: np.ndarray       # [P][mult]
    grad_z: np.ndarray  # [B][(lmax_out+1)^2][mult]


def count_paths(lmax_in, lmax_sh, lmax_out):
    """Number of (l1, l2, l3) triples allowed by the triangle rule (shape only)."""
    return sum(1 for l1 in range(lmax_in + 1) for l2 in range(lmax_sh + 1)
               for l3 in range(abs(l1 - l2), min(l1 + l2, lmax_out) + 1))


def _features(rng, n, lmax, mult):
    return rng.standard_normal((n, (lmax + 1) ** 2, mult)).astype(np.float32)


def _mlp(rng, n_paths, mult):
    W1 = (rng.standard_normal((N_BASIS, HIDDEN)) / np.sqrt(N_BASIS)).astype(np.float32)
    W2 = (rng.standard_normal((HIDDEN, n_paths * mult)) / np.sqrt(HIDDEN)).astype(np.float32)
    return W1, W2


def _energy_grad(n, lmax_out, mult):
    g = np.zeros((n, (lmax_out + 1) ** 2, mult), dtype=np.float32)
    g[:, 0, :] = 1.0
    return g


def _uniform_box(rng, n, side):
    return (rng.random((n, 3)) * side).astype(np.float32)


def _rejection_graph(rng, n, side, rmin):
    pts = np.zeros((0, 3), dtype=np.float32)
    while pts.shape[0] < n:
        cand = (rng.random(3) * side).astype(np.float32)
        if pts.shape[0]:
            d = pts.astype(np.float64) - cand.astype(np.float64)
            if np.min(np.sum(d * d, axis=1)) < rmin * rmin:
                continue
        pts = np.vstack([pts, cand[None, :]])
    return pts


def tiny(seed=0):
    rng = np.random.default_rng(seed)
    L = (1, 1, 1)
    P = count_paths(*L)
    pos = _uniform_box(rng, 32, 5.0)
    x = _features(rng, 32, L[0], 8)
    W1, W2 = _mlp(rng, P, 8)
    g = rng.standard_normal((32, (L[2] + 1) ** 2, 8)).astype(np.float32)
    return ConvWorkload("tiny", seed, *L, 8, P, 3.0, None, pos, None, x, W1, W2, g, False)


def tp_batch(seed=1, batch=1000, mult=128):
    rng = np.random.default_rng(seed)
    L = (2, 2, 2)
    P = count_paths(*L)
    x = _features(rng, batch, L[0], mult)
    y = _features(rng, batch, L[1], mult)
    w = (rng.standard_normal((P, mult)) / np.sqrt(P)).astype(np.float32)
    g = rng.standard_normal((batch, (L[2] + 1) ** 2, mult)).astype(np.float32)
    return TPWorkload("tp_batch", seed, *L, mult, P, x, y, w, g)


def bulk(seed=2, n=1000, mult=64, density=0.1):
    rng = np.random.default_rng(seed)
    L = (2, 2, 2)
    P = count_paths(*L)
    side = float(np.float32((n / density) ** (1.0 / 3.0)))
    pos = _uniform_box(rng, n, side)
    x = _features(rng, n, L[0], mult)
    W1, W2 = _mlp(rng, P, mult)
    g = rng.standard_normal((n, (L[2] + 1) ** 2, mult)).astype(np.float32)
    return ConvWorkload("bulk", seed, *L, mult, P, 5.0, side, pos, None, x, W1, W2, g, False)


def bulk_large(seed=3, n=20000, mult=128, density=0.1):
    rng = np.random.default_rng(seed)
    L = (3, 3, 3)
    P = count_paths(*L)
    side = float(np.float32((n / density) ** (1.0 / 3.0)))
    pos = _uniform_box(rng, n, side)
    x = _features(rng, n, L[0], mult)
    W1, W2 = _mlp(rng, P, mult)
    g = _energy_grad(n, L[2], mult)
    return ConvWorkload("bulk_large", seed, *L, mult, P, 5.0, side, pos, None, x, W1, W2, g, True)


def molecules(seed=4, n_graphs=256, atoms=30, mult=128, side=8.0, rmin=0.9):
    rng = np.random.default_rng(seed)
    L = (2, 4, 2)
    P = count_paths(*L)
    pos = np.concatenate([_rejection_graph(rng, atoms, side, rmin) for _ in range(n_graphs)])
    gid = np.repeat(np.arange(n_graphs, dtype=np.int32), atoms)
    n = n_graphs * atoms
    x = _features(rng, n, L[0], mult)
    W1, W2 = _mlp(rng, P, mult)
    g = _energy_grad(n, L[2], mult)
    return ConvWorkload("molecules", seed, *L, mult, P, 5.0, None, pos, gid, x, W1, W2, g, True,
                        graph_size=atoms)


def random_graph_features(rng, n, lmax, mult):
    """Standard-normal irreps features [n][(lmax+1)^2][mult] (for unit tests)."""
    return _features(rng, n, lmax, mult)


WORKLOADS = {"tiny": tiny, "tp_batch": tp_batch, "bulk": bulk,
             "bulk_large": bulk_large, "molecules": molecules}
