"""fp64 CPU oracle for the Clebsch-Gordan tensor-product (CGTP) convolution.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code, table or constant with the CUDA
library; it takes plain NumPy arrays and returns plain NumPy arrays.

What it computes, and the passage each part follows:

* ``cg``      -- complex Clebsch-Gordan coefficients by the Racah closed form,
                 the complex->real change of basis, and the real-basis
                 coefficients of every path (l1, l2, l3) allowed by the
                 selection rules |l1-l2| <= l3 <= l1+l2, m3 = m1+m2
                 ("Tensor Decomposition Networks ...", reply to reviewer S6y1,
                 low-rank discussion).
* ``sh``      -- real spherical harmonics (component normalisation) from the
                 explicit associated-Legendre sum, and their Cartesian
                 Jacobian by complex-step differentiation.
* ``wigner``  -- real Wigner-D matrices (closed-form small-d and a least-squares
                 fit to the harmonics); used only by equivariance pins.
* ``graph``   -- brute-force all-pairs neighbour list with the fp64 predicate,
                 minimum-image shift and CSR/CSC ordering.
* ``conv``    -- the CGTP convolution written as the literal sum over edges,
                 paths and nonzero (m1, m2, m3) ("LunaTP: Enabling Efficient and
                 Scalable Tensor Product for Equivariant MLIPs", abstract), its
                 analytic adjoints and the per-atom forces.
* ``radial``  -- the Gaussian-RBF -> SiLU -> linear radial network that makes
                 the per-edge, per-path, per-channel weights, and its
                 derivative with respect to the edge length.
* ``tp``      -- the edge-free channelwise tensor product of batched pairs
                 ("Tensor Decomposition Networks ...", reply to reviewer S6y1,
                 timing at batch 1000 and multiplicity 128) and its adjoints.
* ``cp``      -- the CP-decomposed surrogate z = A (B^T x (*) C^T y) of that
                 product, its input and factor gradients, and the fit of the
                 factors by least squares on standard-normal batches (same
                 pages, reply to reviewer S6y1 on the backward and on Figure 3).

Every function is pinned by tests under ``tests/`` against closed forms,
library routines (sympy's Clebsch-Gordan values, scipy's spherical
harmonics), invariants (orthogonality, equivariance, adjoint identities) and
finite differences.
"""
