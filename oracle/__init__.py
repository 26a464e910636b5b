"""Float64 CPU oracle for the edge-conditioned O(3) tensor-product convolution.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The CUDA library never imports, links or calls it, and it shares no code, table or
helper with the library: both sides only share the seeded input generator, which
holds none of the method's arithmetic.

What it computes follows "Sobek: Streaming Equivariant Tensor Product
Convolutions" (arXiv 2607.18074), section 2:

* ``irreps``  -- feature fields, flattened width and the CG selection rule (eqs. 3-5),
  path weight counts (eqs. 9-10);
* ``so3``     -- real spherical harmonics of the edge direction and the real
  Clebsch-Gordan coupling tensors (eq. 5, eq. 32's ``c^pi``);
* ``radial``  -- the radial embedding ``phi(|r|)`` (the pages leave its form open);
* ``conv``    -- the materialised per-edge operator (eqs. 6-7, 11-13), its first-order
  adjoints (eqs. 18-22), second-order directional adjoints (eqs. 23-30) and the double
  backward's position gradient (through second derivatives of Y and phi), plus a
  second evaluation in the receiver-factorised streaming order (eqs. 16, 32-35) used
  only to check that both orders agree.

Everything is evaluated in float64; inputs given as float32 are promoted.

Pins (tests/test_oracle_*.py): CG closed forms for small l, CG orthogonality and
equivariance, spherical-harmonic identities (addition theorem, parity, explicit
Cartesian forms, quadrature orthonormality), radial-basis orthonormality and cutoff
smoothness, operator equivariance under random O(3) elements, translation and
permutation invariance, the scalar-input special case, agreement of the two
evaluation orders, central finite differences for every gradient and for the
double backward, and for the second derivatives of Y and phi a closed form, Euler's
relation, the radial Hessian form and Hessian symmetry.  Parity unpinned: the absolute orientation of the real SH basis and
the sign of each CG tensor are conventions the pages do not fix; every observable
invariant checked above is independent of them.
"""

from . import irreps, so3, radial, conv, graph  # noqa: F401
