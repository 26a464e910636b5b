"""Pins for the oracle's embedded-input interface (conv.forward_embedded and
conv.backward_embedded: phi_e and Y_e given per edge, adjoints phi_bar and Y_bar returned
per edge).

* with Y_e and phi_e computed from positions, they reproduce the position-based oracle;
* phi_bar and Y_bar, pushed through dY/dr and dphi/dr, give the position gradient;
* phi_bar and Y_bar against central finite differences of <forward_embedded, m_bar>;
* the forward is linear in phi.
"""

import numpy as np
import pytest

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, radial, so3

BESSEL = radial.RadialSpec(radial.BESSEL, 6, 2.5)
GAUSS = radial.RadialSpec(radial.GAUSSIAN, 5, 3.0, 0.0, 3.0)
CASES = {
    "uvw": ("3x0e+2x1o+2x2e", 3, "2x0e+3x1o+2x2e+1x3o", "uvw", BESSEL),
    "uvu": ("3x0e+3x1o+3x2e", 2, "3x0e+3x1o+3x2e", "uvu", GAUSS),
}


def _problem(case, n=10, k=4, seed=3):
    ii, lmax, io, mode, rs = CASES[case]
    plan = conv.make_plan(ii, lmax, io, mode, rs)
    rng = np.random.default_rng(seed)
    pos = rng.uniform(0, 2.5, size=(n, 3))
    row_ptr, src = workloads.knn_csr(pos, np.full(n, k))
    x = rng.normal(size=(n, plan.dim_in))
    A = rng.normal(size=(rs.num_basis, plan.n_w)) / 3
    mbar = rng.normal(size=(n, plan.dim_out))
    dst = conv.receivers_of(row_ptr)
    r = pos[src] - pos[dst]
    return plan, x, pos, row_ptr, src, A, mbar, r, rs


@pytest.mark.parametrize("case", sorted(CASES))
def test_embedded_matches_position_oracle(case):
    plan, x, pos, row_ptr, src, A, mbar, r, rs = _problem(case)
    N = pos.shape[0]
    Y = so3.sh(plan.lmax, r)
    phi, _ = radial.basis_of_vectors(rs, r)
    out = conv.forward_embedded(plan, x, Y, phi, row_ptr, N, src, A)
    assert np.allclose(out, conv.forward(plan, x, pos, row_ptr, src, A), rtol=0, atol=1e-12)
    gx, gA, gphi, gY = conv.backward_embedded(plan, x, Y, phi, row_ptr, N, src, A, mbar)
    rx, rpos, rA = conv.backward(plan, x, pos, row_ptr, src, A, mbar)
    assert np.allclose(gx, rx, atol=1e-12) and np.allclose(gA, rA, atol=1e-12)
    # chain rule through the geometry reproduces the position gradient
    _, dY = so3.sh_with_grad(plan.lmax, r)
    dphi = _radial_grad(rs, r)
    g = np.einsum("esk,es->ek", dY, gY) + np.einsum("eqk,eq->ek", dphi, gphi)
    dst = conv.receivers_of(row_ptr)
    gpos = np.zeros((N, 3))
    np.add.at(gpos, src, g)
    np.add.at(gpos, dst, -g)
    assert np.allclose(gpos, rpos, atol=1e-10)


def _radial_grad(rs, r, h=1e-6):
    """d phi / d r by central differences of the oracle's radial basis (the oracle's own
    analytic derivative is pinned elsewhere; this only links the two interfaces)."""
    out = np.zeros(r.shape[:1] + (rs.num_basis, 3))
    for k in range(3):
        d = np.zeros(3)
        d[k] = h
        p, _ = radial.basis_of_vectors(rs, r + d)
        m, _ = radial.basis_of_vectors(rs, r - d)
        out[:, :, k] = (p - m) / (2 * h)
    return out


@pytest.mark.parametrize("case", sorted(CASES))
def test_embedded_adjoints_finite_differences(case):
    plan, x, pos, row_ptr, src, A, mbar, r, rs = _problem(case, n=7, k=3, seed=5)
    N = pos.shape[0]
    rng = np.random.default_rng(11)
    Y = rng.normal(size=(src.size, plan.n_sh))           # any per-edge inputs, not only harmonics
    phi = rng.normal(size=(src.size, rs.num_basis))
    _, _, gphi, gY = conv.backward_embedded(plan, x, Y, phi, row_ptr, N, src, A, mbar)

    def L(Yv, phiv):
        return float(np.sum(conv.forward_embedded(plan, x, Yv, phiv, row_ptr, N, src, A) * mbar))

    h = 1e-6
    for e, q in [(0, 0), (3, 2), (src.size - 1, rs.num_basis - 1)]:
        d = np.zeros_like(phi)
        d[e, q] = h
        fd = (L(Y, phi + d) - L(Y, phi - d)) / (2 * h)
        assert abs(fd - gphi[e, q]) <= 1e-6 * max(1.0, abs(fd))
    for e, s in [(1, 0), (4, 2), (src.size - 2, plan.n_sh - 1)]:
        d = np.zeros_like(Y)
        d[e, s] = h
        fd = (L(Y + d, phi) - L(Y - d, phi)) / (2 * h)
        assert abs(fd - gY[e, s]) <= 1e-6 * max(1.0, abs(fd))


def test_embedded_forward_linear_in_phi():
    plan, x, pos, row_ptr, src, A, mbar, r, rs = _problem("uvw")
    rng = np.random.default_rng(2)
    Y = rng.normal(size=(src.size, plan.n_sh))
    p1 = rng.normal(size=(src.size, rs.num_basis))
    p2 = rng.normal(size=(src.size, rs.num_basis))
    N = pos.shape[0]
    f = lambda p: conv.forward_embedded(plan, x, Y, p, row_ptr, N, src, A)  # noqa: E731
    assert np.allclose(f(2.0 * p1 - 3.0 * p2), 2.0 * f(p1) - 3.0 * f(p2), atol=1e-11)
