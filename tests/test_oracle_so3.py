"""Pins for the oracle's spherical harmonics and Clebsch-Gordan tensors.

Each check is a fact of the mathematics that a wrong sign, index, normalisation or
transposition in oracle/so3.py would break: closed forms of small invariant
tensors, orthogonality, equivariance under rotations, the addition theorem, parity,
explicit Cartesian forms of low-order harmonics, and quadrature orthonormality.
"""

import itertools
from math import sqrt

import numpy as np
import pytest
from scipy.spatial.transform import Rotation

from oracle import so3


def _wigner_d(l, R, rng):
    """Fit D_l(R) from Y_l(R r) = D Y_l(r) on random directions (least squares)."""
    pts = rng.normal(size=(64, 3))
    s = slice(l * l, (l + 1) ** 2)
    Y = so3.sh(l, pts)[:, s]
    YR = so3.sh(l, pts @ R.T)[:, s]
    X, res, *_ = np.linalg.lstsq(Y, YR, rcond=None)
    return X.T


# ---------------------------------------------------------------- harmonics

def test_sh_addition_theorem(rng):
    r = rng.normal(size=(500, 3))
    Y = so3.sh(4, r)
    for l in range(5):
        s = (Y[:, l * l:(l + 1) ** 2] ** 2).sum(1)
        assert np.allclose(s, 2 * l + 1, atol=1e-12)


def test_sh_scale_invariant_and_parity(rng):
    r = rng.normal(size=(200, 3))
    Y = so3.sh(4, r)
    assert np.allclose(so3.sh(4, 3.7 * r), Y, atol=1e-13)
    Yn = so3.sh(4, -r)
    for l in range(5):
        s = slice(l * l, (l + 1) ** 2)
        assert np.allclose(Yn[:, s], (-1) ** l * Y[:, s], atol=1e-13)


def test_sh_pole_value():
    Y = so3.sh(4, np.array([[0.0, 0.0, 2.0]]))[0]
    for l in range(5):
        e = np.zeros(2 * l + 1)
        e[l] = sqrt(2 * l + 1)
        assert np.allclose(Y[l * l:(l + 1) ** 2], e, atol=1e-14)


def test_sh_cartesian_forms(rng):
    """Textbook Cartesian forms of the component-normalised real harmonics, l <= 2."""
    r = rng.normal(size=(100, 3))
    x, y, z = (r / np.linalg.norm(r, axis=1, keepdims=True)).T
    Y = so3.sh(2, r)
    assert np.allclose(Y[:, 0], 1.0)
    assert np.allclose(Y[:, 1:4], sqrt(3) * np.stack([y, z, x], 1), atol=1e-13)
    s15 = sqrt(15)
    Y2 = np.stack([s15 * x * y, s15 * y * z, sqrt(5) / 2 * (3 * z * z - 1), s15 * x * z,
                   s15 / 2 * (x * x - y * y)], 1)
    assert np.allclose(Y[:, 4:9], Y2, atol=1e-13)


def test_sh_orthonormal_quadrature():
    """(1/4pi) int Y_a Y_b dOmega = delta_ab, exact with Gauss-Legendre x uniform phi."""
    L = 4
    ct, wt = np.polynomial.legendre.leggauss(L + 2)
    nphi = 2 * L + 3
    ph = 2 * np.pi * np.arange(nphi) / nphi
    CT, PH = np.meshgrid(ct, ph, indexing="ij")
    ST = np.sqrt(1 - CT ** 2)
    pts = np.stack([ST * np.cos(PH), ST * np.sin(PH), CT], -1).reshape(-1, 3)
    wq = (wt[:, None] * np.full(nphi, 2 * np.pi / nphi)[None, :]).reshape(-1)
    Y = so3.sh(L, pts)
    G = (Y * wq[:, None]).T @ Y / (4 * np.pi)
    assert np.allclose(G, np.eye(Y.shape[1]), atol=1e-12)


def test_sh_gradient_matches_finite_differences(rng):
    r = rng.normal(size=(50, 3))
    _, dY = so3.sh_with_grad(3, r)
    h = 1e-6
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        fd = (so3.sh(3, r + e) - so3.sh(3, r - e)) / (2 * h)
        assert np.allclose(dY[:, :, k], fd, atol=1e-7)


def test_sh_rotation_is_orthogonal_homomorphism(rng):
    R1 = Rotation.random(random_state=3).as_matrix()
    R2 = Rotation.random(random_state=4).as_matrix()
    for l in range(5):
        D1, D2 = _wigner_d(l, R1, rng), _wigner_d(l, R2, rng)
        D12 = _wigner_d(l, R1 @ R2, rng)
        assert np.allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
        assert np.allclose(D12, D1 @ D2, atol=1e-12)


def test_zero_vector_direction():
    # a direction-less edge: only the invariant Y_0 survives (any nonzero l > 0 value
    # would single out an axis and break rotation equivariance), with zero derivatives
    Y, dY = so3.sh_with_grad(3, np.zeros((1, 3)))
    assert np.array_equal(Y[0], np.eye(16)[0])
    assert np.array_equal(dY, np.zeros_like(dY))
    Y2, dY2, H2 = so3.sh_with_hessian(3, np.zeros((2, 3)))
    assert np.array_equal(Y2, np.tile(np.eye(16)[0], (2, 1)))
    assert not np.any(dY2) and not np.any(H2)
    # the mask acts on exactly the zero vector: a tiny but nonzero edge keeps its direction
    r = np.array([[0.0, 0.0, 1e-6]])
    assert np.allclose(so3.sh(3, r), so3.sh(3, np.array([[0.0, 0.0, 1.0]])), atol=1e-12)


# ---------------------------------------------------------------- CG

TRIPLES = [t for t in itertools.product(range(4), repeat=3)
           if abs(t[0] - t[1]) <= t[2] <= t[0] + t[1]]


def test_cg_closed_forms():
    for l in range(4):
        d = 2 * l + 1
        assert np.allclose(so3.real_cg_unit(0, l, l)[0], np.eye(d) / sqrt(d), atol=1e-14)
        assert np.allclose(so3.real_cg_unit(l, 0, l)[:, 0, :], np.eye(d) / sqrt(d), atol=1e-14)
        assert np.allclose(so3.real_cg_unit(l, l, 0)[:, :, 0], np.eye(d) / sqrt(d), atol=1e-14)
    eps = np.zeros((3, 3, 3))
    for a, b, c in itertools.permutations(range(3)):
        eps[a, b, c] = np.linalg.det(np.eye(3)[[a, b, c]])
    # (y, z, x) is a cyclic relabelling of (x, y, z), so epsilon is unchanged
    assert np.allclose(so3.real_cg_unit(1, 1, 1), eps / sqrt(6), atol=1e-14)


def test_cg_112_symmetric_traceless():
    """1 x 1 -> 2 couples two vectors into the symmetric traceless part, expressed in
    the l=2 harmonics' quadratic forms Y_2m(r) = r^T Q_m r (|r| = 1)."""
    s15 = sqrt(15)
    # Cartesian axes in the l=1 component order (y, z, x)
    ax = [1, 2, 0]
    Q = np.zeros((5, 3, 3))
    Q[0][0, 1] = Q[0][1, 0] = s15 / 2                  # sqrt15 x y
    Q[1][1, 2] = Q[1][2, 1] = s15 / 2                  # sqrt15 y z
    Q[2] = sqrt(5) / 2 * np.diag([-1.0, -1.0, 2.0])   # sqrt5/2 (3z^2 - 1) on |r|=1
    Q[3][0, 2] = Q[3][2, 0] = s15 / 2                  # sqrt15 x z
    Q[4] = s15 / 2 * np.diag([1.0, -1.0, 0.0])         # sqrt15/2 (x^2 - y^2)
    w = np.einsum("mab->abm", Q[:, ax][:, :, ax])
    w /= np.linalg.norm(w)
    got = so3.real_cg_unit(1, 1, 2)
    assert np.allclose(got, w, atol=1e-14) or np.allclose(got, -w, atol=1e-14)


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_orthogonality(t):
    l1, l2, l3 = t
    w = so3.real_cg_unit(l1, l2, l3)
    G = np.einsum("abk,abn->kn", w, w)
    assert np.allclose(G, np.eye(2 * l3 + 1) / (2 * l3 + 1), atol=1e-13)


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_equivariant(t, rng):
    l1, l2, l3 = t
    w = so3.real_cg_unit(l1, l2, l3)
    R = Rotation.random(random_state=sum(t) + 7).as_matrix()
    D1, D2, D3 = (_wigner_d(l, R, rng) for l in t)
    lhs = np.einsum("abc,ai,bj->ijc", w, D1, D2)
    rhs = np.einsum("ijk,ck->ijc", w, D3)
    assert np.allclose(lhs, rhs, atol=1e-12)


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_permutation_symmetry(t):
    l1, l2, l3 = t
    a = so3.real_cg_unit(l1, l2, l3)
    b = np.transpose(so3.real_cg_unit(l2, l1, l3), (1, 0, 2))
    sign = (-1) ** (l1 + l2 + l3)
    assert np.allclose(a, sign * b, atol=1e-13) or np.allclose(a, -sign * b, atol=1e-13)


def test_cg_sign_rule_and_coupling_norm():
    for t in TRIPLES:
        w = so3.real_cg_unit(*t).reshape(-1)
        first = w[np.argmax(np.abs(w) > 1e-9)]
        assert first > 0
        c = so3.path_coupling(*t)
        assert np.isclose(np.linalg.norm(c), sqrt(2 * t[2] + 1))


def test_cg_complex_known_values():
    """Tabulated complex CG values (Condon-Shortley)."""
    assert np.isclose(so3.cg_complex(1, 1, 1, -1, 0, 0), 1 / sqrt(3))
    assert np.isclose(so3.cg_complex(1, 0, 1, 0, 0, 0), -1 / sqrt(3))
    assert np.isclose(so3.cg_complex(1, 1, 1, 0, 2, 1), 1 / sqrt(2))
    assert np.isclose(so3.cg_complex(1, 0, 1, 0, 2, 0), sqrt(2 / 3))
    assert np.isclose(so3.cg_complex(1, 1, 1, -1, 1, 0), 1 / sqrt(2))
    assert np.isclose(so3.cg_complex(2, 2, 1, -1, 2, 1), sqrt(1 / 3))
