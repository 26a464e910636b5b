"""Pins for the oracle's radial embedding (oracle/radial.py)."""

import numpy as np

from oracle import radial
from oracle.dual import Dual


def _d(vals):
    v = np.asarray(vals, dtype=np.float64)
    g = np.zeros((v.shape[0], 3))
    g[:, 0] = 1.0          # d/dd carried in slot 0
    return Dual(v, g)


def test_envelope_boundary_values():
    t = _d([0.0, 1.0 - 1e-12, 1.0, 1.5])
    u = radial.envelope(t, 6)
    assert np.isclose(u.v[0], 1.0) and abs(u.g[0, 0]) < 1e-15
    assert abs(u.v[1]) < 1e-20 and abs(u.v[2]) == 0.0 and u.v[3] == 0.0
    # u(1) = u'(1) = u''(1) = 0 with u'''(1) != 0  <=>  u(1 - h) ~ c h^3 as h -> 0
    h = 1e-3
    a = radial.envelope(_d([1.0 - h]), 6).v[0]
    b = radial.envelope(_d([1.0 - 2 * h]), 6).v[0]
    assert abs(a) > 0 and abs(a / b - 0.125) < 2e-3


def test_envelope_derivative_matches_fd():
    t = np.linspace(0.05, 0.95, 19)
    u = radial.envelope(_d(t), 6)
    h = 1e-6
    fd = (radial.envelope(_d(t + h), 6).v - radial.envelope(_d(t - h), 6).v) / (2 * h)
    assert np.allclose(u.g[:, 0], fd, atol=1e-8)


def test_bessel_bare_basis_orthonormal():
    """sqrt(2/rc) sin(b pi d/rc)/d is orthonormal on [0, rc] with weight d^2."""
    spec = radial.RadialSpec(radial.BESSEL, 8, 5.0)
    x, w = np.polynomial.legendre.leggauss(200)
    d = 0.5 * spec.r_cut * (x + 1)
    w = 0.5 * spec.r_cut * w
    phi = np.stack([q.v for q in radial.basis_dual(spec, _d(d), with_envelope=False)], 1)
    G = (phi * (w * d * d)[:, None]).T @ phi
    assert np.allclose(G, np.eye(8), atol=1e-12)


def test_bessel_is_bare_times_envelope_and_zero_beyond_cutoff():
    spec = radial.RadialSpec(radial.BESSEL, 8, 3.0)
    d = np.array([0.3, 1.0, 2.9, 3.0, 4.0])
    full = np.stack([q.v for q in radial.basis_dual(spec, _d(d))], 1)
    bare = np.stack([q.v for q in radial.basis_dual(spec, _d(d), with_envelope=False)], 1)
    u = radial.envelope(_d(d / spec.r_cut), 6).v
    assert np.allclose(full, bare * u[:, None], atol=1e-15)
    assert np.all(full[3:] == 0.0)


def test_bessel_small_d_limit():
    spec = radial.RadialSpec(radial.BESSEL, 4, 2.0)
    a = np.stack([q.v for q in radial.basis_dual(spec, _d([0.0]))], 1)
    b = np.stack([q.v for q in radial.basis_dual(spec, _d([1e-7]))], 1)
    assert np.allclose(a, b, rtol=1e-10)


def test_gaussian_peaks_and_width():
    spec = radial.RadialSpec(radial.GAUSSIAN, 16, 6.0, 0.0, 6.0)
    sigma = 6.0 / 15
    mu = np.linspace(0, 6, 16)[:-1]
    phi = np.stack([q.v for q in radial.basis_dual(spec, _d(mu), with_envelope=False)], 1)
    assert np.allclose(np.diag(phi[:, :15]), 1.0)
    phi2 = np.stack([q.v for q in radial.basis_dual(spec, _d(mu + sigma), with_envelope=False)], 1)
    assert np.allclose(np.diag(phi2[:, :15]), np.exp(-0.5))


def test_radial_gradient_matches_fd(rng):
    for spec in (radial.RadialSpec(radial.BESSEL, 8, 5.0),
                 radial.RadialSpec(radial.GAUSSIAN, 16, 6.0, 0.0, 6.0)):
        r = rng.normal(size=(40, 3)) * 1.5
        phi, dphi = radial.basis_of_vectors(spec, r)
        h = 1e-6
        for k in range(3):
            e = np.zeros(3)
            e[k] = h
            fd = (radial.basis_of_vectors(spec, r + e)[0] - radial.basis_of_vectors(spec, r - e)[0]) / (2 * h)
            assert np.allclose(dphi[:, :, k], fd, atol=1e-7)
