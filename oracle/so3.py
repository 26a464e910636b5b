"""Real spherical harmonics and real Clebsch-Gordan coupling tensors (oracle side).

The pages build Y_ij from spherical harmonics of the edge direction (Sobek, section 2,
after eq. 8) and let c^pi carry both a path normalisation and the sparse Clebsch-Gordan
coefficients (section 4, eq. 32), but fix neither the basis nor the normalisation.  The
readings taken here:

* Real SH, z polar axis, no Condon-Shortley phase, component normalisation
  (sum_m Y_lm^2 = 2l+1).  For m >= 0
      Y_{l,m}  = N_lm * P_l^{(m)}(z) * Re((x + i y)^m)
      Y_{l,-m} = N_lm * P_l^{(m)}(z) * Im((x + i y)^m)
  with P_l^{(m)} the m-th derivative of the Legendre polynomial P_l,
  N_l0 = sqrt(2l+1) and N_lm = sqrt(2 (2l+1) (l-m)! / (l+m)!).  On the unit sphere
  this is the textbook sqrt(4 pi) * real SH: P_l^m(cos t) cos(m p) with
  sin^m(t) cos(m p) = Re((x+iy)^m).  Component order m = -l..l, so
  Y_1 = sqrt(3) (y, z, x).
* c^pi = sqrt(2 l_out + 1) * w, where w is the real invariant tensor of
  l_in (x) l_sh (x) l_out in this basis with unit Frobenius norm, signed so that its
  first entry (row-major over m_in, m_sh, m_out) with |w| > 1e-9 is positive.  No
  extra path weight: fan-in lives in the weight initialisation.
* w is obtained from the complex Clebsch-Gordan coefficients (Racah's closed form,
  Condon-Shortley convention) by the unitary change of basis between complex and
  real harmonics; the result is real up to one global phase, which is removed.
"""

from fractions import Fraction
from functools import lru_cache
from math import factorial, sqrt

import numpy as np
from numpy.polynomial import legendre as _leg
from numpy.polynomial import polynomial as _poly

from .dual import Dual


# ---------------------------------------------------------------------------
# spherical harmonics
# ---------------------------------------------------------------------------

@lru_cache(maxsize=None)
def _legendre_deriv_coeffs(l, m):
    """Power-series coefficients (ascending) of d^m/dz^m P_l(z)."""
    c = np.zeros(l + 1)
    c[l] = 1.0
    p = _leg.leg2poly(c)
    for _ in range(m):
        p = _poly.polyder(p)
    return tuple(float(v) for v in np.atleast_1d(p))


def _norm(l, m):
    if m == 0:
        return sqrt(2 * l + 1)
    return sqrt(2.0 * (2 * l + 1) * factorial(l - m) / factorial(l + m))


def _horner(coeffs, z):
    n = z.v.shape[0]
    acc = Dual.const(0.0, n)
    for c in reversed(coeffs):
        acc = acc * z + c
    return acc


def unit_direction(r, second=False):
    """r_hat = r / |r| as Duals (eq. 8).  A zero-length vector maps to r_hat = 0 (and
    sh_dual then sets every l > 0 harmonic of it to zero).
    With ``second`` the Duals also carry Hessians in r."""
    from .dual import edge_vector
    rx, ry, rz = edge_vector(r, second)
    d = (rx * rx + ry * ry + rz * rz).sqrt()
    n = d.v.shape[0]
    zero = d.v < 1e-12
    safe = Dual(np.where(zero, 1.0, d.v), np.where(zero[:, None], 0.0, d.g),
                None if d.h is None else np.where(zero[:, None, None], 0.0, d.h))
    z0 = Dual.const(0.0, n)
    hat = [(c / safe).where(~zero, z0) for c in (rx, ry, rz)]
    return hat, d


def sh_dual(lmax, r, second=False):
    """Real SH of the directions of r [E,3] for l = 0..lmax.

    Returns a list (length (lmax+1)^2, order l-major then m = -l..l) of Duals whose
    gradient is d Y / d r (the raw edge vector, not r_hat); with ``second`` they also
    carry d^2 Y / dr^2.
    """
    (x, y, z), d = unit_direction(r, second)
    n = x.v.shape[0]
    # a zero-length edge has no direction: every l > 0 harmonic is zero there (the only
    # choice that commutes with rotations), while Y_0 = 1 keeps its constant value
    directed = d.v >= 1e-12
    z0 = Dual.const(0.0, n)
    # powers (x + i y)^m as (re, im) Duals
    re = [Dual.const(1.0, n)]
    im = [Dual.const(0.0, n)]
    for m in range(1, lmax + 1):
        a, b = re[-1], im[-1]
        re.append(a * x - b * y)
        im.append(a * y + b * x)
    out = []
    for l in range(lmax + 1):
        row = [None] * (2 * l + 1)
        for m in range(0, l + 1):
            q = _horner(_legendre_deriv_coeffs(l, m), z) * _norm(l, m)
            if m == 0:
                row[l] = q
            else:
                row[l + m] = q * re[m]
                row[l - m] = q * im[m]
        if l > 0:
            row = [q.where(directed, z0) for q in row]
        out.extend(row)
    return out


def sh(lmax, r):
    """Values only: [E, (lmax+1)^2]."""
    return np.stack([d.v for d in sh_dual(lmax, np.atleast_2d(r))], axis=1)


def sh_with_grad(lmax, r):
    """Values [E, n_sh] and d Y / d r as [E, n_sh, 3]."""
    ds = sh_dual(lmax, np.atleast_2d(r))
    return np.stack([d.v for d in ds], axis=1), np.stack([d.g for d in ds], axis=1)


def sh_with_hessian(lmax, r):
    """Values [E, n_sh], d Y / d r [E, n_sh, 3] and d^2 Y / dr^2 [E, n_sh, 3, 3]."""
    ds = sh_dual(lmax, np.atleast_2d(r), second=True)
    n = ds[0].v.shape[0]
    hs = [d.h if d.h is not None else np.zeros((n, 3, 3)) for d in ds]
    return (np.stack([d.v for d in ds], axis=1), np.stack([d.g for d in ds], axis=1),
            np.stack(hs, axis=1))


# ---------------------------------------------------------------------------
# Clebsch-Gordan coefficients
# ---------------------------------------------------------------------------

def _f(n):
    return factorial(n)


def cg_complex(j1, m1, j2, m2, J, M):
    """<j1 m1 j2 m2 | J M>, Racah's closed form (exact rational arithmetic under a
    square root, Condon-Shortley phase convention)."""
    if M != m1 + m2 or not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    pref = Fraction((2 * J + 1) * _f(J + j1 - j2) * _f(J - j1 + j2) * _f(j1 + j2 - J),
                    _f(j1 + j2 + J + 1))
    pref *= _f(J + M) * _f(J - M) * _f(j1 - m1) * _f(j1 + m1) * _f(j2 - m2) * _f(j2 + m2)
    s = Fraction(0)
    for k in range(0, j1 + j2 + J + 2):
        den = [k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k]
        if min(den) < 0:
            continue
        d = 1
        for v in den:
            d *= _f(v)
        s += Fraction((-1) ** k, d)
    return float(s) * sqrt(float(pref))


def real_from_complex(l):
    """U with Y_real = U @ Y_complex (complex harmonics with the Condon-Shortley
    phase; real ones as in the module doc).  Rows/cols indexed m = -l..l."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    U[l, l] = 1.0
    for m in range(1, l + 1):
        s = (-1) ** m
        U[l + m, l + m] = s / sqrt(2)
        U[l + m, l - m] = 1 / sqrt(2)
        U[l - m, l + m] = -1j * s / sqrt(2)
        U[l - m, l - m] = 1j / sqrt(2)
    return U


@lru_cache(maxsize=None)
def _real_cg_cached(l1, l2, l3):
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        return None
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for a in range(-l1, l1 + 1):
        for b in range(-l2, l2 + 1):
            M = a + b
            if abs(M) <= l3:
                C[a + l1, b + l2, M + l3] = cg_complex(l1, a, l2, b, l3, M)
    U1, U2, U3 = real_from_complex(l1), real_from_complex(l2), real_from_complex(l3)
    # Real coefficient vectors transform as conj(U) D U^T; couple in the complex
    # basis and map back.
    w = np.einsum("ai,bj,ck,ijk->abc", U1, U2, np.conj(U3), C)
    if np.linalg.norm(w.imag) > np.linalg.norm(w.real):
        w = w.imag
    else:
        w = w.real
    w = np.where(np.abs(w) < 1e-14, 0.0, w)
    w = w / np.linalg.norm(w)
    flat = w.reshape(-1)
    first = flat[np.argmax(np.abs(flat) > 1e-9)]
    if first < 0:
        w = -w
    return w


def real_cg_unit(l1, l2, l3):
    """Unit-Frobenius real invariant tensor w[m_in, m_sh, m_out] (see module doc)."""
    w = _real_cg_cached(l1, l2, l3)
    if w is None:
        raise ValueError("triangle condition violated")
    return w.copy()


def path_coupling(l_in, l_sh, l_out):
    """c^pi of eq. 32: sqrt(2 l_out + 1) times the unit invariant tensor."""
    return sqrt(2 * l_out + 1) * real_cg_unit(l_in, l_sh, l_out)
