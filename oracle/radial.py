"""Radial edge embedding phi(|r|) in R^K (oracle side).

The pages call phi_ij "a radial or more general invariant edge embedding" (Sobek,
section 2, after eq. 8) and fix neither its form nor its cutoff.  Readings taken:

* Bessel basis (K functions, b = 1..K):
      phi_b(d) = sqrt(2 / r_c) * sin(b pi d / r_c) / d * u(d / r_c)
  Without u these are orthonormal on [0, r_c] with weight d^2.
* Gaussian basis: centres mu_b = linspace(r_min, r_max, K), width
  sigma = (r_max - r_min) / (K - 1):
      phi_b(d) = exp(-(d - mu_b)^2 / (2 sigma^2)) * u(d / r_c)
* Polynomial envelope with p = 6 (for 0 <= t < 1, else 0):
      u(t) = 1 - (p+1)(p+2)/2 t^p + p(p+2) t^(p+1) - p(p+1)/2 t^(p+2)
  so that u(0) = 1 and u, u', u'' vanish at t = 1.
* An edge with d >= r_c is kept and contributes exactly zero; a zero-length edge
  takes the d -> 0 limit of phi (sin(b pi d / r_c) / d -> b pi / r_c).

All functions take Duals so that d phi / d r (and, for the double backward's position
gradient, d^2 phi / dr^2) comes out exactly (see dual.py).
"""

from dataclasses import dataclass
from math import pi, sqrt

import numpy as np

from .dual import Dual

BESSEL = "bessel"
GAUSSIAN = "gaussian"


@dataclass(frozen=True)
class RadialSpec:
    kind: str
    num_basis: int
    r_cut: float
    r_min: float = 0.0
    r_max: float = 0.0
    poly_p: int = 6


def envelope(t, p=6):
    """u(t) of the module doc, on Duals (t = d / r_c)."""
    n = t.v.shape[0]
    a = (p + 1) * (p + 2) / 2.0
    b = float(p * (p + 2))
    c = p * (p + 1) / 2.0
    u = 1.0 - a * t ** p + b * t ** (p + 1) - c * t ** (p + 2)
    inside = t.v < 1.0
    return u.where(inside, Dual.const(0.0, n))


def basis_dual(spec, d, with_envelope=True):
    """phi_b(d) for b = 0..K-1 as a list of Duals; d is a Dual (edge length).

    with_envelope=False drops u (only used to check the bare basis)."""
    n = d.v.shape[0]
    u = envelope(d / spec.r_cut, spec.poly_p) if with_envelope else Dual.const(1.0, n)
    out = []
    if spec.kind == BESSEL:
        tiny = d.v < 1e-12
        safe_d = Dual(np.where(tiny, 1.0, d.v), np.where(tiny[:, None], 0.0, d.g),
                      None if d.h is None else np.where(tiny[:, None, None], 0.0, d.h))
        for b in range(1, spec.num_basis + 1):
            k = b * pi / spec.r_cut
            f = (safe_d * k).sin() / safe_d * sqrt(2.0 / spec.r_cut)
            lim = Dual.const(sqrt(2.0 / spec.r_cut) * k, n)
            out.append(f.where(~tiny, lim) * u)
    elif spec.kind == GAUSSIAN:
        K = spec.num_basis
        sigma = (spec.r_max - spec.r_min) / (K - 1)
        for b in range(K):
            mu = spec.r_min + (spec.r_max - spec.r_min) * b / (K - 1)
            t = (d - mu) / sigma
            out.append((t * t * -0.5).exp() * u)
    else:
        raise ValueError(f"unknown radial kind {spec.kind!r}")
    return out


def basis_of_vectors(spec, r):
    """phi [E, K] and d phi / d r [E, K, 3] for edge vectors r [E, 3]."""
    from .so3 import unit_direction
    _, d = unit_direction(np.atleast_2d(r))
    ds = basis_dual(spec, d)
    return np.stack([q.v for q in ds], axis=1), np.stack([q.g for q in ds], axis=1)


def basis_with_hessian(spec, r):
    """phi [E, K], d phi / d r [E, K, 3] and d^2 phi / dr^2 [E, K, 3, 3]."""
    from .so3 import unit_direction
    _, d = unit_direction(np.atleast_2d(r), second=True)
    ds = basis_dual(spec, d)
    n = d.v.shape[0]
    hs = [q.h if q.h is not None else np.zeros((n, 3, 3)) for q in ds]
    return (np.stack([q.v for q in ds], axis=1), np.stack([q.g for q in ds], axis=1),
            np.stack(hs, axis=1))
