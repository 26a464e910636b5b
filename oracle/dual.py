"""Forward-mode dual numbers over R^3 (value + gradient), vectorised over edges.

The oracle needs dY/dr and dphi/dr for the position chain rule of eqs. 20 and 22 and
for the directional terms of eqs. 23-24.  Rather than hand-deriving derivative
polynomials, every edge quantity is computed once on Dual numbers whose gradient
slot starts as the identity on the edge vector r; the derivative is then exact up
to rounding by construction.
"""

import numpy as np


class Dual:
    __slots__ = ("v", "g")

    def __init__(self, v, g):
        self.v = np.asarray(v, dtype=np.float64)          # [E]
        self.g = np.asarray(g, dtype=np.float64)          # [E, 3]

    @staticmethod
    def const(c, n):
        return Dual(np.full(n, float(c)), np.zeros((n, 3)))

    # arithmetic ---------------------------------------------------------------
    def __add__(self, o):
        if isinstance(o, Dual):
            return Dual(self.v + o.v, self.g + o.g)
        return Dual(self.v + o, self.g)

    __radd__ = __add__

    def __neg__(self):
        return Dual(-self.v, -self.g)

    def __sub__(self, o):
        return self + (-o)

    def __rsub__(self, o):
        return (-self) + o

    def __mul__(self, o):
        if isinstance(o, Dual):
            return Dual(self.v * o.v, self.g * o.v[:, None] + o.g * self.v[:, None])
        return Dual(self.v * o, self.g * o)

    __rmul__ = __mul__

    def __truediv__(self, o):
        if isinstance(o, Dual):
            inv = 1.0 / o.v
            return Dual(self.v * inv, (self.g - o.g * (self.v * inv)[:, None]) * inv[:, None])
        return Dual(self.v / o, self.g / o)

    def __pow__(self, n):
        assert isinstance(n, int) and n >= 0
        out = Dual.const(1.0, self.v.shape[0])
        for _ in range(n):
            out = out * self
        return out

    # elementary functions -----------------------------------------------------
    def sqrt(self):
        s = np.sqrt(self.v)
        with np.errstate(divide="ignore", invalid="ignore"):
            d = np.where(s > 0, 0.5 / s, 0.0)
        return Dual(s, self.g * d[:, None])

    def sin(self):
        return Dual(np.sin(self.v), self.g * np.cos(self.v)[:, None])

    def cos(self):
        return Dual(np.cos(self.v), -self.g * np.sin(self.v)[:, None])

    def exp(self):
        e = np.exp(self.v)
        return Dual(e, self.g * e[:, None])

    def where(self, mask, other):
        """Select self where mask else other (both Duals)."""
        return Dual(np.where(mask, self.v, other.v), np.where(mask[:, None], self.g, other.g))


def edge_vector(r):
    """Wrap edge vectors r [E,3] as three Duals with d r_k / d r = e_k."""
    r = np.asarray(r, dtype=np.float64)
    n = r.shape[0]
    comps = []
    for k in range(3):
        g = np.zeros((n, 3))
        g[:, k] = 1.0
        comps.append(Dual(r[:, k], g))
    return comps
