"""Forward-mode dual numbers over R^3 (value, gradient and optionally Hessian),
vectorised over edges.

The oracle needs dY/dr and dphi/dr for the position chain rule of eqs. 20 and 22 and
for the directional terms of eqs. 23-24, and the second derivatives for the position
gradient of the double backward (the tangent of the first-order position gradient,
whose own chain rule runs through dY/dr and dphi/dr again).  Rather than
hand-deriving derivative polynomials, every edge quantity is computed once on Dual
numbers whose gradient slot starts as the identity on the edge vector r (and whose
Hessian slot, when requested, starts at zero); the derivatives are then exact up to
rounding by construction.  A Dual without a Hessian slot (``h is None``) behaves as a
first-order number; mixing the two treats the missing slot as zero.
"""

import numpy as np


def _hsum(a, b):
    if a is None:
        return b
    if b is None:
        return a
    return a + b


def _outer(a, b):
    return a[:, :, None] * b[:, None, :]


class Dual:
    __slots__ = ("v", "g", "h")

    def __init__(self, v, g, h=None):
        self.v = np.asarray(v, dtype=np.float64)          # [E]
        self.g = np.asarray(g, dtype=np.float64)          # [E, 3]
        self.h = None if h is None else np.asarray(h, dtype=np.float64)   # [E, 3, 3]

    @staticmethod
    def const(c, n):
        return Dual(np.full(n, float(c)), np.zeros((n, 3)))

    def _chain(self, f0, f1, f2):
        """f(self) given f, f' and f'' evaluated at self.v."""
        h = None
        if self.h is not None:
            h = f2[:, None, None] * _outer(self.g, self.g) + f1[:, None, None] * self.h
        return Dual(f0, self.g * f1[:, None], h)

    # arithmetic ---------------------------------------------------------------
    def __add__(self, o):
        if isinstance(o, Dual):
            return Dual(self.v + o.v, self.g + o.g, _hsum(self.h, o.h))
        return Dual(self.v + o, self.g, self.h)

    __radd__ = __add__

    def __neg__(self):
        return Dual(-self.v, -self.g, None if self.h is None else -self.h)

    def __sub__(self, o):
        return self + (-o)

    def __rsub__(self, o):
        return (-self) + o

    def __mul__(self, o):
        if isinstance(o, Dual):
            h = None
            if self.h is not None or o.h is not None:
                h = _outer(self.g, o.g) + _outer(o.g, self.g)
                if self.h is not None:
                    h = h + self.h * o.v[:, None, None]
                if o.h is not None:
                    h = h + o.h * self.v[:, None, None]
            return Dual(self.v * o.v, self.g * o.v[:, None] + o.g * self.v[:, None], h)
        return Dual(self.v * o, self.g * o, None if self.h is None else self.h * o)

    __rmul__ = __mul__

    def __truediv__(self, o):
        if isinstance(o, Dual):
            inv = 1.0 / o.v
            q = Dual(self.v * inv, (self.g - o.g * (self.v * inv)[:, None]) * inv[:, None])
            if self.h is not None or o.h is not None:
                # from self = q * o:  H_self = H_q o + g_q g_o^T + g_o g_q^T + q H_o
                h = -(_outer(q.g, o.g) + _outer(o.g, q.g))
                if self.h is not None:
                    h = h + self.h
                if o.h is not None:
                    h = h - o.h * q.v[:, None, None]
                q.h = h * inv[:, None, None]
            return q
        return Dual(self.v / o, self.g / o, None if self.h is None else self.h / o)

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
            d1 = np.where(s > 0, 0.5 / s, 0.0)
            d2 = np.where(s > 0, -0.25 / (s * s * s), 0.0)
        return self._chain(s, d1, d2)

    def sin(self):
        s, c = np.sin(self.v), np.cos(self.v)
        return self._chain(s, c, -s)

    def cos(self):
        s, c = np.sin(self.v), np.cos(self.v)
        return self._chain(c, -s, -c)

    def exp(self):
        e = np.exp(self.v)
        return self._chain(e, e, e)

    def where(self, mask, other):
        """Select self where mask else other (both Duals)."""
        h = None
        if self.h is not None or other.h is not None:
            n = self.v.shape[0]
            a = self.h if self.h is not None else np.zeros((n, 3, 3))
            b = other.h if other.h is not None else np.zeros((n, 3, 3))
            h = np.where(mask[:, None, None], a, b)
        return Dual(np.where(mask, self.v, other.v), np.where(mask[:, None], self.g, other.g), h)


def edge_vector(r, second=False):
    """Wrap edge vectors r [E,3] as three Duals with d r_k / d r = e_k (and, with
    ``second``, a zero Hessian slot so that second derivatives are carried)."""
    r = np.asarray(r, dtype=np.float64)
    n = r.shape[0]
    comps = []
    for k in range(3):
        g = np.zeros((n, 3))
        g[:, k] = 1.0
        comps.append(Dual(r[:, k], g, np.zeros((n, 3, 3)) if second else None))
    return comps
