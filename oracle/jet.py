"""Second-order forward-mode differentiation of functions of a 3-vector (fp64).

Test infrastructure only (see ``oracle/__init__``).

A Jet carries, for arrays of points, a value f, its gradient df/dr (3) and
its Hessian d2f/dr2 (3x3) with respect to one 3-vector r.  Sums, products,
integer powers, reciprocals and square roots follow the first and second
order chain and product rules:

    (a b)'  = a' b + a b'          (a b)'' = a'' b + a b'' + a' b'^T + b' a'^T
    f(a)'   = f'(a) a'             f(a)''  = f'(a) a'' + f''(a) a' a'^T

so any function written with these operations (the polynomial real
spherical harmonics of ``oracle.sh`` among them) yields exact derivatives up
to rounding.  This is the textbook construction of forward-mode automatic
differentiation, carried to second order.
"""
import numpy as np


class Jet:
    __array_priority__ = 100  # numpy scalars defer to Jet's reflected operators

    def __init__(self, v, g, h):
        self.v = np.asarray(v, dtype=np.float64)
        self.g = np.asarray(g, dtype=np.float64)
        self.h = np.asarray(h, dtype=np.float64)

    @staticmethod
    def variables(r):
        """The three coordinates of points r [..., 3] as Jets."""
        r = np.asarray(r, dtype=np.float64)
        shape = r.shape[:-1]
        out = []
        for k in range(3):
            g = np.zeros(shape + (3,))
            g[..., k] = 1.0
            out.append(Jet(r[..., k], g, np.zeros(shape + (3, 3))))
        return out

    def _const(self, c):
        c = np.asarray(c, dtype=np.float64)
        v = np.broadcast_to(c, self.v.shape).astype(np.float64)
        return Jet(v, np.zeros(self.g.shape), np.zeros(self.h.shape))

    def _lift(self, o):
        return o if isinstance(o, Jet) else self._const(o)

    def __add__(self, o):
        o = self._lift(o)
        return Jet(self.v + o.v, self.g + o.g, self.h + o.h)

    __radd__ = __add__

    def __neg__(self):
        return Jet(-self.v, -self.g, -self.h)

    def __sub__(self, o):
        return self + (-self._lift(o))

    def __rsub__(self, o):
        return self._lift(o) - self

    def __mul__(self, o):
        if not isinstance(o, Jet):
            c = np.asarray(o, dtype=np.float64)
            return Jet(self.v * c, self.g * c[..., None], self.h * c[..., None, None])
        outer = self.g[..., :, None] * o.g[..., None, :]
        return Jet(self.v * o.v,
                   self.g * o.v[..., None] + self.v[..., None] * o.g,
                   self.h * o.v[..., None, None] + self.v[..., None, None] * o.h + outer
                   + np.swapaxes(outer, -1, -2))

    __rmul__ = __mul__

    def __pow__(self, n):
        if not isinstance(n, int) or n < 0:
            raise ValueError("only non-negative integer powers")
        out = self._const(1.0)
        for _ in range(n):
            out = out * self
        return out

    def _chain(self, f0, f1, f2):
        """f(self) given f, f' and f'' evaluated at self.v."""
        outer = self.g[..., :, None] * self.g[..., None, :]
        return Jet(f0, f1[..., None] * self.g, f1[..., None, None] * self.h + f2[..., None, None] * outer)

    def reciprocal(self):
        v = self.v
        return self._chain(1.0 / v, -1.0 / v ** 2, 2.0 / v ** 3)

    def sqrt(self):
        s = np.sqrt(self.v)
        return self._chain(s, 0.5 / s, -0.25 / (s * self.v))

    def __truediv__(self, o):
        if not isinstance(o, Jet):
            return self * (1.0 / np.asarray(o, dtype=np.float64))
        return self * o.reciprocal()
