"""Seeded synthetic workloads: node positions, receiver-sorted kNN graphs, features.

This module is shared by the tests, the benchmark and the float64 oracle's callers.
It holds no tensor-product arithmetic: it draws positions and random arrays and
builds graphs.  Shapes that depend on the operator (feature widths, weight count,
per-column fan-in, which output columns are scalars) are passed in by the caller.

Workload recipes (the pages name no dataset; these stand in for the molecular and
materials graphs they describe):

* positions uniform in an open cube (no periodic images); side chosen from a stated
  number density (0.1 per cubic Angstrom unless a side is given);
* fixed-degree kNN: receiver i's in-neighbours are its k nearest other nodes
  (float64 distances, ties broken by lower index, self excluded);
* variable degree: d_i drawn from the discrete power law P(d) ~ d^-alpha on
  [d_min, d_max], neighbours are the d_i nearest other nodes;
* within a receiver row the sources are listed in ascending node index, rows in
  receiver order (a dst-sorted CSR: row_ptr[N+1], src[E], int32);
* features, weights and upstream gradients ~ N(0, 1) drawn in float64 and rounded
  to float32 (weights then divided by sqrt(fan_in) per column).

Seed of configuration c is 1000 + c unless given; draw order is positions, degrees,
x, W, grad_out, F_ref, tangents.
"""

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Config:
    cfg: int
    name: str
    n_nodes: int
    k: int                   # fixed degree, or 0 for the power-law degree draw
    irreps_in: str
    sh_lmax: int
    irreps_out: str
    mode: str                # "uvw" | "uvu"
    radial: str              # "bessel" | "gaussian"
    num_basis: int
    r_cut: float
    r_min: float = 0.0
    r_max: float = 0.0
    side: float = 0.0        # 0: from density
    density: float = 0.1
    deg_alpha: float = 2.0
    deg_min: int = 16
    deg_max: int = 512
    passes: tuple = ("fwd",)

    def cube_side(self, n=None):
        n = self.n_nodes if n is None else n
        if self.side > 0 and n == self.n_nodes:
            return self.side
        if self.side > 0:
            return self.side * (n / self.n_nodes) ** (1.0 / 3.0)
        return (n / self.density) ** (1.0 / 3.0)


CONFIGS = {
    1: Config(1, "tiny uvw forward, N=64 k=8", 64, 8, "8x0e+8x1o", 2, "8x0e+8x1o+8x2e",
              "uvw", "bessel", 8, 3.0, side=6.0, passes=("fwd",)),
    2: Config(2, "uvw forward+backward, N=4096 k=32, 64x(0e+1o+2e), lmax 3", 4096, 32,
              "64x0e+64x1o+64x2e", 3, "64x0e+64x1o+64x2e", "uvw", "bessel", 8, 5.0,
              passes=("fwd", "bwd")),
    3: Config(3, "uvu forward+backward, N=16384 k=24, 128x(0e+1o+2e), lmax 2", 16384, 24,
              "128x0e+128x1o+128x2e", 2, "128x0e+128x1o+128x2e", "uvu", "gaussian", 16, 6.0,
              r_min=0.0, r_max=6.0, passes=("fwd", "bwd")),
    4: Config(4, "edge-scaling uvw, N=50000 power-law degree 16..512", 50000, 0,
              "128x0e+64x1o+32x2e+16x3o", 3, "128x0e+64x1o+32x2e+16x3o", "uvw", "bessel", 8,
              6.0, passes=("fwd", "bwd")),
    5: Config(5, "force-training double backward, N=8192 k=32, 32x(0e+1o+2e)", 8192, 32,
              "32x0e+32x1o+32x2e", 2, "32x0e+32x1o+32x2e", "uvw", "bessel", 8, 5.0,
              passes=("fwd", "bwd", "dbl")),
}


# Feature-profile grids.  The pages time sixteen fully connected uvw profiles on a fixed
# graph, varying angular order, channel width, scalar fraction and radial-operator size,
# and channelwise uvu at three equal-multiplicity widths for each angular order; they do
# not list the profiles.  Reading used here: uvw = lmax {2, 3} x width C {32, 64} x
# {evenly spread: C per l; scalar-heavy: 4C x 0e, C/2 x 1o, C/4 x 2e, C/8 x 3o} x Bessel
# K {8, 16}; uvu = lmax {1, 2, 3} x C {32, 64, 128} with C per l, Gaussian K=16 on
# [0, 6].  Irreps in = out, SH lmax = feature lmax, natural parity (0e, 1o, 2e, 3o).  The
# fixed graph is the uvw forward+backward workload's (N=4096, kNN k=32, density 0.1).

_PARITY = "eoeo"


def _irreps(mults):
    return "+".join(f"{m}x{l}{_PARITY[l]}" for l, m in enumerate(mults) if m > 0)


def profile_configs(n_nodes=4096, k=32):
    out = []
    idx = 100
    for lmax in (2, 3):
        for c in (32, 64):
            for kind in ("even", "scalar-heavy"):
                if kind == "even":
                    mults = [c] * (lmax + 1)
                else:
                    mults = [4 * c, c // 2, c // 4, c // 8][:lmax + 1]
                irr = _irreps(mults)
                for kb in (8, 16):
                    out.append(Config(idx, f"uvw lmax {lmax} C{c} {kind} K{kb}: {irr}", n_nodes, k, irr, lmax,
                                      irr, "uvw", "bessel", kb, 5.0, passes=("fwd", "bwd", "dbl")))
                    idx += 1
    for lmax in (1, 2, 3):
        for c in (32, 64, 128):
            irr = _irreps([c] * (lmax + 1))
            out.append(Config(idx, f"uvu lmax {lmax} C{c}: {irr}", n_nodes, k, irr, lmax, irr, "uvu",
                              "gaussian", 16, 6.0, r_min=0.0, r_max=6.0, passes=("fwd", "bwd", "dbl")))
            idx += 1
    return out


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))


def powerlaw_degrees(rng, n, alpha, dmin, dmax):
    d = np.arange(dmin, dmax + 1, dtype=np.float64)
    p = d ** (-alpha)
    p /= p.sum()
    return rng.choice(np.arange(dmin, dmax + 1), size=n, p=p).astype(np.int64)


def knn_csr(pos, degrees):
    """Receiver-sorted CSR of the degrees[i] nearest other nodes of every node i."""
    from scipy.spatial import cKDTree
    pos64 = np.asarray(pos, dtype=np.float64)
    n = pos64.shape[0]
    degrees = np.asarray(degrees, dtype=np.int64)
    if n == 0:
        return np.zeros(1, np.int32), np.zeros(0, np.int32)
    if degrees.max(initial=0) > n - 1:
        raise ValueError("degree larger than the number of other nodes")
    tree = cKDTree(pos64)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(degrees)
    src = np.zeros(row_ptr[-1], dtype=np.int64)
    order = np.argsort(degrees, kind="stable")
    chunk = 2048
    for s in range(0, n, chunk):
        ids = order[s:s + chunk]
        kq = int(degrees[ids].max()) + 1
        # a few extra candidates so that distance ties at the boundary resolve by index
        kq = min(n, kq + 4)
        _, nb = tree.query(pos64[ids], k=kq)
        nb = np.atleast_2d(nb)
        for row, i in enumerate(ids):
            cand = nb[row]
            cand = cand[(cand != i) & (cand < n)]
            dist = np.sum((pos64[cand] - pos64[i]) ** 2, axis=1)
            sel = cand[np.lexsort((cand, dist))][:degrees[i]]
            src[row_ptr[i]:row_ptr[i + 1]] = np.sort(sel)
    return row_ptr.astype(np.int32), src.astype(np.int32)


@dataclass
class Graph:
    pos: np.ndarray       # float32 [N, 3]
    row_ptr: np.ndarray   # int32 [N + 1]
    src: np.ndarray       # int32 [E]

    @property
    def n_nodes(self):
        return self.pos.shape[0]

    @property
    def n_edges(self):
        return self.src.shape[0]


def make_graph(cfg, n_nodes=None, seed=None, k=None):
    """Positions and kNN graph of configuration ``cfg`` (optionally resized)."""
    c = CONFIGS[cfg] if isinstance(cfg, int) else cfg
    n = c.n_nodes if n_nodes is None else int(n_nodes)
    rng = np.random.default_rng(1000 + c.cfg if seed is None else seed)
    side = c.cube_side(n)
    pos = _f32(rng.uniform(0.0, side, size=(n, 3)))
    kk = c.k if k is None else k
    if kk > 0:
        deg = np.full(n, min(kk, max(n - 1, 0)), dtype=np.int64)
    else:
        deg = powerlaw_degrees(rng, n, c.deg_alpha, c.deg_min, min(c.deg_max, n - 1))
    row_ptr, src = knn_csr(pos.astype(np.float64), deg)
    return Graph(pos, row_ptr, src), rng


def normal(rng, shape):
    return _f32(rng.standard_normal(size=shape))


def weights(rng, num_basis, fan_in_per_column):
    fan = np.asarray(fan_in_per_column, dtype=np.float64)
    w = rng.standard_normal(size=(num_basis, fan.shape[0])) / np.sqrt(fan)[None, :]
    return _f32(w)

