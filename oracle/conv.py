"""The edge-conditioned tensor-product convolution, evaluated the plain way (oracle).

Sobek: Streaming Equivariant Tensor Product Convolutions (arXiv 2607.18074):

* forward: eq. 11 with the radial projection of eqs. 12-13 materialised per edge
  (w_e = phi_e A), each path contributing eq. 6 (uvw) or eq. 7 (uvu);
* backward: eqs. 18-22 (edge scalar h, radial-parameter adjoint A_bar, embedding
  adjoint phi_bar, operand adjoints x_bar and Y_bar), then the position gradient by
  the chain rule through Y(r_hat) and phi(|r|) with r_e = pos[src] - pos[dst]
  (eq. 8, j = source, i = receiver);
* double backward: eqs. 23-27 and 29-30 for directions (x_dot, pos_dot, A_dot) and
  the first-order adjoint direction set to zero, which is what an autograd engine
  asks for after a first backward taken with create_graph: for
      Lambda = <gg_x, x_bar> + <gg_pos, pos_bar> + <gg_A, A_bar>
  it returns dLambda/dx (eq. 30), dLambda/dA (eq. 27) and dLambda/dm_bar (eq. 25);
  double_backward_pos adds dLambda/dpos, the tangent of the first-order position
  gradient, through the second derivatives of Y and phi.
* forward_streaming: the receiver-factorised order of eqs. 16 and 32-35 (state S,
  then m = S A).  Used only by the self-test that both orders agree (eq. 15 = eq. 16).
* forward_embedded / backward_embedded: the same with the edge embedding phi_e and the
  harmonics Y_e given per edge instead of computed from positions (the pages' own
  interface, which returns the edge-owned adjoints phi_bar and Y_bar).

Notation: for path pi with coupling c^pi[m_in, m_sh, m_out] (so3.path_coupling),
    C_{pi,u,mo}(x_j, Y) = sum_{mi,my} c^pi x_{j,u,mi} Y_my             (eq. 32)
and T_{pi,a} with a = (u, w) (uvw) or a = u (uvu) is the output-space vector whose
entries at (block_out, mo, w) (resp. (block_out, mo, u)) equal C_{pi,u,mo}.

Edges are given by a receiver-sorted CSR: receiver i owns edges row_ptr[i] ..
row_ptr[i+1]-1, and src[e] is the source of edge e.  Every function takes an optional
``edges`` array restricting the sums to a subset of edge ids (used to evaluate sampled
rows of large problems exactly).
"""

from dataclasses import dataclass, field

import numpy as np

from . import irreps as _irreps
from . import so3, radial as _radial


@dataclass
class Plan:
    blocks_in: list
    blocks_out: list
    lmax: int
    mode: str
    radial: _radial.RadialSpec
    paths: list
    coupling: list = field(default_factory=list)

    @property
    def dim_in(self):
        return _irreps.width(self.blocks_in)

    @property
    def dim_out(self):
        return _irreps.width(self.blocks_out)

    @property
    def n_w(self):
        return _irreps.num_weights(self.paths)

    @property
    def n_sh(self):
        return (self.lmax + 1) ** 2

    def fan_in_per_column(self):
        """Fan-in used to scale N(0,1) weights (uvw: K*C_in, uvu: K), per column."""
        f = np.zeros(self.n_w)
        K = self.radial.num_basis
        for p in self.paths:
            f[p.w_offset:p.w_offset + p.w_count] = K * (p.c_in if self.mode == "uvw" else 1)
        return f


def make_plan(irreps_in, lmax, irreps_out, mode, radial_spec):
    bi = _irreps.parse(irreps_in)
    bo = _irreps.parse(irreps_out)
    ps = _irreps.paths(bi, lmax, bo, mode)
    cs = [so3.path_coupling(p.l_in, p.l_sh, p.l_out) for p in ps]
    return Plan(bi, bo, lmax, mode, radial_spec, ps, cs)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def receivers_of(row_ptr):
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    return np.repeat(np.arange(row_ptr.shape[0] - 1), np.diff(row_ptr))


def _edge_batches(n_edges, n_w, edges):
    ids = np.arange(n_edges) if edges is None else np.asarray(edges, dtype=np.int64)
    # temporaries stay below ~16 MB so the allocator reuses memory across batches
    step = max(1, int(2 ** 21 // max(1, n_w)))
    for s in range(0, ids.shape[0], step):
        yield ids[s:s + step]


def _block(arr, b):
    """Rows of a node tensor restricted to block b, as [E, 2l+1, C]."""
    return arr[:, b.offset:b.offset + b.size].reshape(arr.shape[0], b.dim, b.mul)


def _couple(c, xj, ysh):
    """Eq. 32: C[e, mo, u] = sum_{mi,my} c[mi,my,mo] x[e,mi,u] Y[e,my]."""
    return np.einsum("ijk,eiu,ej->eku", c, xj, ysh, optimize=True)


def _couple_adj_x(c, ysh, g):
    """Adjoint of x -> C(x, Y): returns [e, mi, u] from g[e, mo, u]."""
    return np.einsum("ijk,ej,eku->eiu", c, ysh, g, optimize=True)


def _couple_adj_y(c, xj, g):
    """Adjoint of Y -> C(x, Y): returns [e, my] from g[e, mo, u]."""
    return np.einsum("ijk,eiu,eku->ej", c, xj, g, optimize=True)


def _geometry(plan, pos, src, dst, eb, need_grad):
    r = pos[src[eb]] - pos[dst[eb]]                   # eq. 8, r_ij = r_j - r_i
    if need_grad:
        Y, dY = so3.sh_with_grad(plan.lmax, r)
        phi, dphi = _radial.basis_of_vectors(plan.radial, r)
        return Y, dY, phi, dphi
    Y = so3.sh(plan.lmax, r)
    phi, _ = _radial.basis_of_vectors(plan.radial, r)
    return Y, None, phi, None


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def _radial_project(phi, A):
    """Eq. 12: w_{e,c} = sum_q phi_{e,q} A_{q,c}, written out as a sum over q (a BLAS
    matmul with this very short inner dimension is pathologically slow in OpenBLAS)."""
    w = np.zeros((phi.shape[0], A.shape[1]))
    for q in range(A.shape[0]):
        w += phi[:, q:q + 1] * A[q][None, :]
    return w


def _wslice(plan, p, w):
    """Per-edge weights of path p as [E, C_in, C_out] (uvw) or [E, C_in] (uvu)."""
    s = w[:, p.w_offset:p.w_offset + p.w_count]
    if plan.mode == "uvw":
        return s.reshape(w.shape[0], p.c_in, p.c_out)
    return s


def _apply_weights(plan, C, wp):
    """sum_a w_a T_a restricted to one path: [e, mo, w] from C[e, mo, u]."""
    if plan.mode == "uvw":
        return np.einsum("eku,euw->ekw", C, wp, optimize=True)
    return C * wp[:, None, :]


def _adjoint_weights(plan, mb, wp):
    """sum_a w_a (D T_a)^* contracted over the output channel: [e, mo, u]."""
    if plan.mode == "uvw":
        return np.einsum("ekw,euw->eku", mb, wp, optimize=True)
    return mb * wp[:, None, :]


def _edge_h(plan, mb, C):
    """Eq. 18 for one path: h[e, a] = <m_bar_i, T_a>, a flattened like the weights."""
    if plan.mode == "uvw":
        return np.einsum("ekw,eku->euw", mb, C, optimize=True).reshape(C.shape[0], -1)
    return np.einsum("eku,eku->eu", mb, C, optimize=True)


# ---------------------------------------------------------------------------
# forward, eqs. 11-13
# ---------------------------------------------------------------------------

def forward(plan, x, pos, row_ptr, src, A, edges=None):
    pos = _f64(pos)
    src = np.asarray(src, dtype=np.int64)
    dst = receivers_of(row_ptr)
    geo = lambda eb, need: _geometry(plan, pos, src, dst, eb, need)  # noqa: E731
    return _forward(plan, x, src, dst, A, geo, pos.shape[0], edges)


def forward_embedded(plan, x, Y, phi, row_ptr, n_nodes, src, A, edges=None):
    """Forward with the edge embedding given per edge (Sobek's interface, section 3:
    any invariant phi_e, e.g. a learned function of |r_e|, and the harmonics Y_e):
    Y [E, (lmax+1)^2] and phi [E, K] in receiver-CSR edge order."""
    src = np.asarray(src, dtype=np.int64)
    Y, phi = _f64(Y), _f64(phi)
    dst = receivers_of(row_ptr)
    geo = lambda eb, need: (Y[eb], None, phi[eb], None)  # noqa: E731
    return _forward(plan, x, src, dst, A, geo, n_nodes, edges)


def _forward(plan, x, src, dst, A, geo, N, edges):
    x, A = _f64(x), _f64(A)
    out = np.zeros((N, plan.dim_out))
    for eb in _edge_batches(src.shape[0], plan.n_w, edges):
        if eb.size == 0:
            continue
        Y, _, phi, _ = geo(eb, False)
        w = _radial_project(phi, A)                     # eqs. 12-13: W = phi A
        xs = x[src[eb]]
        z = np.zeros((eb.size, plan.dim_out))
        for p, c in zip(plan.paths, plan.coupling):
            bi, bo = plan.blocks_in[p.block_in], plan.blocks_out[p.block_out]
            C = _couple(c, _block(xs, bi), Y[:, p.l_sh ** 2:(p.l_sh + 1) ** 2])
            zz = _apply_weights(plan, C, _wslice(plan, p, w))   # eq. 6 / eq. 7
            z[:, bo.offset:bo.offset + bo.size] += zz.reshape(eb.size, -1)
        np.add.at(out, dst[eb], z)                      # eq. 11: sum over j in N(i)
    return out


# ---------------------------------------------------------------------------
# backward, eqs. 18-22 + chain rule to positions
# ---------------------------------------------------------------------------

def backward(plan, x, pos, row_ptr, src, A, grad_out, edges=None):
    """Returns (grad_x [N, dim_in], grad_pos [N, 3], grad_A [K, N_w])."""
    pos = _f64(pos)
    src = np.asarray(src, dtype=np.int64)
    dst = receivers_of(row_ptr)
    N = pos.shape[0]
    gpos = np.zeros((N, 3))

    def edge_adjoints(eb, dY, dphi, ybar, phibar):
        g = np.einsum("esk,es->ek", dY, ybar) + np.einsum("eqk,eq->ek", dphi, phibar)
        np.add.at(gpos, src[eb], g)
        np.add.at(gpos, dst[eb], -g)

    geo = lambda eb, need: _geometry(plan, pos, src, dst, eb, need)  # noqa: E731
    gx, gA = _backward(plan, x, src, dst, A, grad_out, geo, N, edges, edge_adjoints)
    return gx, gpos, gA


def backward_embedded(plan, x, Y, phi, row_ptr, n_nodes, src, A, grad_out, edges=None):
    """Backward of forward_embedded.  Returns (grad_x [N, dim_in], grad_A [K, N_w],
    grad_phi [E, K] (eq. 20), grad_Y [E, (lmax+1)^2] (eq. 22)), the last two edge-owned."""
    src = np.asarray(src, dtype=np.int64)
    Y, phi = _f64(Y), _f64(phi)
    dst = receivers_of(row_ptr)
    gphi = np.zeros_like(phi)
    gY = np.zeros_like(Y)

    def edge_adjoints(eb, dY, dphi, ybar, phibar):
        gY[eb] = ybar
        gphi[eb] = phibar

    geo = lambda eb, need: (Y[eb], None, phi[eb], None)  # noqa: E731
    gx, gA = _backward(plan, x, src, dst, A, grad_out, geo, n_nodes, edges, edge_adjoints)
    return gx, gA, gphi, gY


def _backward(plan, x, src, dst, A, grad_out, geo, N, edges, edge_adjoints):
    x, A, mbar = _f64(x), _f64(A), _f64(grad_out)
    gx = np.zeros((N, plan.dim_in))
    gA = np.zeros_like(A)
    for eb in _edge_batches(src.shape[0], plan.n_w, edges):
        if eb.size == 0:
            continue
        Y, dY, phi, dphi = geo(eb, True)
        w = _radial_project(phi, A)
        xs = x[src[eb]]
        mb_rows = mbar[dst[eb]]
        h = np.zeros((eb.size, plan.n_w))
        ybar = np.zeros((eb.size, plan.n_sh))
        xbar = np.zeros((eb.size, plan.dim_in))
        for p, c in zip(plan.paths, plan.coupling):
            bi, bo = plan.blocks_in[p.block_in], plan.blocks_out[p.block_out]
            sl = slice(p.l_sh ** 2, (p.l_sh + 1) ** 2)
            xj = _block(xs, bi)
            mb = _block(mb_rows, bo)
            C = _couple(c, xj, Y[:, sl])
            h[:, p.w_offset:p.w_offset + p.w_count] = _edge_h(plan, mb, C)      # eq. 18
            G = _adjoint_weights(plan, mb, _wslice(plan, p, w))
            xbar[:, bi.offset:bi.offset + bi.size] += _couple_adj_x(c, Y[:, sl], G).reshape(eb.size, -1)  # eq. 21
            ybar[:, sl] += _couple_adj_y(c, xj, G)                               # eq. 22
        gA += phi.T @ h                                                           # eq. 19
        phibar = h @ A.T                                                          # eq. 20
        edge_adjoints(eb, dY, dphi, ybar, phibar)
        np.add.at(gx, src[eb], xbar)
    return gx, gA


# ---------------------------------------------------------------------------
# double backward, eqs. 23-27 and 29-30
# ---------------------------------------------------------------------------

def double_backward(plan, x, pos, row_ptr, src, A, grad_out, gg_x=None, gg_pos=None,
                    gg_A=None, edges=None):
    """Returns (grad_x, grad_A, grad_grad_out) = dLambda/d(x, A, m_bar)."""
    x, pos, A, mbar = _f64(x), _f64(pos), _f64(A), _f64(grad_out)
    src = np.asarray(src, dtype=np.int64)
    dst = receivers_of(row_ptr)
    N = pos.shape[0]
    xd = np.zeros_like(x) if gg_x is None else _f64(gg_x)
    pd = np.zeros_like(pos) if gg_pos is None else _f64(gg_pos)
    Ad = np.zeros_like(A) if gg_A is None else _f64(gg_A)
    gx = np.zeros((N, plan.dim_in))
    gA = np.zeros_like(A)
    mdot = np.zeros((N, plan.dim_out))
    for eb in _edge_batches(src.shape[0], plan.n_w, edges):
        if eb.size == 0:
            continue
        Y, dY, phi, dphi = _geometry(plan, pos, src, dst, eb, True)
        rdot = pd[src[eb]] - pd[dst[eb]]
        Ydot = np.einsum("esk,ek->es", dY, rdot)
        phidot = np.einsum("eqk,ek->eq", dphi, rdot)
        w = _radial_project(phi, A)
        wdot = _radial_project(phidot, A) + _radial_project(phi, Ad)            # eq. 23
        xs, xds = x[src[eb]], xd[src[eb]]
        mb_rows = mbar[dst[eb]]
        h = np.zeros((eb.size, plan.n_w))
        hdot = np.zeros((eb.size, plan.n_w))
        z = np.zeros((eb.size, plan.dim_out))
        xbar2 = np.zeros((eb.size, plan.dim_in))
        for p, c in zip(plan.paths, plan.coupling):
            bi, bo = plan.blocks_in[p.block_in], plan.blocks_out[p.block_out]
            sl = slice(p.l_sh ** 2, (p.l_sh + 1) ** 2)
            xj, xdj = _block(xs, bi), _block(xds, bi)
            mb = _block(mb_rows, bo)
            C = _couple(c, xj, Y[:, sl])
            Cdot = _couple(c, xdj, Y[:, sl]) + _couple(c, xj, Ydot[:, sl])       # eq. 24
            wp, wdp = _wslice(plan, p, w), _wslice(plan, p, wdot)
            zz = _apply_weights(plan, C, wdp) + _apply_weights(plan, Cdot, wp)   # eq. 25
            z[:, bo.offset:bo.offset + bo.size] += zz.reshape(eb.size, -1)
            sw = slice(p.w_offset, p.w_offset + p.w_count)
            h[:, sw] = _edge_h(plan, mb, C)                                      # eq. 18
            hdot[:, sw] = _edge_h(plan, mb, Cdot)                                # eq. 26
            # eqs. 29-30: B^x = D_x T(Y)^* m_bar, its direction uses Y_dot
            G, Gdot = _adjoint_weights(plan, mb, wp), _adjoint_weights(plan, mb, wdp)
            xb = _couple_adj_x(c, Y[:, sl], Gdot) + _couple_adj_x(c, Ydot[:, sl], G)
            xbar2[:, bi.offset:bi.offset + bi.size] += xb.reshape(eb.size, -1)
        gA += phidot.T @ h + phi.T @ hdot                                         # eq. 27
        np.add.at(mdot, dst[eb], z)
        np.add.at(gx, src[eb], xbar2)
    return gx, gA, mdot


def double_backward_pos(plan, x, pos, row_ptr, src, A, grad_out, gg_x=None, gg_pos=None,
                        gg_A=None, edges=None):
    """dLambda/dpos [N, 3] for the Lambda of double_backward.

    The pages stop at the first-order terms of eqs. 23-31 (the position gradient of the
    double backward needs second derivatives of Y and phi, which they do not write out).
    Reading taken: pos_bar = sum_e (+g_e at src, -g_e at dst) with
        g_e = (dphi/dr)^T phi_bar_e + (dY/dr)^T Y_bar_e            (eqs. 20, 22 + chain rule)
    and, Lambda being the derivative of <m_bar, m> along (x_dot, pos_dot, A_dot),
    dLambda/dpos = d/d eps pos_bar(x + eps x_dot, pos + eps pos_dot, A + eps A_dot):
        g_dot_e = (dphi/dr)^T phi_bar_dot + (dY/dr)^T Y_bar_dot
                  + (d2phi/dr2 . r_dot)^T phi_bar + (d2Y/dr2 . r_dot)^T Y_bar,
    with phi_bar_dot = h_dot A^T + h A_dot^T (eqs. 20, 26) and Y_bar_dot the tangent of
    eq. 22 (x -> x_dot, and w -> w_dot of eq. 23), scattered like g_e."""
    x, pos, A, mbar = _f64(x), _f64(pos), _f64(A), _f64(grad_out)
    src = np.asarray(src, dtype=np.int64)
    dst = receivers_of(row_ptr)
    N = pos.shape[0]
    xd = np.zeros_like(x) if gg_x is None else _f64(gg_x)
    pd = np.zeros_like(pos) if gg_pos is None else _f64(gg_pos)
    Ad = np.zeros_like(A) if gg_A is None else _f64(gg_A)
    gpos = np.zeros((N, 3))
    for eb in _edge_batches(src.shape[0], plan.n_w, edges):
        if eb.size == 0:
            continue
        r = pos[src[eb]] - pos[dst[eb]]                                          # eq. 8
        Y, dY, HY = so3.sh_with_hessian(plan.lmax, r)
        phi, dphi, Hphi = _radial.basis_with_hessian(plan.radial, r)
        rdot = pd[src[eb]] - pd[dst[eb]]
        Ydot = np.einsum("esk,ek->es", dY, rdot)
        phidot = np.einsum("eqk,ek->eq", dphi, rdot)
        w = _radial_project(phi, A)
        wdot = _radial_project(phidot, A) + _radial_project(phi, Ad)            # eq. 23
        xs, xds = x[src[eb]], xd[src[eb]]
        mb_rows = mbar[dst[eb]]
        h = np.zeros((eb.size, plan.n_w))
        hdot = np.zeros((eb.size, plan.n_w))
        ybar = np.zeros((eb.size, plan.n_sh))
        ybardot = np.zeros((eb.size, plan.n_sh))
        for p, c in zip(plan.paths, plan.coupling):
            bi, bo = plan.blocks_in[p.block_in], plan.blocks_out[p.block_out]
            sl = slice(p.l_sh ** 2, (p.l_sh + 1) ** 2)
            xj, xdj = _block(xs, bi), _block(xds, bi)
            mb = _block(mb_rows, bo)
            C = _couple(c, xj, Y[:, sl])
            Cdot = _couple(c, xdj, Y[:, sl]) + _couple(c, xj, Ydot[:, sl])       # eq. 24
            sw = slice(p.w_offset, p.w_offset + p.w_count)
            h[:, sw] = _edge_h(plan, mb, C)                                      # eq. 18
            hdot[:, sw] = _edge_h(plan, mb, Cdot)                                # eq. 26
            wp, wdp = _wslice(plan, p, w), _wslice(plan, p, wdot)
            G, Gdot = _adjoint_weights(plan, mb, wp), _adjoint_weights(plan, mb, wdp)
            ybar[:, sl] += _couple_adj_y(c, xj, G)                               # eq. 22
            ybardot[:, sl] += _couple_adj_y(c, xdj, G) + _couple_adj_y(c, xj, Gdot)
        phibar = h @ A.T                                                          # eq. 20
        phibardot = hdot @ A.T + h @ Ad.T
        gdot = (np.einsum("esk,es->ek", dY, ybardot) + np.einsum("eqk,eq->ek", dphi, phibardot)
                + np.einsum("eskl,el,es->ek", HY, rdot, ybar)
                + np.einsum("eqkl,el,eq->ek", Hphi, rdot, phibar))
        np.add.at(gpos, src[eb], gdot)
        np.add.at(gpos, dst[eb], -gdot)
    return gpos


# ---------------------------------------------------------------------------
# receiver-factorised order, eqs. 16 and 32-35 (self-test only)
# ---------------------------------------------------------------------------

def forward_streaming(plan, x, pos, row_ptr, src, A):
    """S_{i,pi,q,u,mo} = sum_j phi_jq C_{pi,u,mo} (eq. 33), then m = S A (eqs. 34-35)."""
    x, pos, A = _f64(x), _f64(pos), _f64(A)
    src = np.asarray(src, dtype=np.int64)
    dst = receivers_of(row_ptr)
    N = pos.shape[0]
    K = plan.radial.num_basis
    eb = np.arange(src.shape[0])
    out = np.zeros((N, plan.dim_out))
    if eb.size == 0:
        return out
    Y, _, phi, _ = _geometry(plan, pos, src, dst, eb, False)
    xs = x[src]
    for p, c in zip(plan.paths, plan.coupling):
        bi, bo = plan.blocks_in[p.block_in], plan.blocks_out[p.block_out]
        C = _couple(c, _block(xs, bi), Y[:, p.l_sh ** 2:(p.l_sh + 1) ** 2])
        S = np.zeros((N, K, bo.dim, p.c_in))
        np.add.at(S, dst, np.einsum("eq,eku->eqku", phi, C))                     # eq. 33
        Ap = A[:, p.w_offset:p.w_offset + p.w_count]
        if plan.mode == "uvw":
            m = np.einsum("nqku,quw->nkw", S, Ap.reshape(K, p.c_in, p.c_out))     # eq. 34
        else:
            m = np.einsum("nqku,qu->nku", S, Ap)
        out[:, bo.offset:bo.offset + bo.size] += m.reshape(N, -1)
    return out
