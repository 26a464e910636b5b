"""Pins for the oracle's convolution operator and its derivatives (oracle/conv.py).

* O(3) equivariance (rotations and reflections) plus translation invariance of the
  forward, with l > 0 blocks rotated by Wigner-D matrices fitted from the harmonics;
* node-permutation equivariance;
* the scalar-input special case, where the coupling reduces to the identity and the
  output is a closed-form sum of phi * A * x * Y;
* eq. 15 (materialised) equals eq. 16 / eqs. 32-35 (receiver-factorised) to rounding;
* every first-order gradient against finite differences of the forward;
* the double backward against finite differences of the first backward.
"""

import numpy as np
import pytest
from scipy.spatial.transform import Rotation

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, graph, radial, so3

BESSEL = radial.RadialSpec(radial.BESSEL, 6, 2.5)
GAUSS = radial.RadialSpec(radial.GAUSSIAN, 5, 3.0, 0.0, 3.0)

CASES = {
    "uvw": ("3x0e+2x1o+2x2e", 3, "2x0e+3x1o+2x2e+1x3o", "uvw", BESSEL),
    "uvw_odd": ("2x0e+2x1o+1x1e", 2, "2x0e+1x1e+2x1o+1x2e+1x2o", "uvw", BESSEL),
    "uvu": ("3x0e+3x1o+3x2e", 2, "3x0e+3x1o+3x2e", "uvu", GAUSS),
}


def _problem(case, n=10, k=4, seed=0):
    ii, lmax, io, mode, rs = CASES[case]
    plan = conv.make_plan(ii, lmax, io, mode, rs)
    rng = np.random.default_rng(seed)
    pos = rng.uniform(0, 2.5, size=(n, 3))
    row_ptr, src = workloads.knn_csr(pos, np.full(n, k))
    x = rng.normal(size=(n, plan.dim_in))
    A = rng.normal(size=(rs.num_basis, plan.n_w)) / 3
    return plan, x, pos, row_ptr, src, A, rng


def _wigner(l, R, rng):
    pts = rng.normal(size=(64, 3))
    s = slice(l * l, (l + 1) ** 2)
    X, *_ = np.linalg.lstsq(so3.sh(l, pts)[:, s], so3.sh(l, pts @ R.T)[:, s], rcond=None)
    return X.T


def _act(blocks, feats, R0, det, rng):
    out = feats.copy()
    for b in blocks:
        D = _wigner(b.l, R0, rng)
        sign = b.parity if det < 0 else 1
        blk = feats[:, b.offset:b.offset + b.size].reshape(-1, b.dim, b.mul)
        out[:, b.offset:b.offset + b.size] = (sign * np.einsum("ij,njc->nic", D, blk)).reshape(-1, b.size)
    return out


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("improper", [False, True])
def test_forward_o3_equivariant(case, improper, rng):
    plan, x, pos, row_ptr, src, A, _ = _problem(case)
    R0 = Rotation.random(random_state=11).as_matrix()
    R = -R0 if improper else R0
    det = np.linalg.det(R)
    t = np.array([0.3, -1.2, 2.0])
    m = conv.forward(plan, x, pos, row_ptr, src, A)
    m2 = conv.forward(plan, _act(plan.blocks_in, x, R0, det, rng), pos @ R.T + t, row_ptr, src, A)
    expect = _act(plan.blocks_out, m, R0, det, rng)
    assert np.abs(m2 - expect).max() <= 1e-10 * max(1.0, np.abs(m).max())
    assert np.abs(m).max() > 1e-3


@pytest.mark.parametrize("improper", [False, True])
def test_forward_equivariant_with_coincident_nodes(improper, rng):
    # a receiver placed on one of its sources: that zero-length edge still carries the
    # radial limit phi(0) != 0 (Bessel), so its l > 0 harmonics must vanish for the
    # operator to stay O(3) equivariant
    plan, x, pos, row_ptr, src, A, _ = _problem("uvw")
    pos = pos.copy()
    pos[3] = pos[src[row_ptr[3]]]
    assert radial.basis_of_vectors(plan.radial, np.zeros((1, 3)))[0].max() > 0.1
    R0 = Rotation.random(random_state=12).as_matrix()
    R = -R0 if improper else R0
    det = np.linalg.det(R)
    m = conv.forward(plan, x, pos, row_ptr, src, A)
    m2 = conv.forward(plan, _act(plan.blocks_in, x, R0, det, rng), pos @ R.T, row_ptr, src, A)
    expect = _act(plan.blocks_out, m, R0, det, rng)
    assert np.abs(m2 - expect).max() <= 1e-10 * max(1.0, np.abs(m).max())


def test_forward_permutation_equivariant():
    plan, x, pos, row_ptr, src, A, rng = _problem("uvw", n=9, k=3)
    perm = rng.permutation(9)           # new node a is old node perm[a]
    inv = np.argsort(perm)
    dst = conv.receivers_of(row_ptr)
    new_dst, new_src = inv[dst], inv[src]
    order = np.lexsort((new_src, new_dst))
    rp = np.zeros(10, np.int64)
    rp[1:] = np.cumsum(np.bincount(new_dst, minlength=9))
    m = conv.forward(plan, x, pos, row_ptr, src, A)
    m2 = conv.forward(plan, x[perm], pos[perm], rp, new_src[order], A)
    assert np.allclose(m2, m[perm], atol=1e-12)


def test_scalar_input_closed_form():
    """With only 0e inputs every path is 0 x l -> l with c = identity, so
    m_i[w, mo] = sum_j sum_q sum_u phi_jq A[q, u, w] x_ju Y_{l,mo}(r_hat_ij)."""
    rs = radial.RadialSpec(radial.BESSEL, 3, 3.0)
    plan = conv.make_plan("4x0e", 2, "3x0e+3x1o+3x2e", "uvw", rs)
    rng = np.random.default_rng(5)
    n = 3
    pos = rng.uniform(0, 1.5, size=(n, 3))
    row_ptr = np.array([0, 2, 4, 6])
    src = np.array([1, 2, 0, 2, 0, 1])
    x = rng.normal(size=(n, 4))
    A = rng.normal(size=(3, plan.n_w))
    m = conv.forward(plan, x, pos, row_ptr, src, A)
    expect = np.zeros_like(m)
    for i in range(n):
        for e in range(row_ptr[i], row_ptr[i + 1]):
            j = src[e]
            r = pos[j] - pos[i]
            Y = so3.sh(2, r[None])[0]
            phi, _ = radial.basis_of_vectors(rs, r[None])
            for p in plan.paths:
                bo = plan.blocks_out[p.block_out]
                Ap = A[:, p.w_offset:p.w_offset + p.w_count].reshape(3, 4, 3)
                for w in range(3):
                    for mo in range(bo.dim):
                        val = sum(phi[0, q] * Ap[q, u, w] * x[j, u] * Y[p.l_sh ** 2 + mo]
                                  for q in range(3) for u in range(4))
                        expect[i, bo.offset + mo * bo.mul + w] += val
    assert np.allclose(m, expect, atol=1e-12)


@pytest.mark.parametrize("case", list(CASES))
def test_materialised_equals_streaming(case):
    plan, x, pos, row_ptr, src, A, _ = _problem(case, n=14, k=5)
    a = conv.forward(plan, x, pos, row_ptr, src, A)
    b = conv.forward_streaming(plan, x, pos, row_ptr, src, A)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


@pytest.mark.parametrize("case", list(CASES))
def test_backward_matches_finite_differences(case):
    plan, x, pos, row_ptr, src, A, rng = _problem(case, n=7, k=3)
    mbar = rng.normal(size=(7, plan.dim_out))
    gx, gpos, gA = conv.backward(plan, x, pos, row_ptr, src, A, mbar)

    def L(x_, pos_, A_):
        return float(np.sum(mbar * conv.forward(plan, x_, pos_, row_ptr, src, A_)))

    # linear in x and A: one-sided differences with h = 1 are exact up to rounding
    vx = rng.normal(size=x.shape)
    vA = rng.normal(size=A.shape)
    assert np.isclose(L(x + vx, pos, A) - L(x, pos, A), np.sum(gx * vx), rtol=1e-10)
    assert np.isclose(L(x, pos, A + vA) - L(x, pos, A), np.sum(gA * vA), rtol=1e-10)
    # positions: central differences, entry by entry
    h = 1e-5
    fd = np.zeros_like(pos)
    for a in range(pos.shape[0]):
        for k in range(3):
            e = np.zeros_like(pos)
            e[a, k] = h
            fd[a, k] = (L(x, pos + e, A) - L(x, pos - e, A)) / (2 * h)
    assert np.abs(fd - gpos).max() <= 1e-7 * max(1.0, np.abs(gpos).max())
    # translation invariance of the loss: sum of position gradients vanishes
    assert np.abs(gpos.sum(0)).max() <= 1e-10 * max(1.0, np.abs(gpos).max())


@pytest.mark.parametrize("case", list(CASES))
def test_backward_edge_subset_is_additive(case):
    plan, x, pos, row_ptr, src, A, rng = _problem(case, n=9, k=3)
    mbar = rng.normal(size=(9, plan.dim_out))
    E = src.shape[0]
    half = np.arange(0, E, 2)
    rest = np.arange(1, E, 2)
    full = conv.backward(plan, x, pos, row_ptr, src, A, mbar)
    a = conv.backward(plan, x, pos, row_ptr, src, A, mbar, edges=half)
    b = conv.backward(plan, x, pos, row_ptr, src, A, mbar, edges=rest)
    for f, u, v in zip(full, a, b):
        assert np.allclose(f, u + v, atol=1e-12)


@pytest.mark.parametrize("case", list(CASES))
def test_double_backward_matches_finite_differences(case):
    plan, x, pos, row_ptr, src, A, rng = _problem(case, n=7, k=3)
    mbar = rng.normal(size=(7, plan.dim_out))
    ggx = rng.normal(size=x.shape)
    ggp = rng.normal(size=pos.shape)
    ggA = rng.normal(size=A.shape)
    gx2, gA2, gmb = conv.double_backward(plan, x, pos, row_ptr, src, A, mbar, ggx, ggp, ggA)

    def Lam(x_, A_, mb_):
        gx, gpos, gA = conv.backward(plan, x_, pos, row_ptr, src, A_, mb_)
        return float(np.sum(ggx * gx) + np.sum(ggp * gpos) + np.sum(ggA * gA))

    # Lambda is linear in each of x, A and m_bar separately
    base = Lam(x, A, mbar)
    vx, vA, vm = rng.normal(size=x.shape), rng.normal(size=A.shape), rng.normal(size=mbar.shape)
    assert np.isclose(Lam(x + vx, A, mbar) - base, np.sum(gx2 * vx), rtol=1e-9)
    assert np.isclose(Lam(x, A + vA, mbar) - base, np.sum(gA2 * vA), rtol=1e-9)
    assert np.isclose(Lam(x, A, mbar + vm) - base, np.sum(gmb * vm), rtol=1e-9)
    # d Lambda / d m_bar is the forward tangent m_dot: check it against a central
    # difference of the forward along (x_dot, pos_dot, A_dot)
    h = 1e-5
    fp = conv.forward(plan, x + h * ggx, pos + h * ggp, row_ptr, src, A + h * ggA)
    fm = conv.forward(plan, x - h * ggx, pos - h * ggp, row_ptr, src, A - h * ggA)
    assert np.abs((fp - fm) / (2 * h) - gmb).max() <= 1e-6 * max(1.0, np.abs(gmb).max())


def test_double_backward_null_tangents_are_zero():
    plan, x, pos, row_ptr, src, A, rng = _problem("uvw", n=6, k=3)
    mbar = rng.normal(size=(6, plan.dim_out))
    out = conv.double_backward(plan, x, pos, row_ptr, src, A, mbar)
    for t in out:
        assert np.all(t == 0.0)


def test_force_training_invariants():
    """E = sum of scalar outputs is translation invariant, so the forces
    F = -dE/dpos sum to zero; with scalar-only input features E is also rotation
    invariant, so the forces exert no net torque."""
    rng = np.random.default_rng(9)
    plan = conv.make_plan("3x0e", 2, "2x0e+2x1o+1x2e", "uvw", BESSEL)
    pos = rng.uniform(0, 2.5, size=(12, 3))
    row_ptr, src = workloads.knn_csr(pos, np.full(12, 4))
    x = rng.normal(size=(12, plan.dim_in))
    A = rng.normal(size=(BESSEL.num_basis, plan.n_w))
    mbar = np.zeros((12, plan.dim_out))
    for b in plan.blocks_out:
        if b.l == 0 and b.parity == 1:
            mbar[:, b.offset:b.offset + b.size] = 1.0
    _, gpos, _ = conv.backward(plan, x, pos, row_ptr, src, A, mbar)
    F = -gpos
    scale = np.abs(F).max()
    assert scale > 1e-6
    assert np.abs(F.sum(0)).max() <= 1e-10 * scale
    assert np.abs(np.cross(pos, F).sum(0)).max() <= 1e-10 * scale * np.abs(pos).max()


def test_source_view_is_stable_grouping():
    row_ptr = np.array([0, 2, 3, 5])
    src = np.array([2, 1, 0, 0, 1])
    t_ptr, t_eid, t_dst = graph.source_view(row_ptr, src, 3)
    assert t_ptr.tolist() == [0, 2, 4, 5]
    assert t_eid.tolist() == [2, 3, 1, 4, 0]
    assert t_dst.tolist() == [1, 2, 0, 2, 0]


def test_paths_selection_rule_counts():
    from oracle import irreps
    bi = irreps.parse("64x0e+64x1o+64x2e")
    ps = irreps.paths(bi, 3, bi, "uvw")
    assert [(p.l_in, p.l_sh, p.l_out) for p in ps] == [
        (0, 0, 0), (0, 1, 1), (0, 2, 2), (1, 0, 1), (1, 1, 0), (1, 1, 2), (1, 2, 1),
        (1, 3, 2), (2, 0, 2), (2, 1, 1), (2, 2, 0), (2, 2, 2), (2, 3, 1)]
    assert irreps.num_weights(ps) == 13 * 64 * 64
    b4 = irreps.parse("128x0e+64x1o+32x2e+16x3o")
    assert len(irreps.paths(b4, 3, b4, "uvw")) == 23
    with pytest.raises(ValueError):
        irreps.paths(irreps.parse("4x0e"), 1, irreps.parse("2x1o"), "uvu")
    with pytest.raises(ValueError):
        irreps.parse("4x0q")
