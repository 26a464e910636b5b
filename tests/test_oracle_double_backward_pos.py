"""Pins for the position gradient of the double backward (oracle/conv.py
double_backward_pos) and for the second derivatives it is built on.

Second derivatives of the edge functions:
* the l = 1 harmonics are sqrt(3) (y, z, x) / |r|, whose Hessian is a closed form;
* every harmonic is homogeneous of degree 0 in r, so (Euler) H_Y r = -dY/dr;
* a radial function f(|r|) has Hessian f'' r_hat r_hat^T + (f'/|r|)(I - r_hat r_hat^T),
  with f' and f'' taken by finite differences of the one-dimensional basis;
* every Hessian is symmetric, and matches central differences of the gradient.
The position gradient of the double backward:
* central differences of Lambda(pos) = <gg_x, x_bar> + <gg_pos, pos_bar> + <gg_A, A_bar>
  taken through the oracle's first backward;
* translation invariance (the gradient sums to zero over nodes);
* symmetry of the position Hessian (<p2, H p1> = <p1, H p2>);
* mixed partials against the double backward's own grad_x and grad_A
  (<p, d2L/dpos dx  x_dot> = <x_dot, d2L/dx dpos  p>, likewise for A);
* a zero-length edge contributes exactly zero.
"""

import numpy as np
import pytest

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, radial, so3

BESSEL = radial.RadialSpec(radial.BESSEL, 6, 2.5)
GAUSS = radial.RadialSpec(radial.GAUSSIAN, 5, 3.0, 0.0, 3.0)

CASES = {
    "uvw": ("3x0e+2x1o+2x2e", 3, "2x0e+3x1o+2x2e+1x3o", "uvw", BESSEL),
    "uvw_odd": ("2x0e+2x1o+1x1e", 2, "2x0e+1x1e+2x1o+1x2e+1x2o", "uvw", BESSEL),
    "uvu": ("3x0e+3x1o+3x2e", 2, "3x0e+3x1o+3x2e", "uvu", GAUSS),
}


def _problem(case, n=7, k=3, seed=3):
    ii, lmax, io, mode, rs = CASES[case]
    plan = conv.make_plan(ii, lmax, io, mode, rs)
    rng = np.random.default_rng(seed)
    pos = rng.uniform(0, 2.5, size=(n, 3))
    row_ptr, src = workloads.knn_csr(pos, np.full(n, k))
    x = rng.normal(size=(n, plan.dim_in))
    A = rng.normal(size=(rs.num_basis, plan.n_w)) / 3
    mbar = rng.normal(size=(n, plan.dim_out))
    return plan, x, pos, row_ptr, src, A, mbar, rng


# ---------------------------------------------------------------------------
# second derivatives of Y and phi
# ---------------------------------------------------------------------------

def test_sh_hessian_l1_closed_form(rng):
    r = rng.normal(size=(40, 3)) * 1.7
    _, _, H = so3.sh_with_hessian(1, r)
    d = np.linalg.norm(r, axis=1)
    I = np.eye(3)
    # d2 (r_a / |r|) / dr_b dr_c
    want = np.empty((r.shape[0], 3, 3, 3))
    for a in range(3):
        for b in range(3):
            for c in range(3):
                want[:, a, b, c] = (-(I[a, b] * r[:, c] + I[a, c] * r[:, b] + I[b, c] * r[:, a]) / d ** 3
                                    + 3 * r[:, a] * r[:, b] * r[:, c] / d ** 5)
    want = np.sqrt(3) * want[:, [1, 2, 0]]          # Y_1 = sqrt(3) (y, z, x)
    assert np.abs(H[:, 1:4] - want).max() <= 1e-12 * np.abs(want).max()
    assert np.all(H[:, 0] == 0.0)


def test_sh_hessian_euler_symmetry_and_fd(rng):
    r = rng.normal(size=(30, 3)) * 2.0
    Y, g, H = so3.sh_with_hessian(3, r)
    scale = np.abs(H).max()
    assert np.abs(H - np.swapaxes(H, 2, 3)).max() <= 1e-12 * scale
    # degree-0 homogeneity: g . r = 0, hence H r + g = 0
    assert np.abs(np.einsum("eskl,el->esk", H, r) + g).max() <= 1e-11 * np.abs(g).max()
    h = 1e-5
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        fd = (so3.sh_with_grad(3, r + e)[1] - so3.sh_with_grad(3, r - e)[1]) / (2 * h)
        assert np.abs(fd - H[..., k]).max() <= 1e-7 * scale


@pytest.mark.parametrize("spec", [BESSEL, GAUSS, radial.RadialSpec(radial.BESSEL, 8, 5.0)])
def test_radial_hessian_closed_form(spec, rng):
    r = rng.normal(size=(30, 3))
    r *= (rng.uniform(0.2, 0.97, size=30) * spec.r_cut / np.linalg.norm(r, axis=1))[:, None]
    _, _, H = radial.basis_with_hessian(spec, r)
    d = np.linalg.norm(r, axis=1)
    u = r / d[:, None]
    # f'(d), f''(d) by central differences of the basis along the radius
    h = 1e-4
    f = lambda dd: radial.basis_of_vectors(spec, u * dd[:, None])[0]  # noqa: E731
    f1 = (f(d + h) - f(d - h)) / (2 * h)
    f2 = (f(d + h) - 2 * f(d) + f(d - h)) / h ** 2
    uu = u[:, :, None] * u[:, None, :]
    want = (f2[:, :, None, None] * uu[:, None] + (f1 / d[:, None])[:, :, None, None] * (np.eye(3) - uu)[:, None])
    assert np.abs(H - want).max() <= 1e-5 * np.abs(want).max()
    assert np.abs(H - np.swapaxes(H, 2, 3)).max() <= 1e-12 * np.abs(H).max()


def test_radial_hessian_vanishes_at_and_beyond_cutoff(rng):
    """u, u' and u'' vanish at t = 1, so the Hessian is continuous through the cutoff."""
    spec = BESSEL
    dirs = rng.normal(size=(8, 3))
    dirs /= np.linalg.norm(dirs, axis=1)[:, None]
    _, _, H_in = radial.basis_with_hessian(spec, dirs * spec.r_cut * (1 - 1e-7))
    _, _, H_out = radial.basis_with_hessian(spec, dirs * spec.r_cut * 1.3)
    _, _, H_mid = radial.basis_with_hessian(spec, dirs * spec.r_cut * 0.5)
    assert np.all(H_out == 0.0)
    assert np.abs(H_in).max() <= 1e-8 * np.abs(H_mid).max()


# ---------------------------------------------------------------------------
# dLambda/dpos
# ---------------------------------------------------------------------------

def _lam(plan, x, pos, row_ptr, src, A, mbar, ggx, ggp, ggA):
    gx, gpos, gA = conv.backward(plan, x, pos, row_ptr, src, A, mbar)
    tot = 0.0
    if ggx is not None:
        tot += np.sum(ggx * gx)
    if ggp is not None:
        tot += np.sum(ggp * gpos)
    if ggA is not None:
        tot += np.sum(ggA * gA)
    return float(tot)


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("which", ["x", "pos", "A", "all"])
def test_double_backward_pos_matches_finite_differences(case, which):
    plan, x, pos, row_ptr, src, A, mbar, rng = _problem(case)
    ggx = rng.normal(size=x.shape) if which in ("x", "all") else None
    ggp = rng.normal(size=pos.shape) if which in ("pos", "all") else None
    ggA = rng.normal(size=A.shape) if which in ("A", "all") else None
    got = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, ggx, ggp, ggA)
    h = 1e-5
    fd = np.zeros_like(pos)
    for i in range(pos.shape[0]):
        for k in range(3):
            pp, pm = pos.copy(), pos.copy()
            pp[i, k] += h
            pm[i, k] -= h
            fd[i, k] = (_lam(plan, x, pp, row_ptr, src, A, mbar, ggx, ggp, ggA)
                        - _lam(plan, x, pm, row_ptr, src, A, mbar, ggx, ggp, ggA)) / (2 * h)
    scale = np.abs(fd).max()
    assert scale > 1e-6
    assert np.abs(got - fd).max() <= 1e-6 * scale


@pytest.mark.parametrize("case", list(CASES))
def test_double_backward_pos_translation_invariant(case):
    plan, x, pos, row_ptr, src, A, mbar, rng = _problem(case, n=9, k=4)
    got = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, rng.normal(size=x.shape),
                                   rng.normal(size=pos.shape), rng.normal(size=A.shape))
    assert np.abs(got.sum(0)).max() <= 1e-11 * np.abs(got).max()


@pytest.mark.parametrize("case", list(CASES))
def test_position_hessian_is_symmetric(case):
    plan, x, pos, row_ptr, src, A, mbar, rng = _problem(case, n=9, k=4)
    p1, p2 = rng.normal(size=pos.shape), rng.normal(size=pos.shape)
    h1 = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, gg_pos=p1)
    h2 = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, gg_pos=p2)
    a, b = np.sum(p2 * h1), np.sum(p1 * h2)
    assert abs(a - b) <= 1e-11 * max(abs(a), 1.0)


@pytest.mark.parametrize("case", list(CASES))
def test_mixed_partials_match_double_backward(case):
    plan, x, pos, row_ptr, src, A, mbar, rng = _problem(case, n=9, k=4)
    p, xd, Ad = rng.normal(size=pos.shape), rng.normal(size=x.shape), rng.normal(size=A.shape)
    gx, gA, _ = conv.double_backward(plan, x, pos, row_ptr, src, A, mbar, gg_pos=p)
    hx = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, gg_x=xd)
    hA = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, gg_A=Ad)
    a, b = np.sum(p * hx), np.sum(xd * gx)
    assert abs(a - b) <= 1e-11 * max(abs(a), 1.0)
    a, b = np.sum(p * hA), np.sum(Ad * gA)
    assert abs(a - b) <= 1e-11 * max(abs(a), 1.0)


def test_double_backward_pos_null_tangents_and_zero_length_edge():
    plan, x, pos, row_ptr, src, A, mbar, rng = _problem("uvw")
    assert np.all(conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar) == 0.0)
    # node 1 moved onto node 0, with an edge 1 -> 0 (first edge of receiver 0)
    pos = pos.copy()
    row_ptr = np.array([0, 1] + [1] * (pos.shape[0] - 1))
    src = np.array([1])
    pos[1] = pos[0]
    got = conv.double_backward_pos(plan, x, pos, row_ptr, src, A, mbar, rng.normal(size=x.shape),
                                   rng.normal(size=pos.shape), rng.normal(size=A.shape))
    assert np.all(got == 0.0)
