"""Embedded-input interface (tpconv_forward_embedded / tpconv_backward_embedded): the
edge embedding phi_e and the harmonics Y_e are given per edge, the backward returns the
edge-owned adjoints phi_bar (eq. 20) and Y_bar (eq. 22).  Checked against the oracle's
embedded variants on arbitrary per-edge inputs, and against the position-based path
when the inputs are the harmonics and radial basis of the edge vectors."""

import numpy as np
import pytest

from helpers import Problem, cuda, lib_plan, rel_l2
from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, radial, so3

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("cfg,n", [(2, 160), (4, 200), (5, 160), (3, 96)])
def test_embedded_parity_arbitrary_inputs(torch, cfg, n):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=n)
    lp = lib_plan(p.cfg)
    rng = np.random.default_rng(99 + cfg)
    Y = workloads.normal(rng, (p.E, p.plan.n_sh))
    phi = workloads.normal(rng, (p.E, p.cfg.num_basis))
    x, rp, src, W, go = (cuda(a) for a in (p.x, p.row_ptr, p.src, p.W, p.gout))
    dY, dphi = cuda(Y), cuda(phi)
    out = binding.tpconv_forward_embedded(lp, x, dY, dphi, rp, src, W)
    ref = conv.forward_embedded(p.plan, p.x, Y, phi, p.row_ptr, p.N, p.src, p.W)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL
    v = binding.tpconv_csr_transpose(rp, src, p.N)
    gx, gw, gphi, gY = binding.tpconv_backward_embedded(lp, x, dY, dphi, rp, src, *v, W, go)
    rx, rw, rphi, rY = conv.backward_embedded(p.plan, p.x, Y, phi, p.row_ptr, p.N, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gw, rw), (gphi, rphi), (gY, rY)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL
    # partial outputs
    gx2, gw2, gphi2, gY2 = binding.tpconv_backward_embedded(lp, x, dY, dphi, rp, src, *v, W, go, need_x=False,
                                                            need_W=False, need_Y=False)
    assert gx2 is None and gw2 is None and gY2 is None
    assert torch.equal(gphi2, gphi)


def test_embedded_with_geometry_matches_position_path(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(2, n_nodes=160)
    lp = lib_plan(p.cfg)
    dst = conv.receivers_of(p.row_ptr)
    r = p.pos[p.src].astype(np.float64) - p.pos[dst].astype(np.float64)
    rs = radial.RadialSpec(p.cfg.radial, p.cfg.num_basis, p.cfg.r_cut, p.cfg.r_min, p.cfg.r_max)
    Y = so3.sh(p.plan.lmax, r).astype(np.float32)
    phi = radial.basis_of_vectors(rs, r)[0].astype(np.float32)
    x, pos, rp, src, W, go = (cuda(a) for a in (p.x, p.pos, p.row_ptr, p.src, p.W, p.gout))
    a = binding.tpconv_forward_embedded(lp, x, cuda(Y), cuda(phi), rp, src, W)
    b = binding.tpconv_forward(lp, x, pos, rp, src, W)
    assert rel_l2(a.cpu().numpy(), b.cpu().numpy()) <= TOL
    v = binding.tpconv_csr_transpose(rp, src, p.N)
    gx, gw, _, _ = binding.tpconv_backward_embedded(lp, x, cuda(Y), cuda(phi), rp, src, *v, W, go)
    hx, _, hw = binding.tpconv_backward(lp, x, pos, rp, src, *v, W, go)
    assert rel_l2(gx.cpu().numpy(), hx.cpu().numpy()) <= TOL
    assert rel_l2(gw.cpu().numpy(), hw.cpu().numpy()) <= TOL
