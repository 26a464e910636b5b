"""Feature-profile grids (sixteen uvw and nine uvu profiles, see workloads.profile_configs):
forward, backward and double backward of every profile against the float64 oracle on a
small graph of the same construction (kNN, density 0.1).  The tolerance is the
library-wide 1e-4 relative L2."""

import numpy as np
import pytest

from helpers import Problem, cuda, lib_plan, rel_l2
from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv

pytestmark = pytest.mark.gpu

TOL = 1e-4
PROFILES = workloads.profile_configs()


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("c", PROFILES, ids=[f"p{c.cfg}" for c in PROFILES])
def test_profile_forward_backward_double_backward(torch, c):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(None, config=c, n_nodes=40, k=8, seed=7000 + c.cfg)
    lp = lib_plan(c)
    x, pos, rp, src, W, go = (cuda(a) for a in (p.x, p.pos, p.row_ptr, p.src, p.W, p.gout))
    out = binding.tpconv_forward(lp, x, pos, rp, src, W)
    assert rel_l2(out.cpu().numpy(), conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)) <= TOL
    v = binding.tpconv_csr_transpose(rp, src, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, x, pos, rp, src, *v, W, go)
    rx, rpos, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gp, rpos), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL
    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    dx, dw, dg = binding.tpconv_double_backward(lp, x, pos, rp, src, *v, W, go, gg_x=cuda(ggx), gg_pos=cuda(ggp),
                                                gg_W=cuda(ggw))
    ex, ew, eg = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, ggx, ggp, ggw)
    for a, b in ((dx, ex), (dw, ew), (dg, eg)):
        assert np.all(np.isfinite(a.cpu().numpy()))
        assert rel_l2(a.cpu().numpy(), b) <= TOL
