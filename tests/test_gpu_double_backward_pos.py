"""GPU parity of the double backward's position gradient, dLambda/dpos, against the
float64 oracle (oracle.conv.double_backward_pos), relative L2 <= 1e-4.

Cases: uvw with the Bessel basis (K = 8) and uvu with the Gaussian basis (K = 16) at
reduced sizes, every combination of tangents; a uvw plan with mixed parities, l = 3 and
K = 16; the force-training step (energy = sum of scalar outputs, loss on the forces),
whose position gradient is what learning positions needs; the full-size force-training
workload on sampled nodes (the oracle sums the edges incident to the sample, which are
all that reach those rows); and the degenerate inputs (no tangents, no edges,
coincident nodes).
"""

import numpy as np
import pytest

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv

from helpers import Problem, cuda, lib_plan, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _dev(p):
    return dict(x=cuda(p.x), pos=cuda(p.pos), row_ptr=cuda(p.row_ptr), src=cuda(p.src), W=cuda(p.W),
                gout=cuda(p.gout))


def _views(d, N):
    from equivariant_gnn_tensor_dst_b200 import binding
    return binding.tpconv_csr_transpose(d["row_ptr"], d["src"], N)


def _run(p, lp, d, v, gout, tx, tp, tw, **kw):
    from equivariant_gnn_tensor_dst_b200 import binding
    return binding.tpconv_double_backward(
        lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], gout,
        gg_x=None if tx is None else cuda(tx), gg_pos=None if tp is None else cuda(tp),
        gg_W=None if tw is None else cuda(tw), need_pos=True, **kw)


MIXED = workloads.Config(9, "mixed parities, l = 3, K = 16", 90, 12, "24x0e+17x1o+8x1e+5x3o", 3,
                         "16x0e+8x1e+24x1o+8x2e+4x2o+4x3e+4x3o", "uvw", "gaussian", 16, 4.0, 0.0, 4.0)


@pytest.mark.parametrize("which", [5, 3, "mixed"])
def test_double_backward_pos_parity(torch, which):
    p = Problem(None, config=MIXED) if which == "mixed" else Problem(which, n_nodes=96 if which == 3 else 160)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _views(d, p.N)
    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    for tx, tp, tw in ((ggx, ggp, ggw), (None, ggp, None), (ggx, None, None), (None, None, ggw)):
        gx, gw, gg, gp = _run(p, lp, d, v, d["gout"], tx, tp, tw)
        ref = conv.double_backward_pos(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, tx, tp, tw)
        assert rel_l2(gp.cpu().numpy(), ref) <= TOL, (tx is None, tp is None, tw is None)
        # the other outputs of the same call are unchanged by asking for grad_pos
        rx, rw, rg = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, tx, tp, tw)
        assert rel_l2(gx.cpu().numpy(), rx) <= TOL
        assert rel_l2(gw.cpu().numpy(), rw) <= TOL
        assert rel_l2(gg.cpu().numpy(), rg) <= TOL


def test_double_backward_pos_only_and_translation_invariance(torch):
    p = Problem(2, n_nodes=160)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _views(d, p.N)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    _, _, _, gp = _run(p, lp, d, v, d["gout"], None, ggp, ggw, need_x=False, need_W=False, need_grad_out=False)
    ref = conv.double_backward_pos(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, None, ggp, ggw)
    got = gp.cpu().numpy().astype(np.float64)
    assert rel_l2(got, ref) <= TOL
    assert np.abs(got.sum(0)).max() <= 1e-4 * np.abs(got).max() * np.sqrt(p.E)


def test_force_training_position_gradient(torch):
    """E = sum of scalar outputs, F = -dE/dpos, loss |F - F_ref|^2: the loss gradient
    with respect to the positions is dLambda/dpos with gg_pos = -2 (F - F_ref)."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(5, n_nodes=160)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _views(d, p.N)
    mbar = np.tile(p.scalar_mask(), (p.N, 1))
    F_ref = workloads.normal(p.rng, (p.N, 3))
    _, gpos, _ = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                         cuda(mbar), need_x=False, need_W=False)
    gg_pos = (-2.0 * (-gpos.cpu().numpy() - F_ref)).astype(np.float32)
    _, _, _, gp = _run(p, lp, d, v, cuda(mbar), None, gg_pos, None, need_x=False, need_grad_out=False)
    ref = conv.double_backward_pos(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, mbar, None, gg_pos, None)
    assert rel_l2(gp.cpu().numpy(), ref) <= TOL


def test_force_training_full_size_sampled(torch):
    """Full-size force-training workload (N = 8192, k = 32): rows of 24 sampled nodes."""
    p = Problem(5)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _views(d, p.N)
    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    _, _, _, gp = _run(p, lp, d, v, d["gout"], ggx, ggp, ggw, need_x=False, need_W=False, need_grad_out=False)
    got = gp.cpu().numpy()
    sample = np.sort(p.rng.choice(p.N, size=24, replace=False))
    dst = conv.receivers_of(p.row_ptr)
    inc = np.nonzero(np.isin(dst, sample) | np.isin(p.src, sample))[0]
    ref = conv.double_backward_pos(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, ggx, ggp, ggw,
                                   edges=inc)
    assert rel_l2(got[sample], ref[sample]) <= TOL


def test_double_backward_pos_degenerate(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(5, n_nodes=40)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _views(d, p.N)
    # no tangents: zero
    _, _, _, gp = _run(p, lp, d, v, d["gout"], None, None, None)
    assert torch.count_nonzero(gp).item() == 0
    # no edges: zero
    row_ptr = np.zeros(p.N + 1, np.int32)
    src = np.zeros(0, np.int32)
    de = dict(d, row_ptr=cuda(row_ptr), src=cuda(src))
    ve = binding.tpconv_csr_transpose(de["row_ptr"], de["src"], p.N)
    ggp = workloads.normal(p.rng, p.pos.shape)
    _, _, _, gp = _run(p, lp, de, ve, d["gout"], None, ggp, None)
    assert torch.count_nonzero(gp).item() == 0
    # node 1 moved onto node 0: the zero-length edge between them contributes nothing
    pos = p.pos.copy()
    pos[1] = pos[0]
    row_ptr = np.array([0, 1] + [1] * (p.N - 1), np.int32)
    src = np.array([1], np.int32)
    dz = dict(d, pos=cuda(pos), row_ptr=cuda(row_ptr), src=cuda(src))
    vz = binding.tpconv_csr_transpose(dz["row_ptr"], dz["src"], p.N)
    ggx = workloads.normal(p.rng, p.x.shape)
    _, _, _, gp = _run(p, lp, dz, vz, d["gout"], ggx, ggp, None)
    assert torch.count_nonzero(gp).item() == 0
