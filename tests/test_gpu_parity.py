"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Every comparison uses the same seeded float32 inputs on both sides.  The bar is the
relative L2 error per output tensor, ||gpu - oracle|| / ||oracle|| <= 1e-4 (fp32
arithmetic against float64; the accumulation order differs, so results agree to
rounding only).  Graph views are compared bit for bit.

Sizes: reduced node counts of every workload (several GEMM tiles with a ragged tail,
receivers with more than 32 edges), the tiny workload at full size, and the full-size
uvw forward+backward workload checked on sampled receivers (the upstream gradient is
nonzero only on the sample, so the oracle sums exactly the edges that contribute).
"""

import numpy as np
import pytest

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, graph

from helpers import Problem, cuda, lib_plan, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-4
REDUCED = {1: None, 2: 160, 3: 120, 4: 200, 5: 160}


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _dev(p):
    import torch
    return dict(x=cuda(p.x), pos=cuda(p.pos), row_ptr=cuda(p.row_ptr), src=cuda(p.src), W=cuda(p.W),
                gout=cuda(p.gout))


def _graph_views(d, N):
    from equivariant_gnn_tensor_dst_b200 import binding
    return binding.tpconv_csr_transpose(d["row_ptr"], d["src"], N)


# ---------------------------------------------------------------------------
# graph utilities
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cfg,n", [(1, None), (2, 300), (4, 400)])
def test_csr_transpose_bit_exact(torch, cfg, n):
    p = Problem(cfg, n_nodes=n)
    d = _dev(p)
    t_ptr, t_eid, t_dst = _graph_views(d, p.N)
    r_ptr, r_eid, r_dst = graph.source_view(p.row_ptr, p.src, p.N)
    assert np.array_equal(t_ptr.cpu().numpy(), r_ptr)
    assert np.array_equal(t_eid.cpu().numpy(), r_eid)
    assert np.array_equal(t_dst.cpu().numpy(), r_dst)


def test_csr_transpose_isolated_nodes_and_empty(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    row_ptr = np.array([0, 0, 3, 3, 5, 5], np.int32)
    src = np.array([4, 0, 4, 1, 4], np.int32)
    t_ptr, t_eid, t_dst = binding.tpconv_csr_transpose(cuda(row_ptr), cuda(src), 5)
    r = graph.source_view(row_ptr, src, 5)
    assert np.array_equal(t_ptr.cpu().numpy(), r[0])
    assert np.array_equal(t_eid.cpu().numpy(), r[1])
    assert np.array_equal(t_dst.cpu().numpy(), r[2])
    empty = np.zeros(4, np.int32)
    t_ptr, t_eid, _ = binding.tpconv_csr_transpose(cuda(empty), cuda(np.zeros(1, np.int32))[:0], 3)
    assert np.array_equal(t_ptr.cpu().numpy(), [0, 0, 0, 0])


def test_validate_graph_codes(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(1)
    d = _dev(p)
    assert int(binding.tpconv_validate_graph(d["row_ptr"], d["src"], p.N).item()) == 0
    bad = p.src.copy()
    bad[7] = p.N + 3
    assert int(binding.tpconv_validate_graph(d["row_ptr"], cuda(bad), p.N).item()) == 3
    rp = p.row_ptr.copy()
    rp[10], rp[11] = rp[11], rp[10]
    assert int(binding.tpconv_validate_graph(cuda(rp), d["src"], p.N).item()) == 2


# ---------------------------------------------------------------------------
# forward / backward / double backward at reduced sizes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_forward_parity(torch, cfg):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=REDUCED[cfg])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    ref = conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_backward_parity(torch, cfg):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=REDUCED[cfg])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    t_ptr, t_eid, t_dst = _graph_views(d, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], t_ptr, t_eid, t_dst,
                                         d["W"], d["gout"])
    rx, rp, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    assert rel_l2(gx.cpu().numpy(), rx) <= TOL
    assert rel_l2(gp.cpu().numpy(), rp) <= TOL
    assert rel_l2(gw.cpu().numpy(), rw) <= TOL


@pytest.mark.parametrize("cfg", [2, 3])
def test_backward_partial_outputs(torch, cfg):
    """Requesting a subset of the gradients gives the same values."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=REDUCED[cfg])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    full = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    only_pos = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"],
                                       need_x=False, need_W=False)
    only_w = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"],
                                     need_x=False, need_pos=False)
    assert only_pos[0] is None and only_pos[2] is None
    assert torch.equal(only_pos[1], full[1])
    assert torch.equal(only_w[2], full[2])


@pytest.mark.parametrize("cfg", [5, 3])
def test_double_backward_parity(torch, cfg):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=96 if cfg == 3 else REDUCED[cfg])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    for tx, tp, tw in ((ggx, ggp, ggw), (None, ggp, None), (ggx, None, None), (None, None, ggw)):
        gx, gw, gg = binding.tpconv_double_backward(
            lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"],
            gg_x=None if tx is None else cuda(tx), gg_pos=None if tp is None else cuda(tp),
            gg_W=None if tw is None else cuda(tw))
        rx, rw, rg = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, tx, tp, tw)
        assert rel_l2(gx.cpu().numpy(), rx) <= TOL
        assert rel_l2(gw.cpu().numpy(), rw) <= TOL
        assert rel_l2(gg.cpu().numpy(), rg) <= TOL


@pytest.mark.parametrize("cfg", [2, 5])
@pytest.mark.parametrize("mode", ["tf32", "bf16"])
def test_reduced_precision_math_modes(torch, cfg, mode):
    """TF32 contractions (one tensor-core product per term) and BF16 contractions (both
    operands rounded to bf16, one kind::f16 product): every pass within the 1e-2 relative
    bar for reduced-precision modes, and measurably away from the fp32 result (the mode
    is in effect); the default mode stays within 1e-4."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=REDUCED[cfg])
    lp = lib_plan(p.cfg)
    lp.set_math(binding.MATH_TF32 if mode == "tf32" else binding.MATH_BF16)
    d = _dev(p)
    v = _graph_views(d, p.N)
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    ref = conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)
    err = rel_l2(out.cpu().numpy(), ref)
    assert 1e-5 < err <= 1e-2
    gx, gp, gw = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    rx, rp, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gp, rp), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= 1e-2
    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    dx, dw, dg = binding.tpconv_double_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                                d["gout"], gg_x=cuda(ggx), gg_pos=cuda(ggp), gg_W=cuda(ggw))
    ex, ew, eg = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, ggx, ggp, ggw)
    for a, b in ((dx, ex), (dw, ew), (dg, eg)):
        assert rel_l2(a.cpu().numpy(), b) <= 1e-2
    lp.set_math(binding.MATH_FP32)
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    assert rel_l2(out.cpu().numpy(), conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)) <= TOL


def test_force_training_step(torch):
    """Energy = sum of scalar outputs, forces F = -dE/dpos, loss |F - F_ref|^2, then the
    gradient of the loss w.r.t. W and x through the double backward."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(5, n_nodes=REDUCED[5])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    mbar = np.tile(p.scalar_mask(), (p.N, 1))
    F_ref = workloads.normal(p.rng, (p.N, 3))
    _, gpos, _ = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                         cuda(mbar), need_x=False, need_W=False)
    F = -gpos.cpu().numpy()
    _, rpos, _ = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, mbar)
    assert rel_l2(F, -rpos) <= TOL
    gg_pos = (-2.0 * (F - F_ref)).astype(np.float32)
    gx, gw, _ = binding.tpconv_double_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                               cuda(mbar), gg_pos=cuda(gg_pos), need_grad_out=False)
    rx, rw, _ = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, mbar, None, gg_pos, None)
    assert rel_l2(gx.cpu().numpy(), rx) <= TOL
    assert rel_l2(gw.cpu().numpy(), rw) <= TOL


def test_general_parities_forward_backward(torch):
    """Odd-sum paths (1o x 1o -> 1e and friends) and l = 3 blocks."""
    from equivariant_gnn_tensor_dst_b200 import binding
    c = workloads.Config(9, "mixed parities", 90, 12, "40x0e+33x1o+8x1e+5x3o", 3,
                         "16x0e+8x1e+24x1o+8x2e+4x2o+4x3e+4x3o", "uvw", "bessel", 6, 4.0)
    p = Problem(None, config=c)
    lp = lib_plan(c)
    d = _dev(p)
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    assert rel_l2(out.cpu().numpy(), conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)) <= TOL
    v = _graph_views(d, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    rx, rp, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gp, rp), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL


def test_many_paths_overflow_one_gemm_batch(torch):
    """34 paths whose weight-gradient contractions need more segments (one per m
    component, 134 in all) than one grouped launch holds: the library splits them over
    several launches."""
    from equivariant_gnn_tensor_dst_b200 import binding
    irr = "8x0e+8x1o+8x2e+8x3o+8x0o+8x1e"
    c = workloads.Config(9, "many paths", 60, 10, irr, 3, irr, "uvw", "bessel", 8, 4.0)
    p = Problem(None, config=c)
    lp = lib_plan(c)
    assert len(lp.paths()) == 34
    assert sum(2 * q["l_out"] + 1 for q in lp.paths()) > 128
    d = _dev(p)
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    assert rel_l2(out.cpu().numpy(), conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)) <= TOL
    v = _graph_views(d, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    rx, rp, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gp, rp), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def test_no_edges_and_isolated_receivers(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(2, n_nodes=40)
    lp = lib_plan(p.cfg)
    # drop every edge of receivers 5..19: isolated receivers get zero output
    keep = np.ones(p.E, bool)
    for i in range(5, 20):
        keep[p.row_ptr[i]:p.row_ptr[i + 1]] = False
    deg = np.diff(p.row_ptr).copy()
    deg[5:20] = 0
    row_ptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    src = p.src[keep]
    out = binding.tpconv_forward(lp, cuda(p.x), cuda(p.pos), cuda(row_ptr), cuda(src), cuda(p.W))
    ref = conv.forward(p.plan, p.x, p.pos, row_ptr, src, p.W)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL
    assert np.all(out.cpu().numpy()[5:20] == 0)
    # no edges at all
    row0 = np.zeros(p.N + 1, np.int32)
    src0 = cuda(np.zeros(1, np.int32))[:0]
    out = binding.tpconv_forward(lp, cuda(p.x), cuda(p.pos), cuda(row0), src0, cuda(p.W))
    assert np.all(out.cpu().numpy() == 0)
    v = binding.tpconv_csr_transpose(cuda(row0), src0, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, cuda(p.x), cuda(p.pos), cuda(row0), src0, *v, cuda(p.W),
                                         cuda(p.gout))
    assert np.all(gx.cpu().numpy() == 0) and np.all(gp.cpu().numpy() == 0) and np.all(gw.cpu().numpy() == 0)


def test_edges_beyond_cutoff_and_coincident_nodes(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(5, n_nodes=64)
    pos = p.pos.copy()
    pos[3] = pos[p.src[p.row_ptr[3]]]          # a zero-length edge
    pos[10] += 50.0                            # every edge of node 10 beyond the cutoff
    lp = lib_plan(p.cfg)
    out = binding.tpconv_forward(lp, cuda(p.x), cuda(pos), cuda(p.row_ptr), cuda(p.src), cuda(p.W))
    ref = conv.forward(p.plan, p.x, pos, p.row_ptr, p.src, p.W)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL
    assert np.all(out.cpu().numpy()[10] == 0)
    v = binding.tpconv_csr_transpose(cuda(p.row_ptr), cuda(p.src), p.N)
    gx, gp, gw = binding.tpconv_backward(lp, cuda(p.x), cuda(pos), cuda(p.row_ptr), cuda(p.src), *v,
                                         cuda(p.W), cuda(p.gout))
    rx, rp, rw = conv.backward(p.plan, p.x, pos, p.row_ptr, p.src, p.W, p.gout)
    for a, b in ((gx, rx), (gp, rp), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL


def test_small_budget_chunks_receivers(torch):
    """A scratch budget of a few receivers forces many receiver ranges; results agree."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(2, n_nodes=REDUCED[2])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    a = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    ga = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    lp.set_workspace_budget(7 * 22016 * 4)
    b = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])
    gb = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"])
    assert torch.equal(a, b)
    for u, w in zip(ga, gb):
        assert rel_l2(w.cpu().numpy(), u.cpu().numpy()) <= 1e-6


def test_deterministic(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(4, n_nodes=REDUCED[4])
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    r1 = [binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])]
    r1 += list(binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"]))
    r2 = [binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"])]
    r2 += list(binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"]))
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# full-size workloads, sampled
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cfg", [2, 5, 3, 4])
def test_full_size_sampled(torch, cfg):
    """Full-size launch.  Forward on 64 sampled receivers plus the four of highest in-degree;
    every backward output for an upstream gradient that is nonzero on 12 sampled receivers
    plus those four (the edge-scaling workload's heaviest receivers have over 400 in-edges,
    16 chunks of 32, and its receivers run in many ranges of the scratch budget)."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg)
    lp = lib_plan(p.cfg)
    d = _dev(p)
    v = _graph_views(d, p.N)
    deg = np.diff(p.row_ptr)
    top = np.argsort(deg, kind="stable")[-4:]
    if cfg == 4:
        assert deg[top].min() >= 400
    rows = np.unique(np.concatenate([p.rng.choice(p.N, size=64, replace=False), top]))
    out = binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"]).cpu().numpy()
    ref = conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, edges=p.edges_of(rows))
    assert rel_l2(out[rows], ref[rows]) <= TOL
    for r in top:   # each heavy receiver on its own, not only inside the sample's norm
        assert rel_l2(out[r], ref[r]) <= TOL
    sample = np.unique(np.concatenate([p.rng.choice(p.N, size=12, replace=False), top]))
    edges = p.edges_of(sample)
    mbar = np.zeros_like(p.gout)
    mbar[sample] = p.gout[sample]
    gx, gp, gw = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], cuda(mbar))
    rx, rp, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, mbar, edges=edges)
    for a, b in ((gx, rx), (gp, rp), (gw, rw)):
        assert rel_l2(a.cpu().numpy(), b) <= TOL
    if cfg == 5:
        ggp = workloads.normal(p.rng, p.pos.shape)
        gx2, gw2, gg2 = binding.tpconv_double_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                                       cuda(mbar), gg_pos=cuda(ggp))
        rx2, rw2, rg2 = conv.double_backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, mbar, None, ggp, None,
                                             edges=edges)
        assert rel_l2(gx2.cpu().numpy(), rx2) <= TOL
        assert rel_l2(gw2.cpu().numpy(), rw2) <= TOL
        assert rel_l2(gg2.cpu().numpy()[sample], rg2[sample]) <= TOL


def test_no_device_error_after_runs(torch):
    """Bounded waits inside the tensor-core kernels never gave up during this session."""
    from equivariant_gnn_tensor_dst_b200 import binding
    assert binding.tpconv_device_error() == 0
