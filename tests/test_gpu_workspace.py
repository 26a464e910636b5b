"""Workspace law and position-gradient staging windows on the GPU.

* Degree sweep (kNN k = 8, 16, 32, 64, 128 at N = 4096, the uvw workload's irreps): the
  peak device allocation of forward, backward and double backward (dLambda/dpos
  included), measured as torch's max_memory_allocated delta with every input and output
  allocated beforehand, is the same for every degree, and equals the declared workspace
  (rounded up to the allocator's 2 MiB block).
  The edge count grows 16x over the sweep; the scratch does not.
* Staging windows smaller than one receiver's in-degree (a tiny scratch budget): the
  position gradients of backward and double backward, staged window by window and summed
  in a fixed order, agree with the default budget's and with the float64 oracle.
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


def test_degree_sweep_peak_workspace_constant(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    lp = lib_plan(workloads.CONFIGS[2])
    dev = torch.device("cuda")
    rows = []
    for k in (8, 16, 32, 64, 128):
        p = Problem(2, k=k)
        d = {n: cuda(a) for n, a in (("x", p.x), ("pos", p.pos), ("row_ptr", p.row_ptr), ("src", p.src),
                                     ("W", p.W), ("gout", p.gout))}
        views = binding.tpconv_csr_transpose(d["row_ptr"], d["src"], p.N)
        tan = [cuda(workloads.normal(p.rng, s)) for s in (p.x.shape, p.pos.shape, p.W.shape)]
        outs = [torch.empty(s, device=dev) for s in ((p.N, lp.dim_out), (p.N, lp.dim_in), (p.N, 3),
                                                     tuple(p.W.shape), (p.N, lp.dim_in), tuple(p.W.shape),
                                                     (p.N, lp.dim_out), (p.N, 3))]
        wsb = lp.workspace_bytes(p.N, p.E)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        mem0 = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        ws = binding.workspace(wsb, dev)
        binding.tpconv_forward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], d["W"], out=outs[0], ws=ws)
        binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *views, d["W"], d["gout"], ws=ws,
                                outputs=(outs[1], outs[2], outs[3]))
        binding.tpconv_double_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *views, d["W"], d["gout"],
                                       gg_x=tan[0], gg_pos=tan[1], gg_W=tan[2], need_pos=True, ws=ws,
                                       outputs=(outs[4], outs[5], outs[6], outs[7]))
        torch.cuda.synchronize()
        delta = torch.cuda.max_memory_allocated(dev) - mem0
        assert binding.tpconv_device_error() == 0
        assert all(bool(torch.isfinite(o).all()) for o in outs)
        rows.append((k, p.E, wsb, delta))
        del ws
    assert len({r[2] for r in rows}) == 1, rows
    assert len({r[3] for r in rows}) == 1, rows
    # the caching allocator hands out large blocks in multiples of 2 MiB
    two_mib = 2 << 20
    assert rows[0][3] <= (rows[0][2] + two_mib - 1) // two_mib * two_mib, rows


@pytest.mark.parametrize("cfg,n,k", [(4, 200, None), (3, 160, None), (5, 120, 40)])
def test_staging_windows_smaller_than_a_receiver(torch, cfg, n, k):
    """With the smallest budget (4 KiB) the staging window holds 32 edges: many windows per
    receiver range, and receivers of more than 32 in-edges cut by window boundaries."""
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=n, k=k)
    lp = lib_plan(p.cfg)
    d = {k: cuda(a) for k, a in (("x", p.x), ("pos", p.pos), ("row_ptr", p.row_ptr), ("src", p.src),
                                 ("W", p.W), ("gout", p.gout))}
    v = binding.tpconv_csr_transpose(d["row_ptr"], d["src"], p.N)
    ggx, ggp, ggw = (workloads.normal(p.rng, s) for s in (p.x.shape, p.pos.shape, p.W.shape))

    def run():
        _, gp, _ = binding.tpconv_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"], d["gout"],
                                           need_x=False, need_W=False)
        *_, dp = binding.tpconv_double_backward(lp, d["x"], d["pos"], d["row_ptr"], d["src"], *v, d["W"],
                                                d["gout"], gg_x=cuda(ggx), gg_pos=cuda(ggp), gg_W=cuda(ggw),
                                                need_x=False, need_W=False, need_grad_out=False, need_pos=True)
        return gp.cpu().numpy(), dp.cpu().numpy()

    ref_gp, ref_dp = run()
    lp.set_workspace_budget(4096)
    # some receiver straddles a window boundary: uvw windows start at each receiver range
    # (one receiver per range at this budget), uvu windows at edge 0
    starts = np.arange(0, p.E, 32) if p.cfg.mode == "uvu" else p.row_ptr[:-1] + 32
    starts = starts[starts < p.E]
    owner = np.searchsorted(p.row_ptr, starts, side="right") - 1
    assert np.any((starts > p.row_ptr[owner]) & (starts < p.row_ptr[owner + 1]))
    gp, dp = run()
    assert binding.tpconv_device_error() == 0
    assert rel_l2(gp, ref_gp) <= 1e-6
    assert rel_l2(dp, ref_dp) <= 1e-6
    _, orp, _ = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    odp = conv.double_backward_pos(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout, ggx, ggp, ggw)
    assert rel_l2(gp, orp) <= TOL
    assert rel_l2(dp, odp) <= TOL
