"""The compute entry points allocate nothing and never synchronise, so a forward +
backward can be captured into a CUDA graph and replayed.  Replays must reproduce the
eager results bit for bit (the library's reductions are in fixed order) and must read
the inputs' current contents."""

import numpy as np
import pytest

from helpers import Problem, cuda, lib_plan

pytestmark = pytest.mark.gpu


def test_forward_backward_capture_and_replay():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(2, n_nodes=300)
    lp = lib_plan(p.cfg)
    x, pos, rp, src, W, go = (cuda(a) for a in (p.x, p.pos, p.row_ptr, p.src, p.W, p.gout))
    views = binding.tpconv_csr_transpose(rp, src, p.N)
    N, E = p.N, p.E
    ws = binding.workspace(lp.workspace_bytes(N, E), x.device)
    out = torch.empty(N, lp.dim_out, device="cuda")
    gx = torch.empty(N, lp.dim_in, device="cuda")
    gp = torch.empty(N, 3, device="cuda")
    gw = torch.empty(lp.num_basis, lp.weight_cols, device="cuda")

    def step():
        binding.tpconv_forward(lp, x, pos, rp, src, W, out=out, ws=ws)
        binding.tpconv_backward(lp, x, pos, rp, src, *views, W, go, ws=ws, outputs=(gx, gp, gw))

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                   # eager warm-up (one-time function attributes)
        torch.cuda.synchronize()
        ref = [t.clone() for t in (out, gx, gp, gw)]
    torch.cuda.current_stream().wait_stream(side)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        for t in (out, gx, gp, gw):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip((out, gx, gp, gw), ref):
            assert torch.equal(a, b)

    # the graph reads the inputs' current contents
    x.mul_(2.0)
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (out, gx, gp, gw)]
    step()
    torch.cuda.synchronize()
    for a, b in zip(got, (out, gx, gp, gw)):
        assert torch.equal(a, b)
    assert not torch.equal(got[0], ref[0])
    del graph


def test_double_backward_capture_and_replay():
    """The double backward with every output, dLambda/dpos included, captured and replayed."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_gnn_tensor_dst_b200 import binding, workloads
    p = Problem(5, n_nodes=200)
    lp = lib_plan(p.cfg)
    x, pos, rp, src, W, go = (cuda(a) for a in (p.x, p.pos, p.row_ptr, p.src, p.W, p.gout))
    ggx, ggp, ggw = (cuda(workloads.normal(p.rng, s)) for s in (p.x.shape, p.pos.shape, p.W.shape))
    views = binding.tpconv_csr_transpose(rp, src, p.N)
    N, E = p.N, p.E
    ws = binding.workspace(lp.workspace_bytes(N, E), x.device)
    outs = (torch.empty(N, lp.dim_in, device="cuda"), torch.empty(lp.num_basis, lp.weight_cols, device="cuda"),
            torch.empty(N, lp.dim_out, device="cuda"), torch.empty(N, 3, device="cuda"))

    def step():
        binding.tpconv_double_backward(lp, x, pos, rp, src, *views, W, go, gg_x=ggx, gg_pos=ggp, gg_W=ggw,
                                       need_pos=True, ws=ws, outputs=outs)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
        torch.cuda.synchronize()
        ref = [t.clone() for t in outs]
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        for t in outs:
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(outs, ref):
            assert torch.equal(a, b)
    del graph
