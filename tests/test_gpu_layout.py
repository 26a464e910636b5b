"""mul_ir boundary layout (tpconv_plan_set_layout): node arrays in blocks [C][2l+1].
Every pass must return exactly the ir_mul results with the block transpose applied (the
same kernels run on the same data), and so match the oracle."""

import numpy as np
import pytest

from helpers import Problem, cuda, lib_plan, rel_l2
from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv

pytestmark = pytest.mark.gpu


def _to_mul_ir(a, blocks):
    """ir_mul [N, dim] -> mul_ir: each block [2l+1][C] transposed to [C][2l+1]."""
    out = np.empty_like(a)
    for b in blocks:
        R = 2 * b.l + 1
        blk = a[:, b.offset:b.offset + b.size].reshape(a.shape[0], R, b.mul)
        out[:, b.offset:b.offset + b.size] = blk.transpose(0, 2, 1).reshape(a.shape[0], -1)
    return out


def _from_mul_ir(a, blocks):
    out = np.empty_like(a)
    for b in blocks:
        R = 2 * b.l + 1
        blk = a[:, b.offset:b.offset + b.size].reshape(a.shape[0], b.mul, R)
        out[:, b.offset:b.offset + b.size] = blk.transpose(0, 2, 1).reshape(a.shape[0], -1)
    return out


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("cfg,n", [(2, 160), (3, 96), (5, 160)])
def test_mul_ir_layout_every_pass(torch, cfg, n):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=n)
    bi, bo = p.plan.blocks_in, p.plan.blocks_out
    a = lib_plan(p.cfg)                      # ir_mul
    m = lib_plan(p.cfg)
    m.set_layout(binding.LAYOUT_MUL_IR)
    assert m.workspace_bytes(p.N, p.E) > a.workspace_bytes(p.N, p.E)
    x, pos, rp, src, W, go = (cuda(v) for v in (p.x, p.pos, p.row_ptr, p.src, p.W, p.gout))
    xm, gom = cuda(_to_mul_ir(p.x, bi)), cuda(_to_mul_ir(p.gout, bo))
    v = binding.tpconv_csr_transpose(rp, src, p.N)

    out_a = binding.tpconv_forward(a, x, pos, rp, src, W).cpu().numpy()
    out_m = binding.tpconv_forward(m, xm, pos, rp, src, W).cpu().numpy()
    assert np.array_equal(_from_mul_ir(out_m, bo), out_a)
    assert rel_l2(out_a, conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)) <= 1e-4

    ga = [t.cpu().numpy() for t in binding.tpconv_backward(a, x, pos, rp, src, *v, W, go)]
    gm = [t.cpu().numpy() for t in binding.tpconv_backward(m, xm, pos, rp, src, *v, W, gom)]
    assert np.array_equal(_from_mul_ir(gm[0], bi), ga[0])
    assert np.array_equal(gm[1], ga[1]) and np.array_equal(gm[2], ga[2])

    ggx = workloads.normal(p.rng, p.x.shape)
    ggp = workloads.normal(p.rng, p.pos.shape)
    ggw = workloads.normal(p.rng, p.W.shape)
    da = [t.cpu().numpy() for t in binding.tpconv_double_backward(a, x, pos, rp, src, *v, W, go, gg_x=cuda(ggx),
                                                                  gg_pos=cuda(ggp), gg_W=cuda(ggw), need_pos=True)]
    dm = [t.cpu().numpy() for t in binding.tpconv_double_backward(m, xm, pos, rp, src, *v, W, gom,
                                                                  gg_x=cuda(_to_mul_ir(ggx, bi)), gg_pos=cuda(ggp),
                                                                  gg_W=cuda(ggw), need_pos=True)]
    assert np.array_equal(_from_mul_ir(dm[0], bi), da[0])
    assert np.array_equal(dm[1], da[1])
    assert np.array_equal(_from_mul_ir(dm[2], bo), da[2])
    assert np.array_equal(dm[3], da[3])          # dLambda/dpos: [N][3] in both layouts

    if p.cfg.mode == "uvw":
        Y = workloads.normal(p.rng, (p.E, p.plan.n_sh))
        phi = workloads.normal(p.rng, (p.E, p.cfg.num_basis))
        ea = binding.tpconv_forward_embedded(a, x, cuda(Y), cuda(phi), rp, src, W).cpu().numpy()
        em = binding.tpconv_forward_embedded(m, xm, cuda(Y), cuda(phi), rp, src, W).cpu().numpy()
        assert np.array_equal(_from_mul_ir(em, bo), ea)
        ba = [t.cpu().numpy() for t in binding.tpconv_backward_embedded(a, x, cuda(Y), cuda(phi), rp, src, *v, W, go)]
        bm = [t.cpu().numpy() for t in binding.tpconv_backward_embedded(m, xm, cuda(Y), cuda(phi), rp, src, *v, W,
                                                                          gom)]
        assert np.array_equal(_from_mul_ir(bm[0], bi), ba[0])
        for u, w in zip(bm[1:], ba[1:]):
            assert np.array_equal(u, w)
