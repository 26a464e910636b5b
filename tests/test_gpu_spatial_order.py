"""Spatial (Morton) node order, graph renumbering and row gathers (include/tpconv_graph.h).

* The permutation equals the definition restated here in numpy: float32 cell indices
  floor((pos - lo) * (1024 / (hi - lo))) clamped to [0, 1023] (the same float32
  operations as the kernel, so the same integer decisions), bits interleaved x, y, z
  from the lowest, nodes sorted by (code, id).  Bit for bit.
* The renumbered CSR equals the relabelling written out in numpy.  Bit for bit.
* The convolution on the renumbered graph is the renumbered convolution: forward and
  backward against the oracle on the original graph, permuted (relative L2 <= 1e-4).
* Degenerate inputs: coincident nodes (identity order), one node, no edges.
"""

import numpy as np
import pytest

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


def _morton_perm(pos):
    pos = np.asarray(pos, np.float32)
    lo, hi = pos.min(0), pos.max(0)
    ext = (hi - lo).astype(np.float32)
    scale = np.where(ext > 0, np.float32(1024.0) / np.where(ext > 0, ext, np.float32(1)), np.float32(0))
    t = np.floor((pos - lo).astype(np.float32) * scale.astype(np.float32)).astype(np.float32)
    c = np.clip(t, 0, 1023).astype(np.uint64)
    code = np.zeros(pos.shape[0], np.uint64)
    for b in range(10):
        for a in range(3):
            code |= ((c[:, a] >> np.uint64(b)) & np.uint64(1)) << np.uint64(3 * b + a)
    return np.lexsort((np.arange(pos.shape[0]), code)).astype(np.int32)


def _relabel(row_ptr, src, perm):
    N = row_ptr.shape[0] - 1
    inv = np.empty(N, np.int32)
    inv[perm] = np.arange(N, dtype=np.int32)
    rows = [inv[src[row_ptr[o]:row_ptr[o + 1]]] for o in perm]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    so = np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, np.int32)
    return rp, so, inv


@pytest.mark.parametrize("cfg,n", [(2, 300), (4, 700), (3, 200)])
def test_spatial_order_and_relabel_bit_exact(torch, cfg, n):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=n)
    perm = binding.tpconv_spatial_order(cuda(p.pos)).cpu().numpy()
    want = _morton_perm(p.pos)
    assert np.array_equal(perm, want)
    rp, so, inv = binding.tpconv_permute_graph(cuda(p.row_ptr), cuda(p.src), cuda(perm))
    wrp, wso, winv = _relabel(p.row_ptr, p.src, perm)
    assert np.array_equal(rp.cpu().numpy(), wrp)
    assert np.array_equal(so.cpu().numpy(), wso)
    assert np.array_equal(inv.cpu().numpy(), winv)
    x2 = binding.tpconv_gather_rows(cuda(p.x), cuda(perm)).cpu().numpy()
    assert np.array_equal(x2, p.x[perm])


@pytest.mark.parametrize("cfg,n", [(2, 160), (3, 96)])
def test_convolution_on_spatial_order(torch, cfg, n):
    from equivariant_gnn_tensor_dst_b200 import binding
    p = Problem(cfg, n_nodes=n)
    lp = lib_plan(p.cfg)
    d_perm = binding.tpconv_spatial_order(cuda(p.pos))
    perm = d_perm.cpu().numpy()
    rp, so, _ = binding.tpconv_permute_graph(cuda(p.row_ptr), cuda(p.src), d_perm)
    x2, pos2, go2 = (binding.tpconv_gather_rows(cuda(a), d_perm) for a in (p.x, p.pos, p.gout))
    W = cuda(p.W)
    out = binding.tpconv_forward(lp, x2, pos2, rp, so, W).cpu().numpy()
    ref = conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W)[perm]
    assert rel_l2(out, ref) <= TOL
    v = binding.tpconv_csr_transpose(rp, so, p.N)
    gx, gp, gw = binding.tpconv_backward(lp, x2, pos2, rp, so, *v, W, go2)
    rx, rpos, rw = conv.backward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, p.gout)
    assert rel_l2(gx.cpu().numpy(), rx[perm]) <= TOL
    assert rel_l2(gp.cpu().numpy(), rpos[perm]) <= TOL
    assert rel_l2(gw.cpu().numpy(), rw) <= TOL


def test_spatial_order_degenerate(torch):
    from equivariant_gnn_tensor_dst_b200 import binding
    pos = np.ones((37, 3), np.float32)                 # coincident: every code is 0
    assert np.array_equal(binding.tpconv_spatial_order(cuda(pos)).cpu().numpy(), np.arange(37))
    one = binding.tpconv_spatial_order(cuda(np.zeros((1, 3), np.float32))).cpu().numpy()
    assert np.array_equal(one, [0])
    rp = np.zeros(6, np.int32)                         # 5 nodes, no edges
    perm = np.array([4, 2, 0, 1, 3], np.int32)
    r2, s2, inv = binding.tpconv_permute_graph(cuda(rp), cuda(np.zeros(0, np.int32)), cuda(perm))
    assert np.array_equal(r2.cpu().numpy(), rp)
    assert s2.numel() == 0
    assert np.array_equal(inv.cpu().numpy()[perm], np.arange(5))
