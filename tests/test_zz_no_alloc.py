"""The forward entry point that allocates nothing (tpconv_forward_no_alloc).

Some callers cannot obtain device memory themselves: a plug-in whose host application owns
every device allocation, or code that must not call cudaMalloc because that call can
synchronise the device in the middle of latency-critical work.  For them the library keeps
its forward scratch in a fixed array compiled into the library.  These tests call that entry
point through the C ABI twice in a row and check each result against the ordinary forward
(caller-provided workspace) on every row, and against the float64 oracle on sampled rows,
within the tolerance the other parity tests use.

The file is named to be collected last, so that a run stopping at the first failure has
already run every other test; it also passes when run alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest

from oracle import conv, radial

from helpers import Problem, cuda, lib_plan, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-4
SCRATCH_BYTES = 32 << 20      # TPCONV_STATIC_SCRATCH_BYTES


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _no_alloc(lp, N, E, x, pos, rp, src, W):
    """Two calls in a row through the C ABI; returns both outputs (host arrays)."""
    import torch
    from equivariant_gnn_tensor_dst_b200 import binding
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = binding.lib()
    outs = []
    for _ in range(2):
        out = torch.full((N, lp.dim_out), float("nan"), dtype=torch.float32, device="cuda")
        st = L.tpconv_forward_no_alloc(lp.handle, N, E, ctypes.c_void_p(x.data_ptr()),
                                       ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(rp.data_ptr()),
                                       ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                                       ctypes.c_void_p(out.data_ptr()), stream)
        assert st == 0, L.tpconv_status_string(st)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        outs.append(got)
    return outs


@pytest.mark.parametrize("cfg,n", [(2, 700), (3, 200), (4, 150)])
def test_forward_no_alloc_matches_forward(cfg, n):
    _torch()
    from equivariant_gnn_tensor_dst_b200 import binding

    p = Problem(cfg, n_nodes=n)
    lp = lib_plan(p.cfg)
    x, pos, rp, src, W = cuda(p.x), cuda(p.pos), cuda(p.row_ptr), cuda(p.src), cuda(p.W)
    ref = binding.tpconv_forward(lp, x, pos, rp, src, W).cpu().numpy()
    rows = np.sort(p.rng.choice(p.N, size=min(p.N, 48), replace=False))
    oracle = conv.forward(p.plan, p.x, p.pos, p.row_ptr, p.src, p.W, edges=p.edges_of(rows))
    for got in _no_alloc(lp, p.N, p.E, x, pos, rp, src, W):
        assert rel_l2(got, ref) <= TOL
        assert rel_l2(got[rows], oracle[rows]) <= TOL


def test_forward_no_alloc_small_state_many_ranges():
    """A plan with a tiny per-receiver state (one scalar channel, K = 1) on a graph with more
    receivers than one range of the fixed scratch holds: the range is sized so that the
    padded arrays fit, and the receivers run in two ranges."""
    _torch()
    from equivariant_gnn_tensor_dst_b200 import binding

    irreps, K, r_cut = "1x0e", 1, 400.0
    lp = binding.Plan(irreps, 0, irreps, "uvw", radial.BESSEL, K, r_cut)
    per_node = 4 * (1 + 8 * 1)            # state + split-K slices, bytes per receiver
    N = 1_000_000
    assert N * per_node > SCRATCH_BYTES
    rng = np.random.default_rng(77)
    pos = rng.uniform(0.0, 100.0, size=(N, 3)).astype(np.float32)
    i = np.arange(N)
    nb = np.stack([(i + 1) % N, (i + 7) % N], axis=1)
    nb.sort(axis=1)
    src = nb.reshape(-1).astype(np.int32)
    row_ptr = (2 * np.arange(N + 1)).astype(np.int32)
    x = rng.standard_normal((N, 1)).astype(np.float32)
    W = rng.standard_normal((K, 1)).astype(np.float32)
    d = [cuda(a) for a in (x, pos, row_ptr, src, W)]
    ref = binding.tpconv_forward(lp, *d).cpu().numpy()
    op = conv.make_plan(irreps, 0, irreps, "uvw", radial.RadialSpec(radial.BESSEL, K, r_cut))
    rows = np.sort(np.concatenate([rng.choice(N, 30, replace=False), [0, N // 2, N - 1]]))
    edges = np.concatenate([np.arange(2 * r, 2 * r + 2) for r in rows])
    oracle = conv.forward(op, x, pos, row_ptr, src, W, edges=edges)
    for got in _no_alloc(lp, N, 2 * N, *d):
        assert rel_l2(got, ref) <= TOL
        assert rel_l2(got[rows], oracle[rows]) <= TOL
