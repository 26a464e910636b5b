"""The forward entry point that allocates nothing (tpconv_forward_no_alloc).

Some callers cannot obtain device memory themselves: a plug-in whose host application owns
every device allocation, or code that must not call cudaMalloc because that call can
synchronise the device in the middle of latency-critical work.  For them the library keeps
its forward scratch in a fixed array compiled into the library.  This test calls that entry
point through the C ABI twice in a row and checks each result against the ordinary forward
(caller-provided workspace) within the tolerance the other parity tests use.

The file is named to be collected last, so that a run stopping at the first failure has
already run every other test; it also passes when run alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest

from helpers import Problem, cuda, lib_plan, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.mark.parametrize("cfg,n", [(2, 700), (3, 200), (4, 150)])
def test_forward_no_alloc_matches_forward(cfg, n):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_gnn_tensor_dst_b200 import binding

    p = Problem(cfg, n_nodes=n)
    lp = lib_plan(p.cfg)
    x, pos, rp, src, W = cuda(p.x), cuda(p.pos), cuda(p.row_ptr), cuda(p.src), cuda(p.W)
    ref = binding.tpconv_forward(lp, x, pos, rp, src, W)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = binding.lib()
    for _ in range(2):
        out = torch.full((p.N, lp.dim_out), float("nan"), dtype=torch.float32, device="cuda")
        st = L.tpconv_forward_no_alloc(lp.handle, p.N, p.E, ctypes.c_void_p(x.data_ptr()),
                                       ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(rp.data_ptr()),
                                       ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                                       ctypes.c_void_p(out.data_ptr()), stream)
        assert st == 0, binding.lib().tpconv_status_string(st)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_l2(got, ref.cpu().numpy()) <= TOL
