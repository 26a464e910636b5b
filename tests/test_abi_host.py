"""Host-side checks of the C ABI (no GPU needed).

* the shared library loads and exports every function declared in include/*.h;
* the plan builder enumerates the same paths, widths and weight offsets as the oracle
  and its coupling tables (computed by a different algorithm at build time) equal the
  oracle's to 1e-12;
* argument errors are reported before anything is launched.
"""

import ctypes
import os
import re

import numpy as np
import pytest

from equivariant_gnn_tensor_dst_b200 import binding
from equivariant_gnn_tensor_dst_b200.workloads import CONFIGS
from oracle import conv, radial

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    """Functions declared in every header under include/."""
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(tpconv_\w+)\s*\(", txt))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(binding.SIGNATURES)


def _oracle_plan(cfg):
    c = CONFIGS[cfg]
    rs = radial.RadialSpec(c.radial, c.num_basis, c.r_cut, c.r_min, c.r_max)
    return conv.make_plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, rs)


def _lib_plan(cfg):
    c = CONFIGS[cfg]
    return binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                        c.r_min, c.r_max)


@pytest.mark.parametrize("cfg", sorted(CONFIGS))
def test_plan_matches_oracle(cfg):
    op, lp = _oracle_plan(cfg), _lib_plan(cfg)
    assert (lp.dim_in, lp.dim_out, lp.weight_cols, lp.num_basis) == (op.dim_in, op.dim_out, op.n_w,
                                                                     op.radial.num_basis)
    assert lp.num_paths == len(op.paths)
    for i, p in enumerate(op.paths):
        q = lp.path(i)
        assert (q["l_in"], q["l_sh"], q["l_out"], q["block_in"], q["block_out"], q["c_in"], q["c_out"],
                q["w_offset"], q["w_count"]) == (p.l_in, p.l_sh, p.l_out, p.block_in, p.block_out, p.c_in,
                                                 p.c_out, p.w_offset, p.w_count)
        idx, val = lp.coupling(i)
        dense = np.zeros_like(op.coupling[i])
        for (a, b, c), v in zip(idx, val):
            dense[a, b, c] = v
        assert np.abs(dense - op.coupling[i]).max() < 1e-12
    assert np.array_equal(lp.fan_in_per_column(), op.fan_in_per_column())


def test_plan_general_parities_match_oracle():
    rs = radial.RadialSpec(radial.BESSEL, 6, 2.5)
    ii, io = "2x0e+2x1o+1x1e+1x3o", "2x0e+1x1e+2x1o+1x2e+1x2o+1x3e"
    op = conv.make_plan(ii, 3, io, "uvw", rs)
    lp = binding.Plan(ii, 3, io, "uvw", "bessel", 6, 2.5)
    assert lp.num_paths == len(op.paths)
    for i, p in enumerate(op.paths):
        idx, val = lp.coupling(i)
        dense = np.zeros_like(op.coupling[i])
        for (a, b, c), v in zip(idx, val):
            dense[a, b, c] = v
        assert np.abs(dense - op.coupling[i]).max() < 1e-12


@pytest.mark.parametrize("args,code", [
    (("4x0q", 2, "4x0e", "uvw"), 2),
    (("4x0e", 2, "", "uvw"), 2),
    (("4x5e", 2, "4x0e", "uvw"), 3),
    (("4x0e", 4, "4x0e", "uvw"), 3),
    (("4x0e+4x1o", 1, "2x1o", "uvu"), 1),
    (("4x0e", 0, "4x1o", "uvw"), 1),   # no valid path
])
def test_plan_errors(args, code):
    with pytest.raises(binding.TPConvError) as e:
        binding.Plan(*args)
    assert e.value.status == code


def test_radial_spec_errors():
    with pytest.raises(binding.TPConvError):
        binding.Plan("4x0e", 1, "4x0e", "uvw", "bessel", 17, 5.0)
    with pytest.raises(binding.TPConvError):
        binding.Plan("4x0e", 1, "4x0e", "uvw", "bessel", 8, -1.0)
    with pytest.raises(binding.TPConvError):
        binding.Plan("4x0e", 1, "4x0e", "uvw", "gaussian", 8, 5.0, 3.0, 1.0)


def test_workspace_is_bounded_and_independent_of_edges():
    lp = _lib_plan(2)
    fwd = [lp.workspace_bytes(4096, 4096 * k, binding.PASS_FORWARD) for k in (8, 32, 128)]
    assert fwd[0] == fwd[1] == fwd[2]
    assert fwd[0] <= (128 << 20) + 4096
    lp.set_workspace_budget(1 << 20)
    assert lp.workspace_bytes(4096, 131072, binding.PASS_FORWARD) < fwd[0]
    lp.set_workspace_budget(128 << 20)
    # backward and double backward: node states, split-K slices and the position-gradient
    # staging window all fit the budget, for any number of edges (the degree sweep k = 8..128
    # at N = 4096, and a graph far larger than one staging window)
    for mask in (binding.PASS_BACKWARD, binding.PASS_DOUBLE_BACKWARD,
                 binding.PASS_FORWARD | binding.PASS_BACKWARD | binding.PASS_DOUBLE_BACKWARD):
        ws = [lp.workspace_bytes(4096, 4096 * k, mask) for k in (8, 16, 32, 64, 128)]
        ws.append(lp.workspace_bytes(4096, 50_000_000, mask))
        assert len(set(ws)) == 1
        assert ws[0] <= (128 << 20) + 8 * 4096 + 4096   # + receiver order and source cursor


def test_forward_rejects_bad_arguments_before_launch():
    L = binding.lib()
    lp = _lib_plan(2)
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced: the checks fail first
    mis = ctypes.c_void_p((1 << 20) + 4)
    ws_need = lp.workspace_bytes(100, 1000, binding.PASS_FORWARD)
    args = [lp.handle, 100, 1000, fake, fake, fake, fake, fake, fake, fake]
    assert L.tpconv_forward(*args, ws_need - 1, None) == 4             # workspace too small
    assert L.tpconv_forward(lp.handle, 100, 1000, mis, fake, fake, fake, fake, fake, fake, ws_need,
                            None) == 5                                 # misaligned
    assert L.tpconv_forward(lp.handle, 100, 1000, None, fake, fake, fake, fake, fake, fake, ws_need,
                            None) == 1                                 # null x
    assert L.tpconv_forward(lp.handle, -1, 1000, fake, fake, fake, fake, fake, fake, fake, ws_need,
                            None) == 1
    assert L.tpconv_forward(None, 100, 1000, fake, fake, fake, fake, fake, fake, fake, ws_need,
                            None) == 1
    # N == 0 is a no-op
    assert L.tpconv_forward(lp.handle, 0, 0, None, None, None, None, None, None, None, 0, None) == 0


def test_double_backward_position_output_checks():
    """dLambda/dpos needs the source view's t_ptr and t_eid, takes 16-byte aligned
    output, and its per-edge staging window is counted in the double backward's workspace
    (a fixed window: the workspace does not grow with the edges).  Every case returns
    before any launch."""
    L = binding.lib()
    lp = _lib_plan(5)
    fake = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 4)
    ptrs = [fake] * 17          # x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out,
    #                             gg_x, gg_pos, gg_W, grad_x, grad_W, grad_grad_out, grad_pos, ws
    ptrs[5] = None              # t_eid missing
    assert L.tpconv_double_backward(lp.handle, 10, 20, *ptrs, 1 << 30, None) == 1
    ptrs = [fake] * 17
    ptrs[15] = mis              # misaligned grad_pos
    assert L.tpconv_double_backward(lp.handle, 10, 20, *ptrs, 1 << 30, None) == 5
    ptrs = [fake] * 17          # workspace one byte short
    need = lp.workspace_bytes(10, 20, binding.PASS_DOUBLE_BACKWARD)
    assert L.tpconv_double_backward(lp.handle, 10, 20, *ptrs, need - 1, None) == 4
    a = lp.workspace_bytes(1000, 64000, binding.PASS_DOUBLE_BACKWARD)
    b = lp.workspace_bytes(1000, 128000, binding.PASS_DOUBLE_BACKWARD)
    assert a == b
    assert a > lp.workspace_bytes(1000, 64000, binding.PASS_FORWARD)   # the staging window


def test_status_strings():
    L = binding.lib()
    for s in range(8):
        assert L.tpconv_status_string(s)
    assert L.tpconv_status_string(99) == b"unknown status"


def test_binding_arity_matches_header():
    txt = open(os.path.join(ROOT, "include", "tpconv.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    for name, params in re.findall(r"\b(tpconv_\w+)\s*\(([^;{]*?)\)\s*;", txt, flags=re.S):
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        assert len(binding.SIGNATURES[name][1]) == n, name


def test_plan_set_math_arguments():
    L = binding.lib()
    p = binding.Plan("8x0e+8x1o", 2, "8x0e+8x1o", "uvw", "bessel", 8, 3.0)
    assert L.tpconv_plan_set_math(p.handle, binding.MATH_TF32) == 0
    assert L.tpconv_plan_set_math(p.handle, binding.MATH_BF16) == 0
    assert L.tpconv_plan_set_math(p.handle, binding.MATH_FP32) == 0
    assert L.tpconv_plan_set_math(p.handle, 7) == 3          # TPCONV_ERR_UNSUPPORTED
    assert L.tpconv_plan_set_math(None, binding.MATH_FP32) == 1   # TPCONV_ERR_INVALID_ARG


def test_plan_set_layout_arguments():
    L = binding.lib()
    p = binding.Plan("8x0e+8x1o", 2, "8x0e+8x1o", "uvw", "bessel", 8, 3.0)
    base = p.workspace_bytes(100, 800)
    assert L.tpconv_plan_set_layout(p.handle, binding.LAYOUT_MUL_IR) == 0
    assert p.workspace_bytes(100, 800) > base
    assert L.tpconv_plan_set_layout(p.handle, 5) == 3          # TPCONV_ERR_UNSUPPORTED
    assert L.tpconv_plan_set_layout(None, 0) == 1              # TPCONV_ERR_INVALID_ARG
    assert L.tpconv_plan_set_layout(p.handle, binding.LAYOUT_IR_MUL) == 0
    assert p.workspace_bytes(100, 800) == base


def test_graph_header_symbols_and_host_checks():
    """Every function of include/tpconv_graph.h is exported; argument checks return
    before any launch."""
    txt = open(os.path.join(ROOT, "include", "tpconv_graph.h")).read()
    names = set(re.findall(r"\b(tpconv_\w+)\s*\(", txt))
    assert names >= {"tpconv_spatial_order", "tpconv_spatial_order_workspace_bytes", "tpconv_permute_graph",
                     "tpconv_gather_rows"}
    L = binding.lib()
    for n in names:
        assert hasattr(L, n), n
    nb = ctypes.c_size_t()
    assert L.tpconv_spatial_order_workspace_bytes(1000, ctypes.byref(nb)) == 0
    assert nb.value == 8 * 1024 + 256                      # keys padded to 1024, then the box
    assert L.tpconv_spatial_order_workspace_bytes(-1, ctypes.byref(nb)) == 1
    fake = ctypes.c_void_p(1 << 20)
    assert L.tpconv_spatial_order(10, fake, fake, fake, 16, None) == 4     # workspace too small
    assert L.tpconv_spatial_order(10, None, fake, fake, 1 << 20, None) == 1
    assert L.tpconv_spatial_order(0, None, None, None, 0, None) == 0       # empty: no-op
    assert L.tpconv_permute_graph(-1, 0, fake, fake, fake, fake, fake, fake, None) == 1
    assert L.tpconv_permute_graph(10, 5, fake, None, fake, fake, fake, fake, None) == 1
    assert L.tpconv_gather_rows(10, 4, None, fake, fake, None) == 1
    assert L.tpconv_gather_rows(0, 4, None, None, None, None) == 0
