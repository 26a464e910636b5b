"""ctypes binding of libtpconv.so (include/tpconv.h).

Argument marshalling only: every computation runs in the library's kernels.  Tensors
are torch tensors (device memory, float32 / int32, contiguous); PyTorch is used to
allocate outputs and workspaces and to name the current CUDA stream.  If the shared
library is missing the import of ``lib()`` fails loudly; there is no fallback.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpconv.so")

UVW, UVU = 0, 1
BESSEL, GAUSSIAN = 0, 1
PASS_FORWARD, PASS_BACKWARD, PASS_DOUBLE_BACKWARD = 1, 2, 4
MATH_FP32, MATH_TF32, MATH_BF16 = 0, 1, 2
LAYOUT_IR_MUL, LAYOUT_MUL_IR = 0, 1

_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p


class RadialSpec(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("num_basis", ctypes.c_int32), ("r_cut", ctypes.c_float),
                ("r_min", ctypes.c_float), ("r_max", ctypes.c_float), ("poly_p", ctypes.c_int32)]


# symbol -> (restype, argtypes); mirrors include/tpconv.h
SIGNATURES = {
    "tpconv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tpconv_plan_create": (ctypes.c_int, [ctypes.POINTER(_c_p), ctypes.c_char_p, ctypes.c_int32,
                                          ctypes.c_char_p, ctypes.c_int32, ctypes.POINTER(RadialSpec)]),
    "tpconv_plan_destroy": (ctypes.c_int, [_c_p]),
    "tpconv_plan_info": (ctypes.c_int, [_c_p] + [ctypes.POINTER(_c_i64)] * 5),
    "tpconv_plan_path": (ctypes.c_int, [_c_p, _c_i64, ctypes.POINTER(ctypes.c_int32)]),
    "tpconv_plan_path_coupling": (ctypes.c_int, [_c_p, _c_i64, ctypes.POINTER(ctypes.c_int32),
                                                 ctypes.POINTER(ctypes.c_double), _c_i64]),
    "tpconv_set_workspace_budget": (ctypes.c_int, [_c_p, ctypes.c_size_t]),
    "tpconv_plan_set_math": (ctypes.c_int, [_c_p, ctypes.c_int32]),
    "tpconv_plan_set_layout": (ctypes.c_int, [_c_p, ctypes.c_int32]),
    "tpconv_workspace_bytes": (ctypes.c_int, [_c_p, _c_i64, _c_i64, ctypes.c_uint32,
                                              ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_csr_transpose_workspace_bytes": (ctypes.c_int, [_c_i64, _c_i64, ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_csr_transpose": (ctypes.c_int, [_c_i64, _c_i64] + [_c_p] * 6 + [ctypes.c_size_t, _c_p]),
    "tpconv_validate_graph": (ctypes.c_int, [_c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p]),
    "tpconv_forward": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 7 + [ctypes.c_size_t, _c_p]),
    "tpconv_backward": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 13 + [ctypes.c_size_t, _c_p]),
    "tpconv_double_backward": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 17 + [ctypes.c_size_t, _c_p]),
    "tpconv_forward_embedded": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 8 + [ctypes.c_size_t, _c_p]),
    "tpconv_backward_embedded": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 15 + [ctypes.c_size_t, _c_p]),
    "tpconv_profile_begin": (ctypes.c_int, [ctypes.c_int32]),
    "tpconv_profile_end": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_c_i64), ctypes.c_int32]),
    "tpconv_profile_category_name": (ctypes.c_char_p, [ctypes.c_int32]),
    "tpconv_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32)]),
    "tpconv_forward_no_alloc": (ctypes.c_int, [_c_p, _c_i64, _c_i64] + [_c_p] * 6 + [_c_p]),
    # include/tpconv_graph.h
    "tpconv_spatial_order_workspace_bytes": (ctypes.c_int, [_c_i64, ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_spatial_order": (ctypes.c_int, [_c_i64, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "tpconv_permute_graph": (ctypes.c_int, [_c_i64, _c_i64] + [_c_p] * 6 + [_c_p]),
    "tpconv_gather_rows": (ctypes.c_int, [_c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p]),
}
PROF_CATEGORIES = 13

_lib = None


def lib():
    """Load libtpconv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not found: build it with "
                               "`python -m equivariant_gnn_tensor_dst_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class TPConvError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        msg = lib().tpconv_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})" if where else msg)


def check(status, where=""):
    if status != 0:
        raise TPConvError(status, where)


# ---------------------------------------------------------------------------
# plan
# ---------------------------------------------------------------------------

class Plan:
    """tpconv_plan_create / tpconv_plan_destroy and the introspection calls."""

    def __init__(self, irreps_in, sh_lmax, irreps_out, mode="uvw", radial="bessel", num_basis=8,
                 r_cut=5.0, r_min=0.0, r_max=0.0, poly_p=6):
        spec = RadialSpec(BESSEL if radial == "bessel" else GAUSSIAN, int(num_basis), float(r_cut),
                          float(r_min), float(r_max), int(poly_p))
        h = _c_p()
        m = UVW if mode == "uvw" else UVU
        check(lib().tpconv_plan_create(ctypes.byref(h), irreps_in.encode(), int(sh_lmax),
                                       irreps_out.encode(), m, ctypes.byref(spec)), "tpconv_plan_create")
        self._h = h
        self.mode = mode
        vals = [_c_i64() for _ in range(5)]
        check(lib().tpconv_plan_info(h, *[ctypes.byref(v) for v in vals]), "tpconv_plan_info")
        self.num_paths, self.dim_in, self.dim_out, self.num_basis, self.weight_cols = (v.value for v in vals)

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            lib().tpconv_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def path(self, i):
        out = (ctypes.c_int32 * 10)()
        check(lib().tpconv_plan_path(self._h, i, out), "tpconv_plan_path")
        keys = ("l_in", "l_sh", "l_out", "block_in", "block_out", "c_in", "c_out", "w_offset",
                "w_count", "nnz")
        return dict(zip(keys, list(out)))

    def paths(self):
        return [self.path(i) for i in range(self.num_paths)]

    def coupling(self, i):
        nnz = self.path(i)["nnz"]
        idx = (ctypes.c_int32 * (3 * max(nnz, 1)))()
        val = (ctypes.c_double * max(nnz, 1))()
        check(lib().tpconv_plan_path_coupling(self._h, i, idx, val, nnz), "tpconv_plan_path_coupling")
        return [tuple(idx[3 * k:3 * k + 3]) for k in range(nnz)], [val[k] for k in range(nnz)]

    def set_workspace_budget(self, nbytes):
        check(lib().tpconv_set_workspace_budget(self._h, int(nbytes)), "tpconv_set_workspace_budget")

    def set_layout(self, layout):
        """LAYOUT_IR_MUL (default, blocks [2l+1][C]) or LAYOUT_MUL_IR (blocks [C][2l+1])."""
        check(lib().tpconv_plan_set_layout(self._h, int(layout)), "tpconv_plan_set_layout")

    def set_math(self, math):
        """MATH_FP32 (default, 3xTF32 contractions), MATH_TF32 (one TF32 product) or
        MATH_BF16 (operands rounded to bf16, one bf16 product)."""
        check(lib().tpconv_plan_set_math(self._h, int(math)), "tpconv_plan_set_math")

    def workspace_bytes(self, n_nodes, n_edges, passes=PASS_FORWARD | PASS_BACKWARD | PASS_DOUBLE_BACKWARD):
        out = ctypes.c_size_t()
        check(lib().tpconv_workspace_bytes(self._h, int(n_nodes), int(n_edges), int(passes),
                                           ctypes.byref(out)), "tpconv_workspace_bytes")
        return out.value

    def fan_in_per_column(self):
        """Per weight column fan-in K*C_in (uvw) or K (uvu), for N(0, 1/fan_in) init."""
        import numpy as np
        f = np.zeros(self.weight_cols)
        for p in self.paths():
            f[p["w_offset"]:p["w_offset"] + p["w_count"]] = self.num_basis * (p["c_in"] if self.mode == "uvw" else 1)
        return f


# ---------------------------------------------------------------------------
# torch-facing calls
# ---------------------------------------------------------------------------

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name):
    import torch
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace(nbytes, device):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def tpconv_csr_transpose(row_ptr, src, n_nodes, stream=None):
    import torch
    _need(row_ptr, torch.int32, "row_ptr")
    _need(src, torch.int32, "src")
    E = src.numel()
    dev = row_ptr.device
    t_ptr = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    t_eid = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
    t_dst = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
    nb = ctypes.c_size_t()
    check(lib().tpconv_csr_transpose_workspace_bytes(n_nodes, E, ctypes.byref(nb)))
    ws = workspace(nb.value, dev)
    check(lib().tpconv_csr_transpose(n_nodes, E, _ptr(row_ptr), _ptr(src), _ptr(t_ptr), _ptr(t_eid),
                                     _ptr(t_dst), _ptr(ws), ws.numel(), _stream(stream)),
          "tpconv_csr_transpose")
    return t_ptr, t_eid[:E], t_dst[:E]


def tpconv_validate_graph(row_ptr, src, n_nodes, stream=None):
    import torch
    err = torch.zeros(4, dtype=torch.int32, device=row_ptr.device)
    check(lib().tpconv_validate_graph(n_nodes, src.numel(), _ptr(row_ptr), _ptr(src), _ptr(err),
                                      _stream(stream)), "tpconv_validate_graph")
    return err[:1]


def tpconv_forward(plan, x, pos, row_ptr, src, W, out=None, ws=None, stream=None):
    import torch
    for t, n in ((x, "x"), (pos, "pos"), (W, "W")):
        _need(t, torch.float32, n)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(src, torch.int32, "src")
    N, E = pos.shape[0], src.numel()
    if out is None:
        out = torch.empty(N, plan.dim_out, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(plan.workspace_bytes(N, E, PASS_FORWARD), x.device)
    check(lib().tpconv_forward(plan.handle, N, E, _ptr(x), _ptr(pos), _ptr(row_ptr), _ptr(src), _ptr(W),
                               _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "tpconv_forward")
    return out


def tpconv_backward(plan, x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, need_x=True,
                    need_pos=True, need_W=True, ws=None, outputs=None, stream=None):
    import torch
    N, E = pos.shape[0], src.numel()
    dev = x.device
    if outputs is None:
        gx = torch.empty(N, plan.dim_in, dtype=torch.float32, device=dev) if need_x else None
        gp = torch.empty(N, 3, dtype=torch.float32, device=dev) if need_pos else None
        gw = torch.empty(plan.num_basis, plan.weight_cols, dtype=torch.float32, device=dev) if need_W else None
    else:
        gx, gp, gw = outputs
    if ws is None:
        ws = workspace(plan.workspace_bytes(N, E, PASS_BACKWARD), dev)
    check(lib().tpconv_backward(plan.handle, N, E, _ptr(x), _ptr(pos), _ptr(row_ptr), _ptr(src),
                                _ptr(t_ptr), _ptr(t_eid), _ptr(t_dst), _ptr(W), _ptr(grad_out),
                                _ptr(gx), _ptr(gp), _ptr(gw), _ptr(ws), ws.numel(), _stream(stream)),
          "tpconv_backward")
    return gx, gp, gw


def tpconv_forward_embedded(plan, x, Y, phi, row_ptr, src, W, out=None, ws=None, stream=None):
    """Forward with the edge embedding given per edge: Y [E, (lmax+1)^2], phi [E, K]."""
    import torch
    for t, n in ((x, "x"), (Y, "Y"), (phi, "phi"), (W, "W")):
        _need(t, torch.float32, n)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(src, torch.int32, "src")
    N, E = row_ptr.numel() - 1, src.numel()
    if out is None:
        out = torch.empty(N, plan.dim_out, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(plan.workspace_bytes(N, E, PASS_FORWARD), x.device)
    check(lib().tpconv_forward_embedded(plan.handle, N, E, _ptr(x), _ptr(Y), _ptr(phi), _ptr(row_ptr), _ptr(src),
                                        _ptr(W), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
          "tpconv_forward_embedded")
    return out


def tpconv_backward_embedded(plan, x, Y, phi, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, need_x=True,
                             need_W=True, need_phi=True, need_Y=True, ws=None, outputs=None, stream=None):
    """Returns (grad_x, grad_W, grad_phi [E, K], grad_Y [E, (lmax+1)^2])."""
    import torch
    N, E = row_ptr.numel() - 1, src.numel()
    dev = x.device
    if outputs is None:
        gx = torch.empty(N, plan.dim_in, dtype=torch.float32, device=dev) if need_x else None
        gw = torch.empty(plan.num_basis, plan.weight_cols, dtype=torch.float32, device=dev) if need_W else None
        gphi = torch.empty(E, plan.num_basis, dtype=torch.float32, device=dev) if need_phi else None
        gY = torch.empty(E, Y.shape[1], dtype=torch.float32, device=dev) if need_Y else None
    else:
        gx, gw, gphi, gY = outputs
    if ws is None:
        ws = workspace(plan.workspace_bytes(N, E, PASS_BACKWARD), dev)
    check(lib().tpconv_backward_embedded(plan.handle, N, E, _ptr(x), _ptr(Y), _ptr(phi), _ptr(row_ptr), _ptr(src),
                                         _ptr(t_ptr), _ptr(t_eid), _ptr(t_dst), _ptr(W), _ptr(grad_out),
                                         _ptr(gx), _ptr(gw), _ptr(gphi), _ptr(gY), _ptr(ws), ws.numel(),
                                         _stream(stream)),
          "tpconv_backward_embedded")
    return gx, gw, gphi, gY


def tpconv_double_backward(plan, x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, gg_x=None,
                           gg_pos=None, gg_W=None, need_x=True, need_W=True, need_grad_out=True,
                           need_pos=False, ws=None, outputs=None, stream=None):
    """Returns (grad_x, grad_W, grad_grad_out), plus grad_pos [N, 3] when need_pos
    (``outputs`` then has four entries)."""
    import torch
    N, E = pos.shape[0], src.numel()
    dev = x.device
    if outputs is None:
        gx = torch.empty(N, plan.dim_in, dtype=torch.float32, device=dev) if need_x else None
        gw = torch.empty(plan.num_basis, plan.weight_cols, dtype=torch.float32, device=dev) if need_W else None
        gg = torch.empty(N, plan.dim_out, dtype=torch.float32, device=dev) if need_grad_out else None
        gp = torch.empty(N, 3, dtype=torch.float32, device=dev) if need_pos else None
    elif need_pos:
        gx, gw, gg, gp = outputs
    else:
        (gx, gw, gg), gp = outputs, None
    if ws is None:
        ws = workspace(plan.workspace_bytes(N, E, PASS_DOUBLE_BACKWARD), dev)
    check(lib().tpconv_double_backward(plan.handle, N, E, _ptr(x), _ptr(pos), _ptr(row_ptr), _ptr(src),
                                       _ptr(t_ptr), _ptr(t_eid), _ptr(t_dst), _ptr(W), _ptr(grad_out),
                                       _ptr(gg_x), _ptr(gg_pos), _ptr(gg_W), _ptr(gx), _ptr(gw), _ptr(gg),
                                       _ptr(gp), _ptr(ws), ws.numel(), _stream(stream)),
          "tpconv_double_backward")
    return (gx, gw, gg, gp) if need_pos else (gx, gw, gg)


def tpconv_spatial_order(pos, stream=None):
    """perm [N] int32: nodes in Morton order of their positions (perm[k] = old id)."""
    import torch
    _need(pos, torch.float32, "pos")
    N = pos.shape[0]
    perm = torch.empty(max(N, 1), dtype=torch.int32, device=pos.device)
    nb = ctypes.c_size_t()
    check(lib().tpconv_spatial_order_workspace_bytes(N, ctypes.byref(nb)), "tpconv_spatial_order_workspace_bytes")
    ws = workspace(nb.value, pos.device)
    check(lib().tpconv_spatial_order(N, _ptr(pos), _ptr(perm), _ptr(ws), ws.numel(), _stream(stream)),
          "tpconv_spatial_order")
    return perm[:N]


def tpconv_permute_graph(row_ptr, src, perm, stream=None):
    """The receiver CSR renumbered by perm: (row_ptr_out, src_out, inv)."""
    import torch
    _need(row_ptr, torch.int32, "row_ptr")
    _need(src, torch.int32, "src")
    _need(perm, torch.int32, "perm")
    N, E = row_ptr.numel() - 1, src.numel()
    dev = row_ptr.device
    rp = torch.empty(N + 1, dtype=torch.int32, device=dev)
    so = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
    inv = torch.empty(max(N, 1), dtype=torch.int32, device=dev)
    check(lib().tpconv_permute_graph(N, E, _ptr(row_ptr), _ptr(src), _ptr(perm), _ptr(rp), _ptr(so), _ptr(inv),
                                     _stream(stream)), "tpconv_permute_graph")
    return rp, so[:E], inv[:N]


def tpconv_gather_rows(a, perm, stream=None):
    """out[k] = a[perm[k]] for a 2-D float32 array (node features, positions)."""
    import torch
    _need(a, torch.float32, "a")
    _need(perm, torch.int32, "perm")
    rows, width = a.shape[0], (a.numel() // a.shape[0] if a.shape[0] else 0)
    out = torch.empty_like(a)
    check(lib().tpconv_gather_rows(perm.numel(), width, _ptr(a), _ptr(perm), _ptr(out), _stream(stream)),
          "tpconv_gather_rows")
    return out


def tpconv_profile_begin(max_records=8192):
    check(lib().tpconv_profile_begin(int(max_records)), "tpconv_profile_begin")


def tpconv_profile_end():
    """Returns {category: (milliseconds, launches)} for the launches since begin()."""
    n = PROF_CATEGORIES
    ms = (ctypes.c_double * n)()
    cnt = (_c_i64 * n)()
    check(lib().tpconv_profile_end(ms, cnt, n), "tpconv_profile_end")
    return {lib().tpconv_profile_category_name(c).decode(): (ms[c], cnt[c]) for c in range(n)}


def tpconv_device_error():
    """Read and clear the library's device error word (0 = no bounded wait gave up)."""
    v = ctypes.c_int32()
    check(lib().tpconv_device_error(ctypes.byref(v)), "tpconv_device_error")
    return v.value
