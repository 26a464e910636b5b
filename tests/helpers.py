"""Shared test helpers: seeded problems for the oracle and the CUDA path."""

import numpy as np

from equivariant_gnn_tensor_dst_b200 import workloads
from oracle import conv, radial

BIG = 1 << 60


def oracle_plan(c):
    rs = radial.RadialSpec(c.radial, c.num_basis, c.r_cut, c.r_min, c.r_max)
    return conv.make_plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, rs)


def lib_plan(c):
    from equivariant_gnn_tensor_dst_b200 import binding
    return binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                        c.r_min, c.r_max)


class Problem:
    """Graph + float32 inputs for one configuration (numpy, host)."""

    def __init__(self, cfg, n_nodes=None, seed=None, k=None, config=None):
        c = config if config is not None else workloads.CONFIGS[cfg]
        self.cfg = c
        self.plan = oracle_plan(c)
        g, rng = workloads.make_graph(c, n_nodes=n_nodes, seed=seed, k=k)
        self.pos, self.row_ptr, self.src = g.pos, g.row_ptr, g.src
        self.N, self.E = g.n_nodes, g.n_edges
        self.x = workloads.normal(rng, (self.N, self.plan.dim_in))
        self.W = workloads.weights(rng, c.num_basis, self.plan.fan_in_per_column())
        self.gout = workloads.normal(rng, (self.N, self.plan.dim_out))
        self.rng = rng

    def scalar_mask(self):
        m = np.zeros(self.plan.dim_out, dtype=np.float32)
        for b in self.plan.blocks_out:
            if b.l == 0 and b.parity == 1:
                m[b.offset:b.offset + b.size] = 1.0
        return m

    def edges_of(self, receivers):
        rp = self.row_ptr.astype(np.int64)
        return np.concatenate([np.arange(rp[i], rp[i + 1]) for i in receivers]) if len(receivers) else \
            np.zeros(0, np.int64)


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return num
    return num / den


def cuda(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()
