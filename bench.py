"""Benchmark of the streaming tensor-product convolution on B200.

One step = one pass of the whole hot path over one batch: forward plus backward
(gradients with respect to x, positions and W) of the edge-scaling uvw workload
"128x0e+64x1o+32x2e+16x3o, SH lmax 3, N=50000, power-law in-degrees 16..512 (E about
2.8M), K=8 Bessel, cutoff 6" (synthetic, seeded), the largest of the method's workloads.
Metric: edges per second of the step (higher is better).  The line also reports
edges/s of each pass on its own (forward and backward of the step's workload, the
force-training double backward, and the N=4096 uvw workload), the roofline of the
whole step (the slower of its FP32 work, tensor-core work and compulsory HBM bytes
at the peaks) and of its dominant kernel, and the peak workspace.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

N > 1 runs under torchrun: every rank processes its own independent graph (weak
scaling, no data-path collective); the time is the max over ranks.  Rank 0 prints one
JSON line.  `--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from equivariant_gnn_tensor_dst_b200 import workloads  # noqa: E402

METRIC = "TP-conv edges/sec fwd/bwd/double-bwd; % of roofline; peak workspace bytes"
UNIT = "edges/s"
CFG = 4                                             # the step's workload (edge scaling, uvw)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SM count x FP32 lanes x FMA x max clock
L2_FLUSH_BYTES = 256 << 20                          # > 126 MB L2
TF32_PER_BF16 = 1.1 / 2.25                          # nominal dense TF32 / BF16 tensor rates
SPLIT_MMAS = 3                                      # 3xTF32: three TF32 products per fp32 product
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per step for a kernel category
# of the step's workload, from an ncu capture of the current kernels on the N=8000 resize of
# the workload, scaled by its edge ratio (2 800 256 / 433 220); profiles/
# edge_scaling_N8000_dram_traffic.md.
TRAFFIC_BYTES_PER_STEP = {
    "uvw_receiver_backward": 10.98e9,
    # the receiver state, source state and contraction kernels have changed since that
    # capture (radial split of the 16-channel paths, per-tile product width): no figure
    "uvw_receiver_state": None,
    "uvw_source_state": None,
    "channel_gemm": None,
}


def measured_peaks():
    """Peaks measured on this machine (MEASURED_PEAKS.json), else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "source": "of measured (MEASURED_PEAKS.json: bf16 burst; the step keeps the SM clock at max)"}
    except (OSError, ValueError, KeyError):
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "source": "of fallback (6.65 TB/s, 1.59 PFLOP/s bf16 burst)"}


def _workload_config(c, g, passes="forward + backward (x, pos, W)"):
    return {"workload": c.name, "nodes": int(g.n_nodes), "edges": int(g.n_edges), "irreps": c.irreps_in,
            "sh_lmax": c.sh_lmax, "mode": c.mode, "radial": f"{c.radial} K={c.num_basis} r_c={c.r_cut}",
            "pass": passes, "l2": "flushed between timed steps"}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_over_ranks(total_ms, edges, device=None):
    """Max of the timed milliseconds and sum of the processed edges over all ranks
    (identity on a single rank).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(total_ms), float(edges)
    dev = device if device is not None else torch.device("cpu")
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e = torch.tensor([float(edges)], dtype=torch.float64, device=dev)
    dist.all_reduce(e, op=dist.ReduceOp.SUM)
    return float(t.item()), float(e.item())


# ---------------------------------------------------------------------------
# algorithmic operation counts (per edge and per node), from the plan's paths
# ---------------------------------------------------------------------------

def flop_model(plan):
    """Per-edge and per-node operation counts of each kernel category, from the plan's
    paths (FMA = 2 flop).  Only the work the streaming evaluation has to do is counted,
    not the materialised per-edge weights it avoids."""
    K = plan.num_basis
    f = dict(state=0, recv=0, src=0, state_tan=0, src_tan=0, gemm_node=0, gemm_fwd_node=0, gemm_dbl_node=0,
             gemm_node_bytes=0, uvu_fwd=0, uvu_recv=0, uvu_gradw=0, uvu_src=0)
    for p in plan.paths():
        ri, ro = 2 * p["l_in"] + 1, 2 * p["l_out"] + 1
        nnz, ci, co = p["nnz"], p["c_in"], p["c_out"]
        # uvu (channelwise, no state): w = phi A per channel, coupling, w * C into m (eqs. 7, 17);
        # receiver adjoint h = m_bar . C, phi_bar, Y_bar; weight gradient phi (m_bar . C);
        # source adjoint w * adj(C)
        f["uvu_fwd"] += 2 * ci * (K + nnz + ro)
        f["uvu_recv"] += 2 * ci * (2 * nnz + 2 * ro + 2 * K)
        f["uvu_gradw"] += 2 * ci * (nnz + ro + K)
        f["uvu_src"] += 2 * ci * (K + nnz + ro)
        f["state"] += 2 * ci * (nnz + K * ro)              # eq. 32 coupling + eq. 33 outer product
        f["recv"] += 2 * ci * (2 * nnz + 2 * K * ro)       # coupling, phi_bar, T_bar, Y_bar
        f["src"] += 2 * co * (nnz + K * ri)                # adjoint coupling + source state
        # tangents along pos_dot (double backward, gg_pos alone): coupling with Y and Y_dot,
        # outer products with phi and phi_dot, on each side
        f["state_tan"] += 2 * ci * (2 * nnz + 2 * K * ro)
        f["src_tan"] += 2 * co * (2 * nnz + 2 * K * ri)
        # S A, m_bar A^T (receiver side); X A^T, x^T X (source side, which also gives A_bar)
        f["gemm_node"] += 2 * K * ci * co * (2 * ro + 2 * ri)
        f["gemm_fwd_node"] += 2 * K * ci * co * ro
        # double backward: grad_W = S_dot^T m_bar, grad_x = X' A^T
        f["gemm_dbl_node"] += 2 * K * ci * co * (ro + ri)
        # fp32 operand bytes of the four channel contractions of a forward+backward step:
        # m = S A (read S, write m), S_bar = m_bar A^T (read m_bar, write S_bar),
        # x_bar = X A^T (read X, write x_bar), A_bar = x^T X (read x, X); the weights stay
        # in L2.
        f["gemm_node_bytes"] += 4 * (2 * ro * K * ci + 2 * ro * co + 2 * ri * K * co + 2 * ri * ci)
    return f


def pass_counts(plan, N, E, which):
    """Algorithmic FP32 (SIMT) flops, tensor-core flops and compulsory HBM bytes of one
    pass ("fwd", "bwd" with x, pos and W gradients, "fwd+bwd", or "dbl": the force-
    training double backward with gg_pos alone, returning grad_x and grad_W).
    Compulsory bytes: every input read once and every output written once (x, pos, the
    graph, A, upstream gradients and tangents; results)."""
    f = flop_model(plan)
    din, dout, nw = plan.dim_in, plan.dim_out, plan.num_basis * plan.weight_cols
    uvu = plan.mode == "uvu"
    graph = 4 * (N + 1) + 4 * E
    tgraph = 4 * (N + 1) + 8 * E
    fwd = dict(simt=E * (f["uvu_fwd"] if uvu else f["state"]), tc=0 if uvu else N * f["gemm_fwd_node"],
               bytes=4 * (N * din + 3 * N + nw + N * dout) + graph)
    bwd = dict(simt=E * ((f["uvu_recv"] + f["uvu_gradw"] + f["uvu_src"]) if uvu else (f["recv"] + f["src"])),
               # backward contractions: S_bar = m_bar A^T (receiver), x_bar = X A^T, A_bar = x^T X
               tc=0 if uvu else N * (f["gemm_node"] - f["gemm_fwd_node"]),
               bytes=4 * (N * din + 3 * N + nw + N * dout) + graph + tgraph + 4 * (N * din + 3 * N + nw))
    dbl = dict(simt=E * (f["state_tan"] + f["src_tan"]), tc=N * f["gemm_dbl_node"],
               bytes=4 * (N * din + 3 * N + nw + N * dout + 3 * N + N * din + nw) + graph + tgraph)
    if which == "fwd":
        return fwd
    if which == "bwd":
        return bwd
    if which == "dbl":
        return dbl
    both = dict(simt=fwd["simt"] + bwd["simt"], tc=fwd["tc"] + bwd["tc"],
                bytes=bwd["bytes"] + 4 * N * dout)   # the forward adds only its output
    return both


def step_roofline(counts, ms, peaks):
    """T_roof = max(F_simt / P_fp32, F_tc / P_tc, B_comp / BW_hbm) against the measured
    time; P_tc for fp32 products is three TF32 products at the nominal TF32/BF16 ratio of
    the measured BF16 peak."""
    tc_peak = peaks["bf16"] * TF32_PER_BF16 / SPLIT_MMAS
    t = {"fp32_alu": counts["simt"] / (FP32_PEAK_TFLOPS * 1e12),
         "tensor_3xtf32": counts["tc"] / (tc_peak * 1e12),
         "hbm": counts["bytes"] / (peaks["hbm_gbs"] * 1e9)}
    bound = max(t, key=t.get)
    t_roof = t[bound]
    return {"bound": bound, "t_roof_ms": round(t_roof * 1e3, 4), "t_measured_ms": round(ms, 4),
            "frac": round(t_roof / (ms / 1e3), 4), "simt_gflop": round(counts["simt"] / 1e9, 3),
            "tc_gflop": round(counts["tc"] / 1e9, 3), "compulsory_mb": round(counts["bytes"] / 1e6, 2),
            "peaks": {"fp32_tflops": round(FP32_PEAK_TFLOPS, 1), "tc_tflops": round(tc_peak, 1),
                      "hbm_gbs": peaks["hbm_gbs"]}}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------

def run_native(args):
    import torch

    from equivariant_gnn_tensor_dst_b200 import binding

    world, rank, local = _dist()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c = workloads.CONFIGS[args.cfg]
    plan = binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                        c.r_min, c.r_max)
    g, rng = workloads.make_graph(c, n_nodes=args.nodes, seed=1000 + args.cfg + 7919 * rank)
    N, E = g.n_nodes, g.n_edges
    x_h = workloads.normal(rng, (N, plan.dim_in))
    W_h = workloads.weights(rng, c.num_basis, plan.fan_in_per_column())
    go_h = workloads.normal(rng, (N, plan.dim_out))

    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    x, pos, row_ptr, src, W, gout = t(x_h), t(g.pos), t(g.row_ptr), t(g.src), t(W_h), t(go_h)
    t_ptr, t_eid, t_dst = binding.tpconv_csr_transpose(row_ptr, src, N)
    out = torch.empty(N, plan.dim_out, device=dev)
    gx = torch.empty(N, plan.dim_in, device=dev)
    gp = torch.empty(N, 3, device=dev)
    gw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
    ws_bytes = plan.workspace_bytes(N, E, binding.PASS_FORWARD | binding.PASS_BACKWARD)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    mem0 = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    ws = binding.workspace(ws_bytes, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        binding.tpconv_forward(plan, x, pos, row_ptr, src, W, out=out, ws=ws, stream=stream)
        binding.tpconv_backward(plan, x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, gout, ws=ws,
                                outputs=(gx, gp, gw), stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    peak_delta = torch.cuda.max_memory_allocated(dev) - mem0

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    # enough records for every launch scope of the timed steps (a scope that finds the pool
    # full is counted but not timed)
    binding.tpconv_profile_begin(8192 + 4096 * args.steps)
    for k in range(args.steps):
        flush.zero_()
        starts[k].record(stream)
        step()
        ends[k].record(stream)
    torch.cuda.synchronize()
    prof = binding.tpconv_profile_end()
    barrier()
    clocks = sampler.stop()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms, edges_all = reduce_over_ranks(total_ms, E, dev)
    ms_step = total_ms / args.steps
    value = edges_all * args.steps / (total_ms / 1e3)

    # a bounded wait inside a tensor-core kernel that gave up skips that launch's work: a
    # timed region that set the device error word is not a measurement
    dev_err = binding.tpconv_device_error()
    if dev_err != 0:
        raise SystemExit(f"device error word {dev_err} set during the timed region: no measurement")

    # live roofline of every kernel category (CUDA events over the timed region)
    fm = flop_model(plan)
    algo = {"uvw_receiver_state": fm["state"] * E, "uvw_receiver_backward": fm["recv"] * E,
            "uvw_source_state": fm["src"] * E, "channel_gemm": fm["gemm_node"] * N,
            "uvu_forward": fm["uvu_fwd"] * E, "uvu_receiver_backward": fm["uvu_recv"] * E,
            "uvu_weight_gradient": fm["uvu_gradw"] * E, "uvu_source_backward": fm["uvu_src"] * E}
    peaks = measured_peaks()
    tc_peak = peaks["bf16"] * TF32_PER_BF16 / SPLIT_MMAS
    kern = {k: v for k, v in prof.items() if v[1] > 0}
    gpu_launches = int(sum(v[1] for v in kern.values()))
    timed_ms = sum(v[0] for v in kern.values())
    rooflines = {}
    for k, (ms, n) in kern.items():
        if k not in algo or ms <= 0:
            continue
        ach = algo[k] / (ms / args.steps / 1e3) / 1e12
        if k == "channel_gemm":
            # the channel contractions are bound by the tensor cores (fp32 products from three
            # TF32 products); their compulsory bytes are a small part of the step's
            rl = {"bound": "tensor", "achieved": round(ach, 3), "peak": round(tc_peak, 1), "unit": "TFLOP/s",
                  "peak_note": f"fp32 products via 3xTF32: bf16 x {TF32_PER_BF16:.3f} (nominal TF32/BF16) "
                               f"/ {SPLIT_MMAS}, bf16 {peaks['source']}"}
        else:
            rl = {"bound": "alu", "achieved": round(ach, 3), "peak": round(FP32_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
                  "peak_note": "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1965 MHz"}
        rl["algorithmic_per_step"] = {"flop": algo[k]}
        rl["frac"] = round(rl["achieved"] / rl["peak"], 4)
        headline = args.cfg == CFG and args.nodes is None
        tb = TRAFFIC_BYTES_PER_STEP.get(k) if headline else None
        rl["traffic"] = round(tb) if tb else None
        if tb:
            rl["traffic_note"] = ("DRAM bytes per step (all launches of the category), ncu capture of the N=8000 "
                                  "resize scaled by the edge ratio")
        rooflines[k] = rl
    dom = max(rooflines, key=lambda k: kern[k][0]) if rooflines else None
    roofline = dict(rooflines[dom], kernel=dom) if dom else None
    breakdown = {k: {"ms_per_step": round(v[0] / args.steps, 4), "launches_per_step": v[1] / args.steps,
                     "share": round(v[0] / timed_ms, 4) if timed_ms else None} for k, v in kern.items()}
    total_algo = sum(v for k, v in algo.items() if k in kern)
    step_roof = step_roofline(pass_counts(plan, N, E, "fwd+bwd"), ms_step, peaks)

    # each pass on its own: forward and backward of this workload, the force-training double
    # backward, and the N=4096 uvw workload's forward and backward
    passes = None
    if not args.no_passes and rank == 0:
        passes = {"this_workload": time_passes(plan, c, N, E, dict(x=x, pos=pos, row_ptr=row_ptr, src=src, W=W,
                                                                   gout=gout, views=(t_ptr, t_eid, t_dst)),
                                               ws, flush, args, peaks, ("fwd", "bwd"))}
        for cfg in (5, 2):
            if cfg != args.cfg:
                passes[f"workload_{cfg}"] = time_workload(cfg, dev, flush, args, peaks)
        err2 = binding.tpconv_device_error()
        if err2 != 0:
            raise SystemExit(f"device error word {err2} set while timing the passes: no measurement")

    # end-to-end through the public API: pinned host inputs in, results out, every step
    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
        hx, hp, hr, hs, hw, hg = pin(x_h), pin(g.pos), pin(g.row_ptr), pin(g.src), pin(W_h), pin(go_h)
        ho, hgx, hgp, hgw = (torch.empty(tuple(a.shape), dtype=a.dtype).pin_memory() for a in (out, gx, gp, gw))
        d_in = [torch.empty_like(a, device=dev) for a in (hx, hp, hr, hs, hw, hg)]
        bi = sum(a.numel() * a.element_size() for a in (hx, hp, hr, hs, hw, hg))
        bo = sum(a.numel() * a.element_size() for a in (ho, hgx, hgp, hgw))
        ne2e = max(3, min(args.steps, 30))

        def e2e_step():
            for d, h in zip(d_in, (hx, hp, hr, hs, hw, hg)):
                d.copy_(h, non_blocking=True)
            xx, pp, rr, ss, WW, GG = d_in
            tp, te, td = binding.tpconv_csr_transpose(rr, ss, N, stream=stream)
            o = binding.tpconv_forward(plan, xx, pp, rr, ss, WW, ws=ws, stream=stream)
            a, b, cc = binding.tpconv_backward(plan, xx, pp, rr, ss, tp, te, td, WW, GG, ws=ws, stream=stream)
            for h, d in zip((ho, hgx, hgp, hgw), (o, a, b, cc)):
                h.copy_(d, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(ne2e):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize()
        e_ms, _ = reduce_over_ranks(s0.elapsed_time(s1), E, dev)
        e2e = {"value": round(edges_all * ne2e / (e_ms / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": int(bi),
               "d2h_bytes_per_step": int(bo), "steps": ne2e,
               "includes": "H2D of x, pos, CSR, W, grad_out; source-view build; forward; backward; "
                           "D2H of out, grad_x, grad_pos, grad_W"}

    extras = run_extras(args, dev, flush) if (args.extras and rank == 0) else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": _workload_config(c, g), "impl": "native",
                "roofline": roofline, "step_roofline": step_roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": gpu_launches,
                "gpu_launches_per_step": gpu_launches / args.steps, "clocks": clocks,
                "workspace_bytes": {"declared": int(ws_bytes), "peak_alloc_delta": int(peak_delta)},
                "device_error_word": 0,
                "step_algorithmic_tflop": round(total_algo / 1e12, 4),
                "step_tflops_achieved": round(total_algo / (ms_step / 1e3) / 1e12, 3),
                "breakdown": breakdown, "rooflines": rooflines, "passes": passes}
        if extras is not None:
            line["extras"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# further workloads (opt-in): every pass of the method on its own workload
# ---------------------------------------------------------------------------

def _timed(fn, flush, steps, warmup):
    import torch
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / steps


def _scalar_mask(c, dim_out):
    mask = np.zeros(dim_out, np.float32)
    off = 0
    for tok in c.irreps_out.split("+"):
        mul, ir = tok.split("x")
        l = int(ir[:-1])
        if l == 0 and ir[-1] == "e":
            mask[off:off + int(mul)] = 1.0
        off += int(mul) * (2 * l + 1)
    return mask


def time_passes(plan, c, N, E, t, ws, flush, args, peaks, which):
    """CUDA-event time, edges/s and step roofline of each pass in `which` on resident
    inputs t (dict of device tensors).  "dbl" is the force-training double backward:
    m_bar = 1 on every scalar output channel, gg_pos = 2 (pos_bar + F_ref) from a first
    backward, outputs grad_x and grad_W."""
    import torch

    from equivariant_gnn_tensor_dst_b200 import binding
    dev = t["x"].device
    steps, warm = max(5, min(args.steps, 20)), 3
    o = torch.empty(N, plan.dim_out, device=dev)
    gx = torch.empty(N, plan.dim_in, device=dev)
    gp = torch.empty(N, 3, device=dev)
    gw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
    rec = {}
    for name in which:
        if name == "fwd":
            fn = lambda: binding.tpconv_forward(plan, t["x"], t["pos"], t["row_ptr"], t["src"], t["W"],  # noqa: E731
                                                out=o, ws=ws)
        elif name == "bwd":
            fn = lambda: binding.tpconv_backward(plan, t["x"], t["pos"], t["row_ptr"], t["src"],  # noqa: E731
                                                 *t["views"], t["W"], t["gout"], ws=ws, outputs=(gx, gp, gw))
        else:
            mbar = torch.from_numpy(np.tile(_scalar_mask(c, plan.dim_out), (N, 1))).to(dev)
            F_ref = torch.from_numpy(workloads.normal(np.random.default_rng(1000 + c.cfg + 1), (N, 3))).to(dev)
            binding.tpconv_backward(plan, t["x"], t["pos"], t["row_ptr"], t["src"], *t["views"], t["W"], mbar,
                                    ws=ws, outputs=(None, gp, None))
            gg = torch.mul(torch.add(gp, F_ref), 2.0)      # d loss / d pos_bar
            fn = lambda: binding.tpconv_double_backward(plan, t["x"], t["pos"], t["row_ptr"], t["src"],  # noqa: E731
                                                        *t["views"], t["W"], mbar, gg_pos=gg, ws=ws,
                                                        outputs=(gx, gw, None))
        ms = _timed(fn, flush, steps, warm)
        key = {"fwd": "forward", "bwd": "backward", "dbl": "double_backward"}[name]
        rec[key] = {"ms": round(ms, 4), "edges_per_s": round(E / ms * 1e3, 1),
                    "roofline": step_roofline(pass_counts(plan, N, E, name), ms, peaks)}
    return rec


def time_workload(cfg, dev, flush, args, peaks):
    """Every pass of workload `cfg` (its own graph and inputs) with time_passes."""
    import torch

    from equivariant_gnn_tensor_dst_b200 import binding
    c = workloads.CONFIGS[cfg]
    plan = binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                        c.r_min, c.r_max)
    g, rng = workloads.make_graph(c)
    N, E = g.n_nodes, g.n_edges
    tt = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    t = dict(x=tt(workloads.normal(rng, (N, plan.dim_in))),
             W=tt(workloads.weights(rng, c.num_basis, plan.fan_in_per_column())),
             gout=tt(workloads.normal(rng, (N, plan.dim_out))), pos=tt(g.pos), row_ptr=tt(g.row_ptr),
             src=tt(g.src))
    t["views"] = binding.tpconv_csr_transpose(t["row_ptr"], t["src"], N)
    wsb = plan.workspace_bytes(N, E)
    ws = binding.workspace(wsb, dev)
    rec = {"workload": c.name, "nodes": N, "edges": E, "workspace_bytes": int(wsb)}
    rec.update(time_passes(plan, c, N, E, t, ws, flush, args, peaks, c.passes))
    del ws, t
    torch.cuda.empty_cache()
    return rec


def run_extras(args, dev, flush):
    """Per-pass edges/s on every workload of the method (forward, backward, double
    backward; uvw and uvu; fixed and power-law degrees)."""
    import torch

    from equivariant_gnn_tensor_dst_b200 import binding
    out = {}
    steps, warm = max(5, min(args.steps, 20)), 3
    for cfg in args.extras_cfgs:
        c = workloads.CONFIGS[cfg]
        t0 = time.time()
        plan = binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                            c.r_min, c.r_max)
        g, rng = workloads.make_graph(c)
        N, E = g.n_nodes, g.n_edges
        tt = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
        x = tt(workloads.normal(rng, (N, plan.dim_in)))
        W = tt(workloads.weights(rng, c.num_basis, plan.fan_in_per_column()))
        go = tt(workloads.normal(rng, (N, plan.dim_out)))
        pos, rp, src = tt(g.pos), tt(g.row_ptr), tt(g.src)
        views = binding.tpconv_csr_transpose(rp, src, N)
        ws = binding.workspace(plan.workspace_bytes(N, E), dev)
        o = torch.empty(N, plan.dim_out, device=dev)
        gx = torch.empty(N, plan.dim_in, device=dev)
        gp = torch.empty(N, 3, device=dev)
        gw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
        fwd = lambda: binding.tpconv_forward(plan, x, pos, rp, src, W, out=o, ws=ws)  # noqa: E731
        bwd = lambda: binding.tpconv_backward(plan, x, pos, rp, src, *views, W, go, ws=ws,  # noqa: E731
                                              outputs=(gx, gp, gw))
        rec = {"workload": c.name, "nodes": N, "edges": E, "mode": c.mode,
               "graph_seconds": round(time.time() - t0, 1)}
        ms_f = _timed(fwd, flush, steps, warm)
        ms_b = _timed(bwd, flush, steps, warm)
        rec.update({"forward_ms": round(ms_f, 4), "forward_edges_per_s": round(E / ms_f * 1e3, 1),
                    "backward_ms": round(ms_b, 4), "backward_edges_per_s": round(E / ms_b * 1e3, 1)})
        # the same passes on the graph renumbered in Morton order of the positions (locality
        # of the x and m_bar row gathers; results are the renumbered results)
        perm = binding.tpconv_spatial_order(pos)
        rp2, src2, _ = binding.tpconv_permute_graph(rp, src, perm)
        x2, pos2, go2 = (binding.tpconv_gather_rows(a, perm) for a in (x, pos, go))
        views2 = binding.tpconv_csr_transpose(rp2, src2, N)
        fwd2 = lambda: binding.tpconv_forward(plan, x2, pos2, rp2, src2, W, out=o, ws=ws)  # noqa: E731
        bwd2 = lambda: binding.tpconv_backward(plan, x2, pos2, rp2, src2, *views2, W, go2, ws=ws,  # noqa: E731
                                               outputs=(gx, gp, gw))
        ms_f2, ms_b2 = _timed(fwd2, flush, steps, warm), _timed(bwd2, flush, steps, warm)
        rec["spatial_order"] = {"forward_ms": round(ms_f2, 4), "backward_ms": round(ms_b2, 4),
                                "forward_backward_edges_per_s": round(E / (ms_f2 + ms_b2) * 1e3, 1)}
        del x2, pos2, go2, views2, rp2, src2
        # the embedded-input interface: phi_e and Y_e given per edge, phi_bar and Y_bar returned
        Ye = tt(workloads.normal(rng, (E, (c.sh_lmax + 1) ** 2)))
        pe = tt(workloads.normal(rng, (E, c.num_basis)))
        gphi = torch.empty(E, c.num_basis, device=dev)
        gY = torch.empty(E, (c.sh_lmax + 1) ** 2, device=dev)
        fe = lambda: binding.tpconv_forward_embedded(plan, x, Ye, pe, rp, src, W, out=o, ws=ws)  # noqa: E731
        be = lambda: binding.tpconv_backward_embedded(plan, x, Ye, pe, rp, src, *views, W, go, ws=ws,  # noqa: E731
                                                      outputs=(gx, gw, gphi, gY))
        ms_ef, ms_eb = _timed(fe, flush, steps, warm), _timed(be, flush, steps, warm)
        rec["embedded_interface"] = {"forward_ms": round(ms_ef, 4), "backward_ms": round(ms_eb, 4),
                                     "forward_backward_edges_per_s": round(E / (ms_ef + ms_eb) * 1e3, 1)}
        if c.mode == "uvw":
            # the optional TF32 and BF16 contraction modes (1e-2 accuracy class), reported separately
            plan.set_math(binding.MATH_TF32)
            ms_tf, ms_tb = _timed(fwd, flush, steps, warm), _timed(bwd, flush, steps, warm)
            plan.set_math(binding.MATH_BF16)
            ms_bf, ms_bb = _timed(fwd, flush, steps, warm), _timed(bwd, flush, steps, warm)
            plan.set_math(binding.MATH_FP32)
            rec["tf32_contractions"] = {"forward_ms": round(ms_tf, 4), "backward_ms": round(ms_tb, 4),
                                        "forward_backward_edges_per_s": round(E / (ms_tf + ms_tb) * 1e3, 1)}
            rec["bf16_contractions"] = {"forward_ms": round(ms_bf, 4), "backward_ms": round(ms_bb, 4),
                                        "forward_backward_edges_per_s": round(E / (ms_bf + ms_bb) * 1e3, 1)}
        if "dbl" in c.passes:
            # force training: energy = sum of scalar outputs, F = -dE/dpos, loss |F - F_ref|^2,
            # then d loss / d(W, x) by the double backward
            mbar = tt(np.tile(_scalar_mask(c, plan.dim_out), (N, 1)))
            F_ref = tt(workloads.normal(rng, (N, 3)))
            dx = torch.empty(N, plan.dim_in, device=dev)
            dw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
            gg = torch.empty(N, 3, device=dev)

            def force_step():
                binding.tpconv_forward(plan, x, pos, rp, src, W, out=o, ws=ws)
                binding.tpconv_backward(plan, x, pos, rp, src, *views, W, mbar, ws=ws, outputs=(None, gp, None))
                torch.mul(torch.add(gp, F_ref), 2.0, out=gg)   # d loss / d pos_bar = 2 (pos_bar + F_ref)
                binding.tpconv_double_backward(plan, x, pos, rp, src, *views, W, mbar, gg_pos=gg, ws=ws,
                                               outputs=(dx, dw, None))

            def dbl_only():
                binding.tpconv_double_backward(plan, x, pos, rp, src, *views, W, mbar, gg_pos=gg, ws=ws,
                                               outputs=(dx, dw, None))
            dpos = torch.empty(N, 3, device=dev)

            def dbl_with_pos():
                # the same double backward also returning d loss / d pos (positions learned)
                binding.tpconv_double_backward(plan, x, pos, rp, src, *views, W, mbar, gg_pos=gg, ws=ws,
                                               need_pos=True, outputs=(dx, dw, None, dpos))
            ms_s = _timed(force_step, flush, steps, warm)
            ms_d = _timed(dbl_only, flush, steps, warm)
            ms_dp = _timed(dbl_with_pos, flush, steps, warm)
            # the tangent receiver kernel of d loss / d pos against the derived FP32 peak: with
            # gg_pos alone it does the receiver backward's arithmetic twice (values and tangents)
            binding.tpconv_profile_begin(8192)
            for _ in range(5):
                flush.zero_()
                dbl_with_pos()
            prof = binding.tpconv_profile_end()
            tan_ms = prof["receiver_backward_tangent"][0] / 5
            if c.mode == "uvw" and tan_ms > 0:
                flop = 2 * flop_model(plan)["recv"] * E
                ach = flop / (tan_ms / 1e3) / 1e12
                rec["position_tangent_kernel"] = {
                    "ms": round(tan_ms, 4), "flop": int(flop), "bound": "alu", "achieved": round(ach, 3),
                    "peak": round(FP32_PEAK_TFLOPS, 1), "unit": "TFLOP/s", "frac": round(ach / FP32_PEAK_TFLOPS, 4),
                    "breakdown_ms": {k: round(v[0] / 5, 4) for k, v in prof.items() if v[1] > 0}}
            rec.update({"double_backward_ms": round(ms_d, 4),
                        "double_backward_edges_per_s": round(E / ms_d * 1e3, 1),
                        "double_backward_with_pos_ms": round(ms_dp, 4),
                        "double_backward_with_pos_edges_per_s": round(E / ms_dp * 1e3, 1),
                        "force_step_ms": round(ms_s, 4), "force_step_edges_per_s": round(E / ms_s * 1e3, 1)})
        out[str(cfg)] = rec
        del ws
        torch.cuda.empty_cache()
    return out


def run_profiles(args):
    """Forward, backward and full double backward (all three tangents) of every feature
    profile (workloads.profile_configs) on one fixed graph; one JSON line."""
    import torch

    from equivariant_gnn_tensor_dst_b200 import binding
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    steps, warm = max(5, min(args.steps, 20)), 3
    profs = workloads.profile_configs()
    g, _ = workloads.make_graph(profs[0], seed=1100)
    N, E = g.n_nodes, g.n_edges
    tt = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    pos, rp, src = tt(g.pos), tt(g.row_ptr), tt(g.src)
    views = binding.tpconv_csr_transpose(rp, src, N)
    rows = []
    for c in profs:
        plan = binding.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, c.radial, c.num_basis, c.r_cut,
                            c.r_min, c.r_max)
        rng = np.random.default_rng(2000 + c.cfg)
        x = tt(workloads.normal(rng, (N, plan.dim_in)))
        W = tt(workloads.weights(rng, c.num_basis, plan.fan_in_per_column()))
        go = tt(workloads.normal(rng, (N, plan.dim_out)))
        ggx, ggp = tt(workloads.normal(rng, (N, plan.dim_in))), tt(workloads.normal(rng, (N, 3)))
        ggw = tt(workloads.normal(rng, (plan.num_basis, plan.weight_cols)))
        wsb = plan.workspace_bytes(N, E)
        ws = binding.workspace(wsb, dev)
        o = torch.empty(N, plan.dim_out, device=dev)
        gx, gp = torch.empty(N, plan.dim_in, device=dev), torch.empty(N, 3, device=dev)
        gw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
        dx, dg = torch.empty(N, plan.dim_in, device=dev), torch.empty(N, plan.dim_out, device=dev)
        dw = torch.empty(plan.num_basis, plan.weight_cols, device=dev)
        fwd = lambda: binding.tpconv_forward(plan, x, pos, rp, src, W, out=o, ws=ws)  # noqa: E731
        bwd = lambda: binding.tpconv_backward(plan, x, pos, rp, src, *views, W, go, ws=ws,  # noqa: E731
                                              outputs=(gx, gp, gw))
        dbl = lambda: binding.tpconv_double_backward(plan, x, pos, rp, src, *views, W, go, gg_x=ggx,  # noqa: E731
                                                     gg_pos=ggp, gg_W=ggw, ws=ws, outputs=(dx, dw, dg))
        rec = {"profile": c.name, "mode": c.mode, "paths": len(plan.paths()), "workspace_bytes": wsb}
        for name, fn in (("forward", fwd), ("backward", bwd), ("double_backward", dbl)):
            ms = _timed(fn, flush, steps, warm)
            rec[name + "_ms"] = round(ms, 4)
            rec[name + "_edges_per_s"] = round(E / ms * 1e3, 1)
        rows.append(rec)
        del ws
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "edges/s per pass on the feature-profile grid", "unit": "edges/s",
                      "graph": {"nodes": N, "edges": E, "knn": profs[0].k, "density": profs[0].density},
                      "l2": "flushed between timed calls", "steps": steps, "profiles": rows}), flush=True)


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def _oracle_sample(seconds_target):
    from oracle import conv, radial
    c = workloads.CONFIGS[CFG]
    rs = radial.RadialSpec(c.radial, c.num_basis, c.r_cut, c.r_min, c.r_max)
    op = conv.make_plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.mode, rs)
    g, rng = workloads.make_graph(c)
    x = workloads.normal(rng, (g.n_nodes, op.dim_in))
    W = workloads.weights(rng, c.num_basis, op.fan_in_per_column())
    go = workloads.normal(rng, (g.n_nodes, op.dim_out))
    rp = g.row_ptr.astype(np.int64)

    def run(n_recv):
        edges = np.arange(rp[0], rp[n_recv])
        t0, c0 = time.perf_counter(), time.process_time()
        conv.forward(op, x, g.pos, g.row_ptr, g.src, W, edges=edges)
        conv.backward(op, x, g.pos, g.row_ptr, g.src, W, go, edges=edges)
        dt = time.perf_counter() - t0
        run.cores = (time.process_time() - c0) / max(dt, 1e-9)   # CPU seconds per wall second
        return dt, edges.size

    # warm up, calibrate on a small sample, then size the sample for the target duration
    run(2)
    t_small, _ = run(16)
    n_recv = int(np.clip(16 * seconds_target / max(t_small, 1e-3), 8, g.n_nodes))
    return run, n_recv, g


def _threads_available():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        return 1


def cpu_baseline(seconds):
    run, n_recv, g = _oracle_sample(seconds)
    dt, ne = run(n_recv)
    # cores = the CPU time the oracle's process used per second of wall time (its numpy
    # kernels use a thread pool only in some steps), not the size of that pool
    return {"value": round(ne / dt, 2), "unit": UNIT, "cores": round(run.cores, 2), "kind": "oracle",
            "threads_available": _threads_available(),
            "sample": f"forward+backward over the first {n_recv} receivers ({ne} edges) of the workload",
            "seconds": round(dt, 2)}


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return
    run, n_recv, g = _oracle_sample(args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        run(min(n_recv, 8))
    times, cores, ne = [], [], 0
    for _ in range(args.steps):
        dt, ne = run(n_recv)
        times.append(dt)
        cores.append(run.cores)
    total = sum(times)
    value = ne * args.steps / total
    c = workloads.CONFIGS[CFG]
    cpu = {"value": round(value, 2), "unit": UNIT, "cores": round(statistics.median(cores), 2), "kind": "oracle",
           "threads_available": _threads_available(),
           "sample": f"each step: forward+backward over the first {n_recv} receivers ({ne} edges)"}
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _workload_config(c, g), "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-passes", action="store_true",
                    help="skip timing each pass on its own (this workload, force training, N=4096 uvw)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--extras", action="store_true",
                    help="also time every pass on the other workloads (adds ~1-2 minutes)")
    ap.add_argument("--extras-cfgs", type=int, nargs="*", default=[2, 3, 5, 4])
    ap.add_argument("--cfg", type=int, default=CFG, choices=sorted(workloads.CONFIGS),
                    help="workload of the timed step (default: the edge-scaling uvw workload)")
    ap.add_argument("--nodes", type=int, default=None,
                    help="resize the workload (same density and degree); for profiling small cases")
    ap.add_argument("--profiles", action="store_true",
                    help="instead of the timed step: every pass of the 25 feature profiles on one graph")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.profiles:
        run_profiles(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
