"""Benchmark: CGTP convolution edges/s (forward + backward) on the molecular
batch workload (256 graphs x 30 atoms, L_in = L_out = 2, harmonics l <= 4,
mult 128), one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cgtp,reference}]

A timed step is one pass of the convolution over the resident batch:
harmonics + forward (one kernel), backward over sources (grad_x, grad_W and
the per-edge harmonic gradient), the harmonic Jacobian (grad_edge_vec) and
the per-atom forces.  The neighbour list and the radial weight network run
in a second timed loop ("pipeline": positions -> graph -> weights -> forward
-> backward -> radial backward -> forces) reported beside the headline.
Every rank processes its own batch (weak scaling, no collective on the data
path); timing uses CUDA events on the launching stream, between a barrier
and a device synchronisation, and the slowest rank's time.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from equivariant_mlip_tensor_b200 import synthetic  # noqa: E402

METRIC = "CGTP conv edges/s (fwd+bwd) at L=2, mult=128; % of HBM roofline"
UNIT = "edges/s"
WORKLOAD = ("molecules: 256 graphs x 30 atoms uniform in an 8 A cube (0.9 A rejection), cutoff 5 A, "
            "one CSR over the batch; x 128x(l=0..2), harmonics l<=4, outputs l<=2, 19 paths, "
            "weights from the radial network; energy = sum of l=0 outputs")


def _load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def _cores():
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling (every 200 ms) during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- measured DRAM traffic
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of each kernel
# family at the molecules workload (97 480 edges), from an ncu capture
# (profiles/conv_molecules_traffic.md), with a hash of the kernel sources it
# was taken on: traffic is reported only while the sources are unchanged.
KERNEL_HEADERS = ("common.cuh", "conv_common.cuh", "sh.cuh", "structure.h", "vec2.cuh", "launch.h")
MEASURED_TRAFFIC = {
    "conv_fwd": {"bytes": 1023000000, "n_edges": 97480, "sources": ("conv_fwd.cu", "conv_fwd_kernel.cuh") + KERNEL_HEADERS,
                 "sha256_16": "35f85179426a59a3"},
    "conv_bwd": {"bytes": 2044400000, "n_edges": 97480, "sources": ("conv_bwd.cu", "conv_bwd_kernel.cuh") + KERNEL_HEADERS,
                 "sha256_16": "002201829139bfa5"},
}


def measured_traffic(kernel, n_edges):
    """Measured DRAM bytes of one launch scaled to n_edges, or None when the
    kernel's sources changed since the capture."""
    import hashlib
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None:
        return None
    m = hashlib.sha256()
    for name in rec["sources"]:
        with open(os.path.join(ROOT, "equivariant_mlip_tensor_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    if m.hexdigest()[:16] != rec["sha256_16"]:
        return None
    return rec["bytes"] * n_edges / rec["n_edges"]


# ---------------------------------------------------------------- algorithmic bytes
def conv_bytes(n, E, P, u, ni, ns, no):
    """Algorithmic bytes of one forward and one backward launch (fp32/int32),
    what the method must move:
      forward  4 [E P u (W) + 4E (edge vectors, sources) + (N+1) (row offsets)
                  + N u ni (x) + N u no (out)]
      backward 4 [2 E P u (W read, grad_W written) + N u (2 ni + no) (x, grad_x,
                  grad_out) + 8E (edge vectors, grad_edge_vec, CSC edge and
                  destination lists) + 2 (N+1) (CSR and CSC offsets)]
    The backward's harmonic-gradient partials (a workspace of this design) are
    not counted; partials_bytes gives them separately."""
    fwd = 4 * (E * P * u + 4 * E + (n + 1) + n * u * ni + n * u * no)
    bwd = 4 * (2 * E * P * u + n * u * (2 * ni + no) + 8 * E + 2 * (n + 1))
    return fwd, bwd


def partials_bytes(E, ns, slices):
    """Bytes of the backward's harmonic-gradient partials (written by the
    chunks, read by the Jacobian epilogue)."""
    return 4 * 2 * slices * E * ns


def structural_counts(li, ls, lo):
    """(T entries, CG entries, sum of 2l3+1) over the paths, from the real-basis
    selection rules (|m3| in {|m1|+|m2|, ||m1|-|m2||}, parity of the negative m's)."""
    def ok(l1, l2, l3, a, b, c):
        if abs(c) not in (abs(a) + abs(b), abs(abs(a) - abs(b))):
            return False
        return ((a < 0) + (b < 0) + (c < 0)) % 2 == (l1 + l2 + l3) % 2
    nT = nnz = osum = 0
    for l1 in range(li + 1):
        for l2 in range(ls + 1):
            for l3 in range(abs(l1 - l2), min(l1 + l2, lo) + 1):
                osum += 2 * l3 + 1
                for a in range(-l1, l1 + 1):
                    for c in range(-l3, l3 + 1):
                        k = sum(ok(l1, l2, l3, a, b, c) for b in range(-l2, l2 + 1))
                        nnz += k
                        nT += k > 0
    return nT, nnz, osum


def conv_flops(E, u, nT, nnz, no_sum, P):
    """Algorithmic FLOPs (FMA = 2) with the per-edge T factorisation:
    forward sum_p(|T^p| + (2l3+1)) per channel-edge; backward t, grad_W, s,
    grad_x and the channel dot products (4 |T| + 2 sum(2l3+1)) per
    channel-edge plus nnz per lane."""
    fwd = 2 * E * u * (nT + no_sum)
    bwd = 2 * E * u * (3 * nT + 2 * no_sum) + 2 * E * nnz * (u // 4)
    return fwd, bwd


# ---------------------------------------------------------------- reference arm / CPU baseline
def oracle_step(w, n_graphs_sample, threads):
    """The oracle's fwd + bwd + forces over the first n_graphs_sample graphs."""
    from oracle import conv as oconv
    from oracle import graph as ograph
    from oracle import radial as oradial
    n = n_graphs_sample * w.graph_size
    pos, gid = w.pos[:n], w.graph_id[:n]
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    o = ograph.neighbour_list(pos, w.rc, None, gid)
    Wo = oradial.radial_forward(o["edge_vec"], w.W1, w.W2, w.rc, w.n_paths, w.mult)
    chunk = max(256, -(-o["col"].size // threads))
    t0 = time.perf_counter()
    oconv.conv_forward(o["row_ptr"], o["col"], o["edge_vec"], w.x[:n], Wo, *L, threads=threads, chunk=chunk)
    _, _, gr = oconv.conv_backward(o["row_ptr"], o["col"], o["edge_vec"], w.x[:n], Wo, w.grad_out[:n], *L,
                                   threads=threads, chunk=chunk)
    oconv.edge_forces(o["row_ptr"], o["col"], gr, n)
    dt = time.perf_counter() - t0
    return o["col"].size, dt


def cpu_baseline(w, budget_s=15.0):
    threads = _cores()
    E1, dt1 = oracle_step(w, 2, threads)
    rate = E1 / dt1
    n_g = int(max(2, min(w.pos.shape[0] // w.graph_size, budget_s * rate / (E1 / 2))))
    E, dt = oracle_step(w, n_g, threads)
    return {"value": E / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {n_g} of 256 molecules ({E} edges): fp64 NumPy forward + backward + forces, "
                      f"{threads} threads over edge chunks, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = synthetic.molecules()
    threads = _cores()
    n_g = 4
    times, edges = [], 0
    for _ in range(args.warmup):
        oracle_step(w, n_g, threads)
    for _ in range(args.steps):
        E, dt = oracle_step(w, n_g, threads)
        times.append(dt)
        edges = E
    ms = 1e3 * float(np.mean(times))
    value = edges / (ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": f"first {n_g} molecules per step ({edges} edges)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"first {n_g} of 256 molecules per step ({edges} edges)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- every workload size
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x FP32 lanes x FMA x max clock


def _time_ms(torch, fn, reps):
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def config_table(torch, api, dev, hbm, reps=20):
    """Forward and backward of every workload (sizes of the pages' configurations),
    each against the HBM and FP32 rooflines, plus the edge-free tensor product."""
    rows = []
    for name in ("tiny", "bulk", "bulk_large", "molecules"):
        w = synthetic.WORKLOADS[name]()
        L = (w.lmax_in, w.lmax_sh, w.lmax_out)
        n, u = w.n_nodes, w.mult
        ni, ns, no = (L[0] + 1) ** 2, (L[1] + 1) ** 2, (L[2] + 1) ** 2
        gp = None
        if w.graph_id is not None:
            gp = torch.from_numpy(np.arange(0, n + 1, w.graph_size, dtype=np.int32)).to(dev)
        g = api.build_graph(torch.from_numpy(w.pos).to(dev), w.rc, box=w.box, graph_ptr=gp)
        plan = api.Plan(*L, u)
        E, P = g.n_edges, plan.n_paths
        W = plan.radial_forward(g.edge_vec, w.rc, torch.from_numpy(w.W1).to(dev), torch.from_numpy(w.W2).to(dev))
        x = torch.from_numpy(w.x).to(dev)
        go = torch.from_numpy(w.grad_out).to(dev)
        out = torch.empty((n, no, u), dtype=torch.float32, device=dev)
        gx = torch.empty((n, ni, u), dtype=torch.float32, device=dev)
        gw = torch.empty_like(W)
        gr = torch.empty((E, 3), dtype=torch.float32, device=dev)
        F = torch.empty((n, 3), dtype=torch.float32, device=dev)
        ws_bytes = plan.conv_backward_workspace_bytes(E)
        ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device=dev)
        k = max(3, reps if E < 500_000 else reps // 4)
        t_f = _time_ms(torch, lambda: plan.conv_forward(g, x, W, out=out), k)
        t_b = _time_ms(torch, lambda: plan.conv_backward(g, x, W, go, grad_x=gx, grad_w=gw, grad_edge_vec=gr,
                                                          workspace=ws), k)
        t_frc = _time_ms(torch, lambda: api.forces(g, gr, out=F), k)
        slices = max(1, int(ws_bytes // (4 * E * ns))) if E else 1
        b_f, b_b = conv_bytes(n, E, P, u, ni, ns, no)
        nT, nnz, no_sum = structural_counts(*L)
        f_f, f_b = conv_flops(E, u, nT, nnz, no_sum, P)
        rows.append({"workload": name, "L": list(L), "mult": u, "n_nodes": n, "n_edges": E, "paths": P,
                     "fwd_ms": t_f, "bwd_ms": t_b, "forces_ms": t_frc,
                     "edges_per_s_fwd_bwd": E / ((t_f + t_b) / 1e3),
                     "hbm_frac": {"fwd": b_f / (t_f / 1e3) / 1e9 / hbm, "bwd": b_b / (t_b / 1e3) / 1e9 / hbm},
                     "fp32_frac": {"fwd": f_f / (t_f / 1e3) / 1e12 / FP32_PEAK_TFLOPS,
                                   "bwd": f_b / (t_b / 1e3) / 1e12 / FP32_PEAK_TFLOPS}})
        if name == "molecules":
            # weights shared by every path (path stride 0): one weight row per edge
            wsh = torch.randn((E, u), device=dev)
            gws = torch.empty_like(wsh)
            t_sf = _time_ms(torch, lambda: plan.conv_forward_shared(g, x, wsh, out=out), k)
            t_sb = _time_ms(torch, lambda: plan.conv_backward_shared(g, x, wsh, go, workspace=ws), k)
            b_sf = 4 * (E * u + n * ni * u + n * no * u + 4 * E + (n + 1))
            b_sb = 4 * (2 * E * u + n * u * (2 * ni + no) + 8 * E + 2 * (n + 1))
            rows.append({"workload": "molecules, weights shared by every path (path stride 0)",
                         "L": list(L), "mult": u, "n_edges": E, "fwd_ms": t_sf, "bwd_ms": t_sb,
                         "edges_per_s_fwd_bwd": E / ((t_sf + t_sb) / 1e3),
                         "hbm_frac": {"fwd": b_sf / (t_sf / 1e3) / 1e9 / hbm, "bwd": b_sb / (t_sb / 1e3) / 1e9 / hbm},
                         "fp32_frac": {"fwd": f_f / (t_sf / 1e3) / 1e12 / FP32_PEAK_TFLOPS,
                                       "bwd": f_b / (t_sb / 1e3) / 1e12 / FP32_PEAK_TFLOPS}})
            del wsh, gws
            # double backward (adjoint of the backward) with all three cotangents
            ggx, ggw, ggr = torch.randn_like(x), torch.randn_like(W), torch.randn((E, 3), device=dev)
            dws = torch.empty(plan.conv_double_backward_workspace_bytes(E) // 4 + 64, dtype=torch.float32,
                              device=dev)
            t_d = _time_ms(torch, lambda: plan.conv_double_backward(g, x, W, go, gg_x=ggx, gg_w=ggw,
                                                                    gg_edge_vec=ggr, workspace=dws), k)
            # algorithmic bytes: read x, gg_x, W, gg_w, grad_out, gg_r, edge vectors; write d_x, d_W,
            # d_grad_out, d_edge_vec
            b_d = 4 * (3 * E * P * u + 3 * n * ni * u + 2 * n * no * u + 9 * E + 2 * (n + 1) + 2 * E)
            # an atomic-free schedule reads W and gg_w twice (once by destination for d grad_out,
            # once by source for d x and d W) and writes d W once: 5 weight-sized transfers
            b_s = b_d + 4 * 2 * E * P * u
            rows.append({"workload": "molecules double backward (adjoint of the backward, all cotangents)",
                         "L": list(L), "mult": u, "n_edges": E, "ms": t_d, "edges_per_s": E / (t_d / 1e3),
                         "hbm_frac": b_d / (t_d / 1e3) / 1e9 / hbm,
                         "hbm_frac_of_atomic_free_schedule": b_s / (t_d / 1e3) / 1e9 / hbm,
                         "launches": "fused: d grad_out by one forward pass (chunks by l3), d x / d W / edge terms "
                                     "by one source-centric pass (chunks by l1), one Jacobian-and-Hessian epilogue"})
            del ggx, ggw, ggr, dws
            # fully connected (uvw) forward, 128 output channels: per-path messages, then one
            # tensor-core GEMM per l3 block
            v = 128
            mix = torch.randn((P, u, v), device=dev) / u ** 0.5
            uws = torch.empty(plan.uvw_forward_workspace_bytes(n, v) // 4 + 64, dtype=torch.float32, device=dev)
            uout = torch.empty((n, no, v), dtype=torch.float32, device=dev)
            t_u = _time_ms(torch, lambda: plan.uvw_forward(g, x, W, mix, out=uout, workspace=uws), k)
            rows_p = no_sum  # sum over paths of 2 l3 + 1
            f_gemm = 2.0 * n * rows_p * u * v
            b_u = 4 * (E * P * u + n * ni * u + n * no * v + P * u * v + 4 * E + (n + 1))
            rows.append({"workload": "molecules fully connected (uvw) forward, 128 -> 128 channels per path",
                         "L": list(L), "mult": u, "mult_out": v, "n_edges": E, "ms": t_u,
                         "edges_per_s": E / (t_u / 1e3), "hbm_frac": b_u / (t_u / 1e3) / 1e9 / hbm,
                         "mixing_gemm_flops": f_gemm,
                         "mixing_tflops_if_whole_call": f_gemm / (t_u / 1e3) / 1e12})
            ugo = torch.randn((n, no, v), device=dev)
            bws = torch.empty(plan.uvw_backward_workspace_bytes(n, E, v) // 4 + 64, dtype=torch.float32, device=dev)
            t_ub = _time_ms(torch, lambda: plan.uvw_backward(g, x, W, mix, ugo, workspace=bws), k)
            rows.append({"workload": "molecules fully connected (uvw) backward (grad_x, grad_W, grad_mix, grad_r)",
                         "L": list(L), "mult": u, "mult_out": v, "n_edges": E, "ms": t_ub,
                         "edges_per_s": E / (t_ub / 1e3),
                         "tensor_gemm_flops": 2 * f_gemm,
                         "launches": "2 tensor-core GEMM sets (per-path output gradients, mixing gradient), "
                                     "per-path backward chunks, per-path forward recompute, harmonic Jacobian"})
            del mix, uws, uout, ugo, bws
        del W, gw, out, gx, gr, F, ws, x, go, g
        torch.cuda.empty_cache()
    t = synthetic.tp_batch()
    L = (t.lmax_in, t.lmax_sh, t.lmax_out)
    plan = api.Plan(*L, t.mult)
    xs, ys, ws_, gz = (torch.from_numpy(a).to(dev) for a in (t.x, t.y, t.w, t.grad_z))
    z = torch.empty_like(gz)
    t_f = _time_ms(torch, lambda: plan.tp_forward(xs, ys, ws_, out=z), reps)
    t_b = _time_ms(torch, lambda: plan.tp_backward(xs, ys, ws_, gz), reps)
    B, u = t.x.shape[0], t.mult
    ni, ns, no = (L[0] + 1) ** 2, (L[1] + 1) ** 2, (L[2] + 1) ** 2
    b_f = 4 * (B * u * (ni + ns + no) + t.w.size)
    b_b = 4 * (B * u * (2 * ni + 2 * ns + no) + 2 * t.w.size)
    rows.append({"workload": "tp_batch (edge-free tensor product)", "L": list(L), "mult": u, "batch": B,
                 "fwd_ms": t_f, "bwd_ms": t_b, "pairs_per_s_fwd_bwd": B / ((t_f + t_b) / 1e3),
                 "hbm_frac": {"fwd": b_f / (t_f / 1e3) / 1e9 / hbm, "bwd": b_b / (t_b / 1e3) / 1e9 / hbm}})
    # CP-decomposed product of the same pairs, rank 40 (factors N(0,1)/sqrt(R): the
    # kernels' cost does not depend on their values)
    R = 40
    gen = torch.Generator(device="cpu").manual_seed(7)
    fA, fB, fC = (torch.randn(sh, generator=gen).div_(R ** 0.5).to(dev) for sh in ((no, R), (ni, R), (ns, R)))
    zc = torch.empty_like(gz)
    t_cf = _time_ms(torch, lambda: plan.cp_forward(fA, fB, fC, xs, ys, out=zc), reps)
    t_cb = _time_ms(torch, lambda: plan.cp_backward(fA, fB, fC, xs, ys, gz, want_factors=False), reps)
    t_cg = _time_ms(torch, lambda: plan.cp_backward(fA, fB, fC, xs, ys, gz), reps)
    items = B * u
    fl_f = items * (2 * R * (ni + ns + no) + R)
    fl_b = items * (2 * R * (ni + ns + no) + 2 * R * (ni + ns) + 3 * R)
    fl_g = fl_b + items * 2 * R * (ni + ns + no)
    rows.append({"workload": "cp_batch (CP-decomposed product of the tp_batch pairs, rank 40)", "L": list(L),
                 "mult": u, "batch": B, "rank": R, "fwd_ms": t_cf, "bwd_ms": t_cb, "bwd_with_factor_grads_ms": t_cg,
                 "pairs_per_s_fwd_bwd": B / ((t_cf + t_cb) / 1e3),
                 "hbm_frac": {"fwd": 4 * items * (ni + ns + no) / (t_cf / 1e3) / 1e9 / hbm,
                              "bwd": 4 * items * (2 * ni + 2 * ns + no) / (t_cb / 1e3) / 1e9 / hbm},
                 "fp32_frac": {"fwd": fl_f / (t_cf / 1e3) / 1e12 / FP32_PEAK_TFLOPS,
                               "bwd": fl_b / (t_cb / 1e3) / 1e12 / FP32_PEAK_TFLOPS,
                               "bwd_with_factor_grads": fl_g / (t_cg / 1e3) / 1e12 / FP32_PEAK_TFLOPS}})
    return rows


def run_op(args):
    """A short loop of one operation at the molecules workload, for profiling
    (ncu launch lists): 'uvw' (fully connected forward), 'uvw_bwd' (its
    backward), 'double' (double backward) or 'cp' (CP-decomposed product of
    the tp_batch pairs, rank 40, forward and backward with factor gradients)."""
    import torch

    from equivariant_mlip_tensor_b200 import api
    dev = torch.device("cuda", 0)
    w = synthetic.molecules(n_graphs=args.graphs)
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n, u = w.n_nodes, w.mult
    gp = torch.from_numpy(np.arange(0, n + 1, w.graph_size, dtype=np.int32)).to(dev)
    g = api.build_graph(torch.from_numpy(w.pos).to(dev), w.rc, graph_ptr=gp)
    plan = api.Plan(*L, u)
    W = plan.radial_forward(g.edge_vec, w.rc, torch.from_numpy(w.W1).to(dev), torch.from_numpy(w.W2).to(dev))
    x = torch.from_numpy(w.x).to(dev)
    go = torch.from_numpy(w.grad_out).to(dev)
    if args.op == "uvw":
        mix = torch.randn((plan.n_paths, u, 128), device=dev) / u ** 0.5
        fn = lambda: plan.uvw_forward(g, x, W, mix)
    elif args.op == "uvw_bwd":
        mix = torch.randn((plan.n_paths, u, 128), device=dev) / u ** 0.5
        ugo = torch.randn((n, (L[2] + 1) ** 2, 128), device=dev)
        fn = lambda: plan.uvw_backward(g, x, W, mix, ugo)
    elif args.op == "cp":
        t = synthetic.tp_batch()
        Lt = (t.lmax_in, t.lmax_sh, t.lmax_out)
        tplan = api.Plan(*Lt, t.mult)
        xs, ys, gz = (torch.from_numpy(a).to(dev) for a in (t.x, t.y, t.grad_z))
        d1, d2, d3 = ((l + 1) ** 2 for l in Lt)
        fA, fB, fC = (torch.randn((d, 40), device=dev) / 40 ** 0.5 for d in (d3, d1, d2))

        def fn():
            tplan.cp_forward(fA, fB, fC, xs, ys)
            tplan.cp_backward(fA, fB, fC, xs, ys, gz)
    else:
        ggx, ggw, ggr = torch.randn_like(x), torch.randn_like(W), torch.randn((g.n_edges, 3), device=dev)
        fn = lambda: plan.conv_double_backward(g, x, W, go, gg_x=ggx, gg_w=ggw, gg_edge_vec=ggr)
    ms = _time_ms(torch, fn, args.steps)
    print(json.dumps({"op": args.op, "n_edges": g.n_edges, "ms": ms}), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch

    from equivariant_mlip_tensor_b200 import api

    from equivariant_mlip_tensor_b200.ranks import Group, Ranks, shard_seed, throughput

    ranks = Ranks.from_env()
    world, rank, local = ranks.world, ranks.rank, ranks.local
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = Group(ranks, "nccl", dev)
    barrier, max_over_ranks = group.barrier, group.max

    w = synthetic.molecules(seed=shard_seed(4, rank), n_graphs=args.graphs)
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    n, u = w.n_nodes, w.mult
    ni, ns, no = (L[0] + 1) ** 2, (L[1] + 1) ** 2, (L[2] + 1) ** 2
    stream = torch.cuda.current_stream()

    # resident inputs
    pos = torch.from_numpy(w.pos).to(dev)
    gp = torch.from_numpy(np.arange(0, n + 1, w.graph_size, dtype=np.int32)).to(dev)
    x = torch.from_numpy(w.x).to(dev)
    go = torch.from_numpy(w.grad_out).to(dev)
    W1 = torch.from_numpy(w.W1).to(dev)
    W2 = torch.from_numpy(w.W2).to(dev)
    plan = api.Plan(*L, u)
    g = api.build_graph(pos, w.rc, graph_ptr=gp, max_edges=int(1.25 * 13 * n))
    E, P = g.n_edges, plan.n_paths
    W = plan.radial_forward(g.edge_vec, w.rc, W1, W2)
    out = torch.empty((n, no, u), dtype=torch.float32, device=dev)
    gx = torch.empty((n, ni, u), dtype=torch.float32, device=dev)
    gw = torch.empty((E, P, u), dtype=torch.float32, device=dev)
    gr = torch.empty((E, 3), dtype=torch.float32, device=dev)
    F = torch.empty((n, 3), dtype=torch.float32, device=dev)
    ws_bytes = plan.conv_backward_workspace_bytes(E)
    ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device=dev)

    def conv_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plan.conv_forward(g, x, W, out=out)
        if ev is not None:
            ev[1].record(stream)
        plan.conv_backward(g, x, W, go, grad_x=gx, grad_w=gw, grad_edge_vec=gr, workspace=ws)
        if ev is not None:
            ev[2].record(stream)
        api.forces(g, gr, out=F)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        conv_step()
    torch.cuda.synchronize()

    # per-kernel breakdown (separate loop, events between launches)
    nb = min(args.steps, 200)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nb)]
    barrier()
    torch.cuda.synchronize()
    for k in range(nb):
        conv_step(evs[k])
    torch.cuda.synchronize()
    t_fwd = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_bwd = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    t_frc = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))

    # headline timed region: exactly K steps between barrier + synchronize
    clocks = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0.record(stream)
    for _ in range(args.steps):
        conv_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    value, ms_step = throughput(group, float(E), e0.elapsed_time(e1) / 1e3, args.steps)
    edges_all = group.sum(float(E))

    if args.conv_only:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                              "ms_per_step": ms_step, "n_edges": E,
                              "kernels_ms": {"conv_fwd": t_fwd, "conv_bwd_incl_sh_jacobian": t_bwd,
                                             "forces": t_frc}}), flush=True)
        group.close()
        return 0

    # pipeline: positions -> graph -> radial weights -> conv -> radial backward -> forces
    ne_dev = torch.empty(1, dtype=torch.int32, device=dev)
    cap = g.col.numel() if g.col.numel() >= E else E
    bufs = dict(row_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
                col=torch.empty(cap, dtype=torch.int32, device=dev),
                ev=torch.empty((cap, 3), dtype=torch.float32, device=dev),
                csc_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
                ce=torch.empty(cap, dtype=torch.int32, device=dev),
                cd=torch.empty(cap, dtype=torch.int32, device=dev))
    from equivariant_mlip_tensor_b200._lib import call
    import ctypes

    def P_(t):
        return ctypes.c_void_p(t.data_ptr())

    gpipe = api.Graph(n, E, bufs["row_ptr"], bufs["col"][:E], bufs["ev"][:E], bufs["csc_ptr"],
                      bufs["ce"][:E], bufs["cd"][:E])
    Wp = torch.empty_like(W)

    def pipeline_step(evp=None, pos_t=pos, x_t=x, go_t=go):
        if evp is not None:
            evp[0].record(stream)
        call("cgtp_graph_build", P_(pos_t), n, ctypes.c_float(0.0), ctypes.c_float(w.rc), P_(gp), gp.numel() - 1,
             P_(bufs["row_ptr"]), P_(bufs["col"]), P_(bufs["ev"]), P_(bufs["csc_ptr"]), P_(bufs["ce"]),
             P_(bufs["cd"]), cap, P_(ne_dev), ctypes.c_void_p(stream.cuda_stream))
        if evp is not None:
            evp[1].record(stream)
        plan.radial_forward(gpipe.edge_vec, w.rc, W1, W2, out=Wp)
        if evp is not None:
            evp[2].record(stream)
        plan.conv_forward(gpipe, x_t, Wp, out=out)
        plan.conv_backward(gpipe, x_t, Wp, go_t, grad_x=gx, grad_w=gw, grad_edge_vec=gr, workspace=ws)
        if evp is not None:
            evp[3].record(stream)
        plan.radial_backward(gpipe.edge_vec, w.rc, W1, W2, gw, gr)
        if evp is not None:
            evp[4].record(stream)
        api.forces(gpipe, gr, out=F)
        if evp is not None:
            evp[5].record(stream)

    for _ in range(3):
        pipeline_step()
    torch.cuda.synchronize()
    assert int(ne_dev.item()) == E
    npipe = max(20, min(args.steps // 4, 500))
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(npipe)]
    barrier()
    torch.cuda.synchronize()
    for k in range(npipe):
        pipeline_step(evp[k])
    torch.cuda.synchronize()
    seg = np.mean([[e[i].elapsed_time(e[i + 1]) for i in range(5)] for e in evp], axis=0)
    t_pipe = max_over_ranks(float(np.mean([e[0].elapsed_time(e[5]) for e in evp])) / 1e3)
    pipe_value = edges_all / t_pipe

    # e2e through the public API with host buffers: pinned positions, features and
    # output gradient in; forces out, every step.  The next step's inputs are copied
    # on a second stream into the other of two device buffer sets while the
    # current step computes (events order each copy after the step that last read
    # its set, and each step after its own copy).
    pos_h = torch.from_numpy(w.pos).pin_memory()
    x_h = torch.from_numpy(w.x).pin_memory()
    go_h = torch.from_numpy(w.grad_out).pin_memory()
    F_h = torch.empty((n, 3), dtype=torch.float32).pin_memory()
    sets = [dict(pos=torch.empty_like(pos), x=torch.empty_like(x), go=torch.empty_like(go)) for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        sb = sets[k % 2]
        with torch.cuda.stream(copy_stream):
            if k >= 2:
                copy_stream.wait_event(free[k % 2])
            sb["pos"].copy_(pos_h, non_blocking=True)
            sb["x"].copy_(x_h, non_blocking=True)
            sb["go"].copy_(go_h, non_blocking=True)
            ready[k % 2].record(copy_stream)
        stream.wait_event(ready[k % 2])
        pipeline_step(pos_t=sb["pos"], x_t=sb["x"], go_t=sb["go"])
        free[k % 2].record(stream)
        F_h.copy_(F, non_blocking=True)

    for k in range(3):
        e2e_step(k)
    torch.cuda.synchronize()
    ne2e = max(10, min(args.steps // 10, 200))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    a0.record(stream)
    copy_stream.wait_event(a0)  # the first copy starts inside the timed region
    for k in range(ne2e):
        e2e_step(k)
    a1.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(a0.elapsed_time(a1) / 1e3 / ne2e)
    h2d = pos_h.numel() * 4 + x_h.numel() * 4 + go_h.numel() * 4
    d2h = F_h.numel() * 4

    # roofline of the dominant kernel (the backward)
    hbm, peak_kind = _load_peaks()
    slices = max(1, int(ws_bytes // (4 * E * ns))) if E else 1
    b_fwd, b_bwd = conv_bytes(n, E, P, u, ni, ns, no)
    dominant = "conv_bwd" if t_bwd >= t_fwd else "conv_fwd"
    b_dom, t_dom = (b_bwd, t_bwd) if dominant == "conv_bwd" else (b_fwd, t_fwd)
    achieved = b_dom / (t_dom / 1e3) / 1e9
    traffic = measured_traffic(dominant, E)
    nT, nnz, no_sum = structural_counts(*L)
    f_fwd, f_bwd = conv_flops(E, u, nT, nnz, no_sum, P)
    step_bytes = b_fwd + b_bwd + 4 * (E * 3 * 2 + n * 3 + 2 * (n + 1) + 2 * E)
    if rank != 0:
        group.close()
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded); weights from the radial network",
        "config": {"workload": WORKLOAD, "n_nodes": n, "n_edges": E, "paths": P, "mult": u,
                   "l2": "inputs larger than L2 (W is %.0f MB per rank, read twice per step)" % (E * P * u * 4 / 1e6),
                   "parallelism": f"independent batch per rank (dp{world})"},
        "gpu_launches": (3 + slices) * args.steps,  # forward, backward chunks, harmonic Jacobian, forces
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "peak_kind": peak_kind,
                     "alg_bytes_per_launch": b_dom,
                     "traffic_over_alg": traffic / b_dom if traffic else None,
                     "frac_with_partials": ((b_dom + (partials_bytes(E, ns, slices) if dominant == "conv_bwd" else 0))
                                            / (t_dom / 1e3) / 1e9 / hbm)},
        "kernels_ms": {"conv_fwd": t_fwd, "conv_bwd_incl_sh_jacobian": t_bwd, "forces": t_frc},
        "step_hbm_frac": (step_bytes / (ms_step / 1e3) / 1e9) / hbm,
        "fp32_tflops": {"conv_fwd": f_fwd / (t_fwd / 1e3) / 1e12, "conv_bwd": f_bwd / (t_bwd / 1e3) / 1e12},
        "pipeline": {"value": pipe_value, "unit": UNIT, "ms_per_step": t_pipe * 1e3,
                     "stages_ms": {"graph": float(seg[0]), "radial_fwd": float(seg[1]),
                                   "conv_fwd_bwd": float(seg[2]), "radial_bwd": float(seg[3]),
                                   "forces": float(seg[4])}},
        "e2e": {"value": edges_all / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": "pinned host positions, features, output gradient -> graph, radial weights, conv fwd+bwd, "
                        "radial bwd, forces -> host forces; next step's copies overlap this step's compute"},
        "clocks": clk,
    }
    if rank == 0 and not args.no_configs:
        line["configs"] = config_table(torch, api, dev, hbm)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    group.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cgtp", "reference"], default="cgtp")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload table")
    ap.add_argument("--op", choices=["uvw", "uvw_bwd", "double", "cp"], default=None,
                    help="time one other operation alone (for profiling) instead of the benchmark")
    ap.add_argument("--graphs", type=int, default=256, help="molecules per rank (profiling uses fewer)")
    ap.add_argument("--conv-only", action="store_true",
                    help="time only the convolution step (no pipeline / e2e / CPU baseline); for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.op is not None:
        return run_op(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
