"""Benchmark of the edge message-passing step (energy + forces) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the seeded N=4096 diamond (8x8x8 conventional cells, sigma 0.02 A,
seed 2), cutoff 6 A (E = 647168 directed edges), C = 128, lmax = 3, three gated
residual layers, 8192-edge receiver-sorted cohorts.  One step = mp_energy_forces
on the frame's resident neighbour graph: forward (radial, rotate, SO(2) mixing,
rotate back, receiver sums, gates, readout) + backward + forces.  The
neighbour list build is timed on its own (nl_ms) and is part of the end-to-end
figure (e2e), not of the step.  Metric: edges/s = E / step time (whole job:
summed over replicas).

N > 1 (launched with torch.distributed.run, one rank per GPU; without it, with
--gpus N > 1, this script launches itself that way): every rank runs its own
replica of the frame (replicas only: weak scaling), timed between barriers, max
over ranks.

--impl reference times the float64 oracle (test infrastructure, CPU) on a
bounded sample of the same workload: the edges of the first receivers.
"""
from __future__ import annotations

import argparse
import gc
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "n4096_diamond"
METRIC = "edges/s fwd+force at N=4096 diamond (E~647k)"
L2_BYTES = 126 * 2 ** 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TF32_OVER_BF16 = 1.1 / 2.25     # nominal dense TF32 / BF16 tensor throughput on B200


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ distributed helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, backend_device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=backend_device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None:
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_dir: str | None = None):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join(out_dir or tempfile.gettempdir(), f"clocks_rank{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
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
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ the oracle arm
def oracle_sample(n_recv: int):
    """The oracle's energy + forces on the edges of the first n_recv receivers."""
    from oracle import model as omodel
    from oracle import nl as onl
    w = synth.workload(WORKLOAD)
    st = w.structure
    g = onl.brute_force(st.pos, st.box, w.spec.cutoff)
    e1 = int(g.recv_off[n_recv])
    sel = slice(0, e1)

    def run():
        return omodel.energy_forces(w.spec, w.weights, st.species, g.recv[sel], g.send[sel], g.r[sel],
                                    st.pos.shape[0])
    return run, e1, g.n_edges


def threads_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(n_recv: int = 48):
    run, e, _ = oracle_sample(n_recv)
    run()                       # warm caches / thread pools
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    return {"value": e / dt, "unit": "edges/s", "cores": threads_used(), "kind": "oracle",
            "sample": f"float64 oracle energy+forces over the {e} edges of the first {n_recv} receivers "
                      f"of the {WORKLOAD} frame (3 layers fwd + reverse mode), one run after one warm-up, "
                      f"{dt:.1f} s"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    n_recv = 32
    run, e, E = oracle_sample(n_recv)
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    dt = sum(times) / len(times)
    v = e / dt
    cores = threads_used()
    sample = (f"float64 oracle energy+forces over the {e} edges of the first {n_recv} receivers of the "
              f"{WORKLOAD} frame per step")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "edges/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "n_atoms": 4096, "n_edges": E, "sample_edges": e, "C": 128,
                       "lmax": 3, "layers": 3, "cohort_edges": 8192},
            "cpu_baseline": {"value": v, "unit": "edges/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ per-kernel HBM figures
# Algorithmic HBM bytes per step of each kernel family, for E edges, N atoms, C channels and
# T layers.  The first layer (degree-0 input) and the last (read through degree 0 only) run the
# receiver-centric kernels first_fwd / first_bwd / last_fwd / last_bwd; only the T - 2 layers
# between them run rotate_in, rotate_back_scatter, bwd_prep and bwd_edge.  Node rows gathered
# per edge (x of the sender, gS or the per-node products of the receiver; arrays of at most
# N*16*C floats that stay in L2) are not counted: their minimal traffic is one pass per layer.
def alg_bytes_step(name: str, C: int, T: int, E: int, N: int) -> float:
    row = 16 * C * 4                      # one [16][C] fp32 row
    d = 84 * 4                            # Wigner-D blocks of an edge
    d0 = 16 * 4                           # the m = 0 rows of the blocks
    mid = max(T - 2, 0)                   # layers between the first and the last
    last = 1 if T >= 2 else 0
    if name == "rotate_in":               # R row in; x~ hi/lo out
        return mid * E * (4 * C * 4 + 2 * row + d)
    if name == "bwd_prep":                # D in; g_y hi/lo out (y is kept from the forward: no x~)
        return mid * E * (2 * row + d)
    if name == "bwd_edge":                # y, g_x~, R, D in; dE/dR hi/lo out
        return mid * E * (2 * row + 4 * C * 4 + d + 2 * 4 * C * 4)
    if name == "rotate_back_scatter":     # y, D in
        return mid * E * (row + d)
    if name == "first_fwd":               # R[l=0], m = 0 rows of D in; Z out (per node)
        return E * (C * 4 + d0) + N * row
    if name == "first_bwd":               # R[l=0], D, r in; dE/dR[l=0] hi/lo out, g_r read-modify-write
        return E * (C * 4 + d + 12 + 2 * C * 4 + 24)
    if name == "last_fwd":                # R, m = 0 rows of D in; X out (per node)
        return last * (E * (4 * C * 4 + d0) + N * 4 * C * 4)
    if name == "last_bwd":                # R, D, r in; dE/dR hi/lo out, g_r and g_x read-modify-write
        return last * (E * (4 * C * 4 + d + 12 + 2 * 4 * C * 4 + 24) + N * 2 * row)
    if name == "radial_fwd":              # d in; R out (C columns in the first layer, 4C after): the fused network
        return E * (4 + C * 4) + (T - 1) * E * (4 + 4 * C * 4)
    if name == "radial_h2":               # d in; h2 hi/lo out
        return T * E * (4 + 2 * 64 * 4)
    if name == "radial_head":             # h2 hi/lo in; R out (C columns in the first layer, 4C after)
        return E * (2 * 64 * 4 + C * 4) + (T - 1) * E * (2 * 64 * 4 + 4 * C * 4)
    if name == "radial_head_bwd":         # dE/dR hi/lo in (C columns in the first layer); dE/dh2 out
        return E * (2 * C * 4 + 64 * 4) + (T - 1) * E * (2 * 4 * C * 4 + 64 * 4)
    if name == "radial_bwd":              # the fused network backward: dE/dR hi/lo (C columns in the first
        # layer, 4C after), d and the edge vector in; g_r read-modify-write
        return E * (2 * C * 4 + 4 + 12 + 2 * 12) + (T - 1) * E * (2 * 4 * C * 4 + 4 + 12 + 2 * 12)
    raise KeyError(name)


def mixing_flops_step(C: int, T: int, E: int) -> float:
    """Useful FP32 flops of the per-edge SO(2) mixings in one energy + force step: they run in the
    T - 2 layers between the first and the last (the end layers mix once per node); each mixes
    every edge twice, forward and backward transpose (the backward reads y kept from the forward),
    2 * 72 * C^2 flops each (the four m-blocks: 16 + 36 + 16 + 4 = 72 C^2 multiply-adds)."""
    return float(E) * 2 * C * C * 2 * 72 * max(T - 2, 0)


HBM_FAMILIES = ("rotate_in", "bwd_prep", "bwd_edge", "rotate_back_scatter", "first_fwd", "first_bwd", "last_fwd",
                "last_bwd", "radial_fwd", "radial_h2", "radial_head", "radial_head_bwd", "radial_bwd")


def hbm_fractions(fam, steps: int, E: int, N: int, C: int, T: int, hbm_gbs: float):
    out = {}
    for name in HBM_FAMILIES:
        if name not in fam or fam[name][0] <= 0:
            continue
        bytes_step = alg_bytes_step(name, C, T, E, N)
        ms = fam[name][0] / steps
        gbs = bytes_step / (ms * 1e-3) / 1e9
        out[name] = {"ms": round(ms, 3), "alg_bytes_per_step": int(bytes_step), "achieved_gbs": round(gbs, 1),
                     "frac_of_hbm": round(gbs / hbm_gbs, 3)}
    return out


# DRAM bytes per launch of the SO(2) mixing kernel (mean over one N=4096 step's 80 launches: 39
# forward launches of two cohorts and one of a single cohort, 39 backward launches of two cohorts and
# one of a single cohort), from ncu captures of the N=512 step's forward and backward two-cohort
# launches, which have the same shapes (profiles/kernels_n512_step.md; a single-cohort launch counted
# at half).  Valid only for the kernel source and the launch structure it was taken on: so2_tc.cuh
# and the marked per-edge product launch code of emp_lib.cu must hash to source_sha1, else the
# roofline's traffic is null.
SO2_TRAFFIC = {"source_sha1": "ddac4e4305648c3a9083e13e1778cad9ba2252c5", "bytes_per_launch": 379.0e6}


def so2_source_hash():
    import hashlib
    csrc = os.path.join(ROOT, "edge_message_passing_b200", "csrc")
    h = hashlib.sha1()
    so2 = os.path.join(csrc, "so2_tc.cuh")
    lib = os.path.join(csrc, "emp_lib.cu")
    if not (os.path.exists(so2) and os.path.exists(lib)):
        return None
    h.update(open(so2, "rb").read())
    text = open(lib).read()
    begin, end = "// [per-edge product launches: begin]", "// [per-edge product launches: end]"
    pos = 0
    while True:
        a = text.find(begin, pos)
        if a < 0:
            break
        b = text.find(end, a)
        if b < 0:
            return None
        h.update(text[a:b].encode())
        pos = b + len(end)
    return h.hexdigest()


def so2_traffic_per_launch():
    # the kernel and the launch structure (which cohorts each launch covers) must both be
    # those the counters were taken on
    ok = SO2_TRAFFIC["source_sha1"] and so2_source_hash() == SO2_TRAFFIC["source_sha1"]
    return SO2_TRAFFIC["bytes_per_launch"] if ok else None


# ------------------------------------------------------------------ the other seeded configs
def other_configs(emp, torch, stream, flush, hbm_gbs: float, steps: int = 10):
    """Edges/s and ns/atom of the energy + force call on the other seeded workloads (the
    same timing: CUDA events, L2 flushed between steps, neighbour graph resident), and
    the radial fold chain (forward + input gradient) against the HBM roofline."""
    out = {}

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush.fill_(1.0)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return sum(ts) / len(ts)

    for name in ("n64_diamond", "n512_diamond", "ternary_n2000"):
        w = synth.workload(name)
        st, spec = w.structure, w.spec
        model = emp.Model(spec, w.weights)
        pos = torch.from_numpy(st.pos).cuda()
        sp = torch.from_numpy(st.species).cuda()
        g = emp.nl_build(pos, st.box, spec.cutoff)
        efg = emp.EnergyForcesGraph(model, g, sp)
        fn = efg.replay
        how = "CUDA-graph replay"
        ms = timed(fn)
        N = st.pos.shape[0]
        out[name] = {"n_atoms": N, "n_edges": g.n_edges, "C": spec.C, "layers": spec.n_layers,
                     "ms_per_step": round(ms, 4), "edges_per_s": g.n_edges / (ms * 1e-3),
                     "ns_per_atom": ms * 1e6 / N, "timed": how}
        del model, g
    # the benchmark frame with the opt-in certified radial tables in place of the radial
    # network's hidden layers (an approximation, certified against float64; not the headline)
    w = synth.workload(WORKLOAD)
    st, spec = w.structure, w.spec
    model = emp.Model(spec, w.weights)
    n_pieces = model.radial_tables(1e-7)
    pos = torch.from_numpy(st.pos).cuda()
    sp = torch.from_numpy(st.species).cuda()
    g = emp.nl_build(pos, st.box, spec.cutoff)
    efg = emp.EnergyForcesGraph(model, g, sp)
    ms = timed(efg.replay)
    # the table kernels alone (event-timed in one eager call) against their HBM bytes
    emp.profile_enable(True)
    emp.mp_energy_forces(model, g, sp)
    torch.cuda.synchronize()
    fam = {n: emp.profile_read(n) for n in ("radial_h2", "radial_bwd")}
    emp.profile_enable(False)
    E, T = g.n_edges, spec.n_layers
    tab_bytes = {"radial_h2": T * E * (4 + 2 * 64 * 4), "radial_bwd": T * E * (4 + 64 * 4 + 12 + 2 * 12)}
    out[WORKLOAD + "_radial_tables"] = {
        "n_atoms": st.pos.shape[0], "n_edges": g.n_edges, "ms_per_step": round(ms, 4),
        "edges_per_s": g.n_edges / (ms * 1e-3), "table_pieces": n_pieces, "timed": "CUDA-graph replay",
        "table_kernels": {k: {"ms": round(v[0], 4), "alg_bytes": tab_bytes[k],
                              "frac_of_hbm": round(tab_bytes[k] / (v[0] * 1e-3) / 1e9 / hbm_gbs, 3)}
                          for k, v in fam.items()},
        "note": "opt-in certified Chebyshev tables (degree 10, tol 1e-7) for the radial hidden layers; an "
                "approximation, not the headline"}
    del efg
    model.radial_tables(0.0)
    # the same frame in the smallest workspace: the backward recomputes y cohort by cohort and no
    # [E, 16C] tensor is kept (the same bits as the headline step)
    efg = emp.EnergyForcesGraph(model, g, sp, compact=True)
    ms_c = timed(efg.replay)
    out[WORKLOAD + "_recompute_y"] = {
        "n_atoms": st.pos.shape[0], "n_edges": g.n_edges, "ms_per_step": round(ms_c, 4),
        "edges_per_s": g.n_edges / (ms_c * 1e-3), "workspace_bytes": int(efg.ws.numel()),
        "timed": "CUDA-graph replay"}
    del efg
    # the weight gradient of the energy (the training path), eager, on the same frame
    for _ in range(2):
        emp.mp_energy_weight_grad(model, g, sp)
    torch.cuda.synchronize()
    emp.profile_enable(True)
    ms_g = timed(lambda: emp.mp_energy_weight_grad(model, g, sp))
    red_ms = emp.profile_read("weight_grad")[0] / (steps + 3)
    blk_ms = emp.profile_read("wgrad_blocks")[0] / (steps + 3)
    emp.profile_enable(False)
    C = spec.C
    # FLOPs of the sums over edges and nodes: the middle layers' SO(2) blocks (3xTF32 products on the
    # tensor cores, with the transposes that make the edge index their K), and on SIMT the radial W3
    # (C or 4C rows), W2, W1 of every layer and the end layers' per-node W0 sums
    blk_flops = 2.0 * E * 72 * C * C * max(T - 2, 0)
    flops = (2.0 * E * 64 * (C + 4 * C * (T - 1)) + 2.0 * T * E * (64 * 64 + 64 * 8)
             + 2.0 * st.pos.shape[0] * (16 * C * C + 4 * C * C))
    clk = _sm_clock_mhz(torch)
    fp32_peak = 148 * 128 * 2 * clk * 1e6 / 1e12 if clk else None          # FMA lanes x 2 flops x SM clock
    rates = sorted(emp.tf32_mma_rate(20000) for _ in range(5))
    tf32_peak = rates[len(rates) // 2] / 3.0                                # 3xTF32: three products each
    out[WORKLOAD + "_weight_grad"] = {
        "ms_per_call": round(ms_g, 3), "edges_per_s": E / (ms_g * 1e-3), "timed": "eager call",
        "so2_block_sums": {"ms": round(blk_ms, 3), "flops": blk_flops,
                           "achieved_tflops": round(blk_flops / (blk_ms * 1e-3) / 1e12, 2) if blk_ms > 0 else None,
                           "bound": "tensor", "peak_tflops": round(tf32_peak, 1) if tf32_peak else None,
                           "frac": round(blk_flops / (blk_ms * 1e-3) / 1e12 / tf32_peak, 3) if tf32_peak and blk_ms > 0 else None,
                           "peak_note": "the measured 3xTF32 rate of the products (as for the mixing); the time includes the transposes"},
        "other_sums": {"ms": round(red_ms, 3), "flops": flops, "achieved_tflops": round(flops / (red_ms * 1e-3) / 1e12, 2),
                       "bound": "alu", "peak_tflops": round(fp32_peak, 1) if fp32_peak else None,
                       "frac": round(flops / (red_ms * 1e-3) / 1e12 / fp32_peak, 3) if fp32_peak else None,
                       "peak_note": "FP32 FMA: 148 SMs x 128 lanes x 2 flops x the SM clock read at the start"},
        "note": "energy, forces and dE/dW of every weight in one call"}
    del model, g
    ci = synth.chain_inputs()
    ch = emp.Chain(ci.U, ci.M)
    x, gk, gy = (torch.from_numpy(t).cuda() for t in (ci.x, ci.g_kc, ci.g_y0))
    E = x.shape[0]
    bufs = (torch.empty((E, 25), device="cuda"), torch.empty((E, 64), device="cuda"), torch.empty_like(x))
    ms = timed(lambda: emp.mp_radial_chain(ch, x, gk, gy, out=bufs))
    alg = E * (4 * 32 * 4 + 25 * 4 + 64 * 4) + E * (25 * 4 + 64 * 4 + 4 * 32 * 4)   # forward + input gradient
    gbs = alg / (ms * 1e-3) / 1e9
    out["radial_chain"] = {"rows": E, "ms": round(ms, 4), "alg_bytes": alg, "achieved_gbs": round(gbs, 1),
                           "frac_of_hbm": round(gbs / hbm_gbs, 3),
                           "note": "forward (x -> kc, y0) + input gradient (g_kc, g_y0 -> g_x) per call"}
    return out


def _sm_clock_mhz(torch):
    """Current SM clock of GPU 0 (nvidia-smi), or None."""
    try:
        outp = subprocess.run(["nvidia-smi", "--query-gpu=clocks.sm", "--format=csv,noheader,nounits", "-i",
                               str(torch.cuda.current_device())], capture_output=True, text=True, timeout=20).stdout
        return float(outp.strip().splitlines()[0])
    except Exception:
        return None


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    import edge_message_passing_b200 as emp

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()
    w = synth.workload(WORKLOAD)
    st, spec = w.structure, w.spec
    N = st.pos.shape[0]
    model = emp.Model(spec, w.weights)
    pos_h = torch.from_numpy(st.pos).pin_memory()
    sp_h = torch.from_numpy(st.species).pin_memory()
    pos = pos_h.cuda()
    sp = sp_h.cuda()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    # the step is mp_energy_forces on a resident neighbour graph (built once: the positions
    # are those of one frame); the neighbour list is timed on its own below
    g0 = emp.nl_build(pos, st.box, spec.cutoff)
    E = g0.n_edges
    for _ in range(max(args.warmup, 3)):
        emp.mp_energy_forces(model, g0, sp)
    torch.cuda.synchronize()
    efg = emp.EnergyForcesGraph(model, g0, sp)     # the step's library launches as one CUDA graph
    for _ in range(max(args.warmup, 3)):
        efg.replay()
    torch.cuda.synchronize()

    def nl_step(p, reuse):
        return emp.nl_build(p, st.box, spec.cutoff, reuse=reuse)

    # ---- device-resident timing: K steps, L2 flushed between steps (outside the events)
    def timed_steps(profile: bool):
        barrier(dev if ws > 1 else None)
        torch.cuda.synchronize()
        emp.profile_enable(profile)
        gc.collect()
        gc.disable()              # no collector pauses between the host calls of a step
        times = []
        for _ in range(args.steps):
            flush.fill_(1.0)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if profile:
                emp.mp_energy_forces(model, g0, sp)    # eager, with an event pair around every launch
            else:
                efg.replay()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        torch.cuda.synchronize()
        barrier(dev if ws > 1 else None)
        gc.enable()
        fam = {n: emp.profile_read(n) for n in emp.profile_names()} if profile else {}
        emp.profile_enable(False)
        return times, fam

    with ClockSampler(dev, args.clocks_dir) as clk:
        # let the sampler start polling before the timed steps (its start-up stalls the driver)
        for _ in range(2):
            efg.replay()
        torch.cuda.synchronize()
        time.sleep(1.0)
        times, _ = timed_steps(False)
        launches = efg.launches * len(times)
        # the same steps again, eagerly, with CUDA events recorded around every library launch
        # (on the launching stream) for the per-kernel times and the roofline
        ptimes, fam = timed_steps(True)
        # latency distribution of the graph-replayed step: at least 50 reps, L2 flushed between
        lat = []
        for _ in range(max(50, args.steps)):
            flush.fill_(1.0)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            efg.replay()
            b.record(stream)
            b.synchronize()
            lat.append(a.elapsed_time(b))
        # the tensor pipe's TF32 rate in the products' own form, under the same conditions
        # (a few warm-up launches, then ~0.5 s back to back: the sustained figure)
        for _ in range(3):
            emp.tf32_mma_rate(20000)
        rates = [emp.tf32_mma_rate(20000) for _ in range(40)]
    # neighbour list alone (cell list + sort + mirror), same frame
    gnl = None                    # own buffers: g0's are captured by the graph
    nl_times = []
    for k in range(args.steps + 1):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gnl = nl_step(pos, gnl)
        b.record(stream)
        b.synchronize()
        if k:
            nl_times.append(a.elapsed_time(b))
    ms_local = sum(times) / len(times)
    ms = reduce_max(ms_local, torch.device("cuda", dev))
    value = E * ws / (ms * 1e-3)
    # ---- end to end through the public API with host buffers (H2D positions + species, D2H energy + forces)
    e_h = torch.empty(1, dtype=torch.float64).pin_memory()
    f_h = torch.empty((N, 3), dtype=torch.float32).pin_memory()
    e2e_times = []
    gc.collect()
    gc.disable()
    for k in range(args.steps + 1):
        flush.fill_(1.0)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        pd = pos_h.to("cuda", non_blocking=True)
        sp.copy_(sp_h, non_blocking=True)
        gnl = nl_step(pd, gnl)
        e, f, _, _ = emp.mp_energy_forces(model, gnl, sp)
        e_h.copy_(e, non_blocking=True)
        f_h.copy_(f, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if k:
            e2e_times.append(a.elapsed_time(b))
    gc.enable()
    e2e_ms = reduce_max(sum(e2e_times) / len(e2e_times), torch.device("cuda", dev))

    # ---- roofline of the dominant kernel family
    pk, pk_kind = peaks()
    dom = max(fam.items(), key=lambda kv: kv[1][0])[0] if fam else None
    C = spec.C
    T = spec.n_layers
    so2_launches = fam.get("so2_tc", (0, 0))[1]
    roof = None
    tf32_rate = statistics.median(rates)             # TF32 TFLOP/s, every product counted
    tf32_rate_first = rates[0]
    if so2_launches:
        so2_ms = fam["so2_tc"][0] / so2_launches
        flops_step = mixing_flops_step(C, T, E)
        achieved = flops_step * len(ptimes) / (fam["so2_tc"][0] * 1e-3) / 1e12
        # the reference: the measured TF32 rate of the same tcgen05 products (operands resident in
        # shared memory, ~0.5 s back to back right after the step) / 3 for 3xTF32
        peak = tf32_rate / 3.0
        bf16_derived = pk["bf16_tflops_sustained"] * TF32_OVER_BF16 / 3.0
        traffic = so2_traffic_per_launch()
        roof = {"bound": "tensor", "kernel": "so2_tc (3xTF32 tcgen05 SO(2) mixing)", "achieved": achieved,
                "flops_per_step": flops_step,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "traffic_unit": "bytes per launch (DRAM read + write, ncu)" if traffic else None,
                "launch_ms": so2_ms, "launches_per_step": so2_launches / len(ptimes), "dominant": dom == "so2_tc",
                "peak_measured_tf32": tf32_rate, "peak_measured_tf32_first_launch": tf32_rate_first,
                "peak_bf16_derived": bf16_derived, "frac_vs_bf16_derived": achieved / bf16_derived,
                "peak_note": f"useful FP32 flops of the per-edge mixings (2*72*C^2 per edge and mixing, two "
                             f"mixings in each of the {max(T - 2, 0)} layers between the first and the last) over "
                             f"the summed launch event time (CUDA events on the launching stream), vs the "
                             f"measured TF32 rate of tcgen05.mma.cta_group::2.kind::tf32 (M=N=256, K=8, "
                             f"operands in shared memory; median of 40 launches after the step) / 3 (3xTF32); "
                             f"bf16-derived: {pk_kind} sustained bf16 x {TF32_OVER_BF16:.3f} / 3; median SM clock "
                             f"during the step {clk.summary().get('sm_mhz')} MHz"}
    elif dom is not None:
        roof = {"bound": "hbm", "kernel": dom, "achieved": None, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": None}
    hbm = hbm_fractions(fam, len(ptimes), E, N, C, T, pk["hbm_gbs"])
    configs = other_configs(emp, torch, stream, flush, pk["hbm_gbs"]) if (ws == 1 and not args.no_configs) else None
    kernel_ms = {k: round(v[0] / len(ptimes), 3) for k, v in sorted(fam.items(), key=lambda kv: -kv[1][0])}

    result = None
    if rank == 0:
        cpu = cpu_baseline() if (ws == 1 and not args.no_cpu_baseline) else None
        result = {"metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": ws, "steps": args.steps,
                  "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                  "vs_baseline": None, "dtype": "f32 (3xTF32 tensor-core mixing)", "data": "synthetic",
                  "config": {"workload": WORKLOAD, "n_atoms": N, "n_edges": E, "C": C, "lmax": 3,
                             "layers": spec.n_layers, "cohort_edges": spec.cohort_edges,
                             "parallelism": "replicas" if ws > 1 else "single",
                             "l2": "flushed between timed steps (256 MB write outside the timed events)",
                             "step": "mp_energy_forces on a resident neighbour graph, replayed as one CUDA graph "
                                     "of the library's launches; neighbour list timed separately (nl_ms)",
                             "workspace_bytes": int(efg.ws.numel()),
                             "backward": "y of the middle layer kept from the forward (mp_workspace_bytes); the "
                                         "recomputing form is timed in configs." + WORKLOAD + "_recompute_y"},
                  "nl_ms": sum(nl_times) / len(nl_times),
                  "p50_ms": statistics.median(lat), "p90_ms": float(np.percentile(lat, 90)), "latency_reps": len(lat),
                  "clocks": clk.summary(), "gpu_launches": launches,
                  "ms_per_step_profiled": sum(ptimes) / len(ptimes),
                  "step_ms": [round(t, 3) for t in times], "step_ms_profiled": [round(t, 3) for t in ptimes],
                  "e2e": {"value": E * ws / (e2e_ms * 1e-3), "unit": "edges/s",
                          "h2d_bytes_per_step": int(pos_h.numel() * 8 + sp_h.numel() * 4),
                          "d2h_bytes_per_step": int(8 + N * 3 * 4)},
                  "roofline": roof, "hbm_kernels": hbm, "cpu_baseline": cpu, "kernel_ms_per_step": kernel_ms,
                  "configs": configs,
                  "ns_per_atom": ms * 1e6 / N}
        print(json.dumps(result))
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other seeded workloads")
    ap.add_argument("--clocks-dir", default=None, help="where the raw nvidia-smi samples go (default: temp dir)")
    args = ap.parse_args()
    ws = os.environ.get("WORLD_SIZE")
    if ws is None and args.gpus > 1:
        # one rank per GPU: launch this script under torch.distributed.run
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
        return subprocess.call(cmd)
    if ws is not None and int(ws) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
