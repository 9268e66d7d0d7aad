#!/usr/bin/env python
"""Benchmark of the SchNet energy/force hot path on B200.

One step = one NVE velocity-Verlet step of 64 replicas of a 269-bead chain (r_cut 12 A,
F 128, K 50 Gaussians, T 3 blocks): kick + drift, neighbour-list rebuild, energy and
forces, kick.  That is every row of the hot path: neighbour build, radial basis, filter
network, message passing + segmented sums, update/readout, the hand-derived backward, and
the integrator.  The metric is energy+force evaluations per second (one per step) and
directed edges per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Inputs are seeded synthetic chains (self-avoiding random walks, 3.8 A bonds, 20 bead
types) and random weights from N(0, 1/fan_in), resident in HBM before timing.  L2 (126 MB)
is flushed between timed steps by writing a 256 MiB buffer; each step is bracketed by CUDA
events on the library's stream; the per-rank sum is max-reduced over ranks.  For N > 1 each
rank runs its own batch of replicas (no collective on the data path; weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402

from schnet_gnn_molecular_cell_b200 import synth  # noqa: E402

METRIC = "energy+force evals/s and edges/s (1 B200); % of HBM/tensor roofline"
CFG = 2
MASS, DT, TEMP = 12.0, 2.0, 300.0
# name -> (ABI precision, dtype string, tensor MMAs per algorithmic product)
PRECISIONS = {"tc32": (2, "f16x2-split (fp32-accurate), f32 accumulate", 3),
              "fp16": (1, "f16, f32 accumulate", 1),
              "fp16_ch": (3, "f16 with per-output-channel weight scales, f32 accumulate", 1),
              "fp32": (0, "f32", 0)}
WORKLOAD = "64 x 269-bead SAW chains, r_cut 12 A, SchNet F128 K50 T3: one velocity-Verlet step " \
           "(neighbour rebuild + energy/forces + integration)"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--precision", default="fp16", choices=list(PRECISIONS),
                    help="network arithmetic: fp16 = fp16 operands on tensor cores, fp32 accumulate "
                         "(W16A16, default), tc32 = fp32-accurate fp16 split on tensor cores, fp32 = CUDA cores")
    ap.add_argument("--no-variants", action="store_true", help="skip the short runs of the other precisions")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the cfg4 / evaluation-only rooflines and the cfg3 1000-step drift runs")
    ap.add_argument("--sweep", action="store_true",
                    help="replica-scaling sweep instead of the benchmark line: one JSON line per "
                         "(replicas, chain kind) with evals/s, steps x replicas/s and workspace bytes")
    return ap.parse_args(argv)


def max_over_ranks(x: float, device) -> float:
    """The maximum of a per-rank number over all ranks of the process group (the number itself
    with one rank): per-step times are reported as the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


# ------------------------------------------------------------------------------ CPU oracle
_NATIVE = None


def native_oracle():
    """The oracle built for this host (-O3 -march=native, same IEEE semantics), compiled here
    at run time into oracle/_build; the build used by every timed CPU leg."""
    global _NATIVE
    if _NATIVE is None:
        from oracle import oracle
        d = ROOT / "oracle" / "_build"
        d.mkdir(exist_ok=True)
        _NATIVE = oracle.build_native(d)
    return _NATIVE


def oracle_md_rate(w, v0, n_rep_sample: int, budget_s: float, min_steps: int = 1, threads: int | None = None):
    """Time the CPU oracle's velocity-Verlet steps on the first n_rep_sample replicas of the
    workload (native build; `threads` OpenMP threads, default all); returns (evals/s scaled to
    the full workload, steps run, seconds, threads)."""
    from oracle import oracle
    with oracle.using(native_oracle()):
        n0 = oracle.num_threads()
        if threads is not None:
            oracle.set_threads(threads)
        try:
            return _oracle_md_rate(oracle, w, v0, n_rep_sample, budget_s, min_steps)
        finally:
            oracle.set_threads(n0)


def _oracle_md_rate(oracle, w, v0, n_rep_sample, budget_s, min_steps):
    n_per = w.system.n_per_replica
    s = synth.SystemCfg(n_per, n_rep_sample, w.system.box)
    n = n_per * n_rep_sample
    pos, vel, types = w.pos[:n], v0[:n], w.types[:n]
    rp, cl = oracle.neighbors(s, w.model.r_cut, pos)
    _, forces, _ = oracle.energy_forces(w.model, w.weights, s, pos, types, rp, cl)
    steps, t0 = 0, time.perf_counter()
    while steps < min_steps or time.perf_counter() - t0 < budget_s:
        pos, vel, forces, *_ = oracle.md_vv(w.model, w.weights, s, pos, vel, types, MASS, DT, 1, forces=forces)
        steps += 1
    dt = time.perf_counter() - t0
    frac = n_rep_sample / w.system.n_replicas
    return steps * frac / dt, steps, dt, oracle.num_threads()


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = synth.make_workload(CFG)
    s = w.system
    v0 = synth.maxwell_boltzmann(s.n_per_replica, s.n_replicas, MASS, TEMP, 4000 + CFG)
    # size the per-step sample so that warm-up + K steps end within ~3 minutes
    probe_rate, _, probe_t, threads = oracle_md_rate(w, v0, 8, 0.0, min_steps=max(1, min(args.warmup, 3)))
    per_rep_s = 1.0 / (probe_rate * s.n_replicas)
    n_sample = int(max(1, min(s.n_replicas, 150.0 / max(1, args.steps) / per_rep_s)))
    rate, steps, secs, threads = oracle_md_rate(w, v0, n_sample, 0.0, min_steps=args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "evals/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": args.warmup, "ms_per_step": 1000.0 / rate, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": rate, "unit": "evals/s", "cores": threads, "kind": "oracle",
                         "build": "gcc -O3 -march=native -fopenmp -ffp-contract=off",
                         "sample": f"{n_sample} of {s.n_replicas} replicas per step, {steps} steps in "
                                   f"{secs:.1f} s; rate scaled to the full batch"},
        "e2e": {"value": rate, "unit": "evals/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.proc = None
        self.uuid = uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        loaded = [r for r in rows if (num(r[3]) or 0) > 0] or rows
        sm = [num(r[0]) for r in loaded if num(r[0]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for k, name in enumerate(names):
                if r[4 + k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][1]),
                "reasons": sorted(reasons), "samples": len(loaded)}


# ------------------------------------------------------------------------------ roofline
def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


def kernel_traffic(kernel: str, src: Path, precision: str = "fp32"):
    """dram bytes per launch of `kernel` from the committed ncu summary, if it was taken on
    the current source (else None)."""
    f = ROOT / "profiles" / "traffic.txt"
    if not f.exists():
        return None
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    for line in f.read_text().splitlines():
        parts = dict(kv.split("=", 1) for kv in line.split()[1:] if "=" in kv)
        if (line.split() and line.split()[0] == kernel and parts.get("src") == sha and parts.get("workload") == "cfg2"
                and parts.get("precision", "fp32") == precision):
            return float(parts["bytes_per_launch"])
    return None


# ------------------------------------------------------------------------------ whole-evaluation roofline
def eval_roofline(m, N: int, E: float, t_s: float, pk: dict, build: bool = False) -> dict:
    """One evaluation (or MD step, build=True) against the roof of the whole path: the slower of
    the minimum fused HBM bytes at the measured copy bandwidth and the filter networks'
    algorithmic FLOPs at the measured sustained dense tensor peak.
      FLOPs: 4 (K F + F^2) per directed edge per block (forward K->F->F, backward F->F->K).
      bytes: per block 8 passes over an [N][F] fp32 array (x read and written, h saved, hbar
             written and read, xbar read and written, p saved) = 32 N F, plus the 4-byte source
             and destination index of every edge; once per evaluation positions in, types,
             forces out (28 N); an MD step adds the list build (positions in, 4-byte counts and
             row offsets, the 4-byte col of every edge) and the integrator's 5 passes over
             [N][3] fp32 arrays."""
    F, K, T = m.F, m.K, m.T
    flops = 4.0 * (K * F + F * F) * E * T
    nbytes = 32.0 * N * F * T + 8.0 * E * T + 28.0 * N
    if build:
        nbytes += 12.0 * N + 8.0 * N + 4.0 * E + 60.0 * N
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * 1e12)
    t_roof = max(t_hbm, t_tc)
    return {"bound": "tensor" if t_tc >= t_hbm else "hbm", "frac": t_roof / t_s,
            "per_s": 1.0 / t_s, "roof_per_s": 1.0 / t_roof, "edges_per_s": E / t_s, "roof_edges_per_s": E / t_roof,
            "flops": flops, "bytes": nbytes, "t_roof_us": t_roof * 1e6, "t_us": t_s * 1e6,
            "peaks": f"{pk['hbm_gbs']:.0f} GB/s, {pk.get('bf16_tflops_sustained', pk['bf16_tflops']):.0f} TFLOP/s"}


def time_evals(cfg: int, precision_code: int, steps: int, dev, stream, flush):
    """Energy + forces alone on one configuration (list built once, outside the timing): CUDA
    events around each evaluation on the library's stream, L2 flushed before each.  Returns
    (seconds per evaluation, N, E, model)."""
    import torch
    from schnet_gnn_molecular_cell_b200 import Context
    w = synth.make_workload(cfg)
    s, m = w.system, w.model
    ctx = Context(m, w.weights, stream=stream, precision=precision_code)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    energy = torch.empty(s.n_replicas, device=dev)
    forces = torch.empty((s.n_atoms, 3), device=dev)
    for q in range(3):
        flush.fill_(float(q))
        ctx.energy_forces(s, pos, types, rp, cl, energy, forces)
    ctx.sync()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for q in range(steps):
        flush.fill_(float(q))
        ev[q][0].record(stream)
        ctx.energy_forces(s, pos, types, rp, cl, energy, forces)
        ev[q][1].record(stream)
    torch.cuda.synchronize()
    ctx.sync()
    t = sum(a.elapsed_time(b) for a, b in ev) / steps / 1e3
    ctx.close()
    return t, s.n_atoms, int(cl.numel()), m


def nve_drift(w, v0, precision_code: int, n_steps: int, dev, stream):
    """cfg3: n_steps of velocity Verlet (dt 2 fs, 12 amu, list rebuilt every step) from the
    seeded start; total energy E_pot + E_kin per replica after every step.  Returns the drift
    figures: max_t |E_tot(t) - E_tot(0)| / (n k_B T) per replica (median and max over
    replicas) and the slope of a linear fit of the replica-mean E_tot / (n k_B T) against
    time, per ns."""
    import torch
    from schnet_gnn_molecular_cell_b200 import Context
    s, m = w.system, w.model
    R, n = s.n_replicas, s.n_per_replica
    ctx = Context(m, w.weights, stream=stream, precision=precision_code)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    e0, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    ctx.reserve(s, 2 * int(cl.numel()) + 4096)
    hist = torch.empty((n_steps, 2, R), device=dev)   # potential and kinetic after each step
    t0 = time.perf_counter()
    for k in range(n_steps):
        ctx.md_step(s, pos, vel, forces, types, MASS, DT, 1, hist[k, 0], hist[k, 1])
    ctx.sync()
    wall = time.perf_counter() - t0
    h = hist.double().cpu().numpy()
    k0 = 0.5 * MASS / synth.KAPPA * (v0.astype(np.float64).reshape(R, n, 3) ** 2).sum(axis=(1, 2))
    etot = np.vstack([e0.double().cpu().numpy() + k0, h[:, 0] + h[:, 1]])
    ctx.close()
    return drift_figures(etot, n, n_steps, wall), etot


def drift_figures(etot, n_per: int, n_steps: int, wall_s: float | None = None) -> dict:
    kT = synth.KB * TEMP
    rel = (etot - etot[:1]) / (n_per * kT)             # [steps + 1][R]
    per_rep = np.abs(rel).max(axis=0)
    t_ns = np.arange(etot.shape[0]) * DT * 1e-6
    slope = float(np.polyfit(t_ns, rel.mean(axis=1), 1)[0])
    out = {"steps": n_steps, "dt_fs": DT, "max_abs_drift_per_nkT": {"median": float(np.median(per_rep)),
                                                                    "max": float(per_rep.max())},
           "slope_per_ns_per_nkT": slope}
    if wall_s is not None:
        out["wall_s"] = wall_s
    return out


def oracle_drift(w, v0, n_rep: int, n_steps: int) -> dict:
    """The oracle's (double-precision) velocity-Verlet drift on the first n_rep replicas."""
    from oracle import oracle
    n = w.system.n_per_replica
    s = synth.SystemCfg(n, n_rep, w.system.box)
    with oracle.using(native_oracle()):
        _, _, _, epot, ekin, _ = oracle.md_vv(w.model, w.weights, s, w.pos[: n * n_rep], v0[: n * n_rep],
                                              w.types[: n * n_rep], MASS, DT, n_steps)
        rp, cl = oracle.neighbors(s, w.model.r_cut, w.pos[: n * n_rep])
        e0, _, _ = oracle.energy_forces(w.model, w.weights, s, w.pos[: n * n_rep], w.types[: n * n_rep], rp, cl)
    k0 = 0.5 * MASS / synth.KAPPA * (v0[: n * n_rep].astype(np.float64).reshape(n_rep, n, 3) ** 2).sum(axis=(1, 2))
    etot = np.vstack([e0 + k0, epot + ekin])
    return drift_figures(etot, n, n_steps)


# ------------------------------------------------------------------------------ our arm
def time_variant(w, v0, precision_code, steps, dev, stream, flush):
    """Short timed run of another precision on the same workload (same protocol, no trace)."""
    import torch
    from schnet_gnn_molecular_cell_b200 import Context
    s, m = w.system, w.model
    ctx = Context(m, w.weights, stream=stream, precision=precision_code)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    _, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    ctx.reserve(s, int(1.5 * cl.numel()) + 4096)
    e = torch.empty(s.n_replicas, device=dev)
    k = torch.empty(s.n_replicas, device=dev)
    for q in range(3):
        flush.fill_(float(q))
        ctx.md_step(s, pos, vel, forces, types, MASS, DT, 1, e, k)
    ctx.sync()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for q in range(steps):
        flush.fill_(float(q))
        starts[q].record(stream)
        ctx.md_step(s, pos, vel, forces, types, MASS, DT, 1, e, k)
        ends[q].record(stream)
    torch.cuda.synchronize()
    ctx.sync()
    t = sum(a.elapsed_time(b) for a, b in zip(starts, ends))
    ctx.close()
    return {"value": steps / (t / 1e3), "unit": "evals/s", "ms_per_step": t / steps, "steps": steps}


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    from schnet_gnn_molecular_cell_b200 import Context

    w = synth.make_workload(CFG)
    s, m = w.system, w.model
    N, R = s.n_atoms, s.n_replicas
    v0 = synth.maxwell_boltzmann(s.n_per_replica, R, MASS, TEMP, 4000 + CFG)
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    prec_code, dtype, mma_per_product = PRECISIONS[args.precision]
    ctx = Context(m, w.weights, stream=stream, precision=prec_code)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    E0 = int(cl.numel())
    _, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    ctx.reserve(s, int(1.5 * E0) + 4096)
    energy = torch.empty(R, device=dev)
    kin = torch.empty(R, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2

    def step():
        ctx.md_step(s, pos, vel, forces, types, MASS, DT, 1, energy, kin)

    for k in range(args.warmup):
        flush.fill_(float(k))
        step()
    ctx.sync()
    # the trajectory moves the edge count; the traced pass below replays the timed steps
    # from this same state
    saved = (pos.clone(), vel.clone(), forces.clone())
    E_start = ctx.md_edges()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for k in range(args.steps):
        flush.fill_(float(k))
        starts[k].record(stream)
        step()
        ends[k].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ctx.sync()
    t_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends))
    E_end = ctx.md_edges()
    # per-kernel times from the library's tracer (CUDA events around every launch) on a
    # separate pass over the first steps of the same trajectory, so that the events do not
    # slow the timed region; E per traced step for the roofline's FLOP count
    n_tr = min(args.steps, 100)
    pos.copy_(saved[0]), vel.copy_(saved[1]), forces.copy_(saved[2])
    ctx.trace(True)
    E_tr = 0
    for k in range(n_tr):
        flush.fill_(float(k))
        step()
        E_tr += ctx.md_edges()
    trace = ctx.trace_read()
    ctx.trace(False)
    ctx.sync()
    E_tr /= n_tr
    t_ms = max_over_ranks(t_ms, dev)
    if world > 1:
        torch.distributed.barrier()
    E_mean = 0.5 * (E_start + E_end)
    value = world * args.steps / (t_ms / 1e3)

    # dominant kernel and its roofline (algorithmic filter-network FLOPs per launch / mean
    # launch time; the backward's forward recompute and the split's extra MMAs not counted)
    dom = max(trace, key=lambda k: trace[k][1])
    launches, dom_ms = trace[dom]
    pk, pk_kind = peaks()
    roofline = None
    if dom in ("edge_fwd", "edge_bwd"):
        flops = 2.0 * (m.K * m.F + m.F * m.F) * E_tr
        achieved = flops / (dom_ms / launches / 1e3) / 1e12
        src = ROOT / "schnet_gnn_molecular_cell_b200" / "csrc" / ("sn_ef_fp32.cu" if prec_code == 0 else "sn_ef_tc.cu")
        if prec_code == 0:
            peak = 148 * 128 * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            bound, peak_src = "alu", (f"fp32 FMA: 148 SM x 128 lanes x 2 x {pk.get('sm_max_mhz', 1965.0):.0f} MHz "
                                      f"({pk_kind} sm_max_mhz)")
        else:
            peak = pk.get("bf16_tflops_sustained", 1398.0)
            bound, peak_src = "tensor", (f"{pk_kind} dense bf16 sustained (fp16 kind::f16 runs at the same rate); "
                                         f"this mode issues {mma_per_product} MMA(s) per product")
        roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": kernel_traffic(dom, src, args.precision),
                    "kernel": dom, "peak_source": peak_src, "flops_per_launch": flops}

    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
        h_pos, h_vel, h_f = pin(pos.cpu().numpy()), pin(vel.cpu().numpy()), pin(forces.cpu().numpy())
        h_types = pin(w.types)
        h_e = pin(np.zeros(R, np.float32))
        h_k = pin(np.zeros(R, np.float32))
        n_e2e = min(args.steps, 100)
        tot = 0.0
        for k in range(n_e2e + 2):
            flush.fill_(float(k))
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            ctx.md_step_host(s, h_pos, h_vel, h_f, h_types, MASS, DT, 1, h_e, h_k)
            t1 = time.perf_counter()
            if k >= 2:
                tot += t1 - t0
        tot = max_over_ranks(tot, dev)
        e2e = {"value": world * n_e2e / tot, "unit": "evals/s",
               "h2d_bytes_per_step": 3 * (3 * N * 4) + N * 4,
               "d2h_bytes_per_step": 3 * (3 * N * 4) + 2 * R * 4,
               "api": "sn_md_step_host (pinned host buffers; copies + step + sync timed by host clock)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, steps, secs, threads = oracle_md_rate(w, v0, R, 10.0)
        r1, steps1, secs1, _ = oracle_md_rate(w, v0, 4, 8.0, threads=1)
        cpu = {"value": rate, "unit": "evals/s", "cores": threads, "kind": "oracle",
               "build": "gcc -O3 -march=native -fopenmp -ffp-contract=off",
               "sample": f"{steps} full velocity-Verlet step(s) of all {R} replicas in {secs:.1f} s",
               "single_thread": {"value": r1, "unit": "evals/s", "cores": 1,
                                 "sample": f"{steps1} step(s) of 4 of {R} replicas in {secs1:.1f} s, "
                                           f"rate scaled to the full batch"}}

    extras = {}
    if rank == 0 and world == 1 and not args.no_extras:
        # the chains' evaluation alone and the 4096- and 65,536-atom periodic boxes (cfg4,
        # cfg5), each mode; the whole-evaluation roofline of these and of the MD step timed above
        extras["roofline_eval"] = {"cfg2_md_step": eval_roofline(m, N, E_mean, t_ms / args.steps / 1e3, pk, build=True)}
        extras["roofline_eval"]["cfg2_md_step"]["steps_x_replicas_per_s"] = value * R
        extras["roofline_eval"]["cfg2_md_step"]["roof_steps_x_replicas_per_s"] = \
            extras["roofline_eval"]["cfg2_md_step"]["roof_per_s"] * R
        for cfg in (2, 4, 5):
            for name in ("fp16", "tc32"):
                t_e, n_e, e_e, m_e = time_evals(cfg, PRECISIONS[name][0], 50, dev, stream, flush)
                extras["roofline_eval"][f"cfg{cfg}_eval_{name}"] = eval_roofline(m_e, n_e, e_e, t_e, pk)
        # cfg3: 1000 NVE steps of the chains in each tensor mode, total-energy drift; the
        # oracle's over the first 100 steps of 4 replicas beside the same window of the GPU run
        drift = {}
        for name in ("fp16", "tc32"):
            fig, etot = nve_drift(w, v0, PRECISIONS[name][0], 1000, dev, stream)
            fig["first_100_steps_replicas_0_3"] = drift_figures(etot[:101, :4], s.n_per_replica, 100)
            drift[name] = fig
        drift["oracle_first_100_steps_replicas_0_3"] = oracle_drift(w, v0, 4, 100)
        extras["nve_drift_cfg3"] = drift

    variants = None
    if rank == 0 and world == 1 and not args.no_variants:
        variants = {}
        for name, (code, vdtype, _) in PRECISIONS.items():
            if name != args.precision:
                v = time_variant(w, v0, code, min(args.steps, 50), dev, stream, flush)
                v["dtype"] = vdtype
                variants[name] = v

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "evals/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
            "config": {"workload": WORKLOAD, "replicas_per_gpu": R, "beads": s.n_per_replica,
                       "edges": {"start": E_start, "end": E_end}, "precision": args.precision,
                       "l2": "flushed between steps (256 MiB write, outside the timed events)",
                       "parallelism": f"{world} rank(s), independent replica batches, no collective"},
            "edges_per_s": value * E_mean,
            "md_steps_x_replicas_per_s": value * R,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": round(sum(v[0] for v in trace.values()) * args.steps / n_tr),
            "precision_variants": variants,
            **extras,
            "clocks": clocks,
            "kernels": {k: {"launches": v[0], "ms_per_launch": v[1] / v[0], "share": v[1] / sum(x[1] for x in trace.values())}
                        for k, v in sorted(trace.items(), key=lambda kv: -kv[1][1])},
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        torch.distributed.destroy_process_group()


def run_sweep(args):
    """Throughput against the number of replicas (1 .. 2048 chains of 269 beads) for extended
    (self-avoiding) and compact (free random walk) chains, with the model and MD step of the
    benchmark: the analogue of the pages' replica-scaling and dynamic-topology figures
    (FlashSchNet §5.3).  Same timing protocol as the benchmark (CUDA events per step, L2 flushed
    before each step); workspace = device memory the library context holds."""
    import torch
    from schnet_gnn_molecular_cell_b200 import Context
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    m = synth.CONFIGS[CFG]["model"]
    w0 = synth.make_workload(CFG)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    prec_code = PRECISIONS[args.precision][0]
    for kind in ("saw", "rw"):
        for R in (1, 4, 16, 64, 256, 1024, 2048):
            s = synth.SystemCfg(269, R)
            pos0 = synth.chains(269, R, 1000 + R, saw=(kind == "saw"))
            types = synth.bead_types(s.n_atoms, m.n_types, 2000 + R)
            v0 = synth.maxwell_boltzmann(269, R, MASS, TEMP, 4000 + R)
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info(dev)[0]
            ctx = Context(m, w0.weights, stream=stream, precision=prec_code)
            pos = torch.from_numpy(pos0.copy()).to(dev)
            vel = torch.from_numpy(v0.copy()).to(dev)
            ty = torch.from_numpy(types).to(dev)
            rp, cl = ctx.neighbors(s, pos)
            E0 = int(cl.numel())
            _, forces = ctx.energy_forces(s, pos, ty, rp, cl)
            forces = forces.clone()
            del rp, cl
            ctx.reserve(s, int(1.5 * E0) + 4096)
            e = torch.empty(R, device=dev)
            k = torch.empty(R, device=dev)
            steps = max(5, min(200, int(2e8 / max(E0, 1))))
            for q in range(3):
                flush.fill_(float(q))
                ctx.md_step(s, pos, vel, forces, ty, MASS, DT, 1, e, k)
            ctx.sync()
            torch.cuda.synchronize()
            workspace = free0 - torch.cuda.mem_get_info(dev)[0]
            t = 0.0
            for q in range(steps):
                flush.fill_(float(q))
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                ctx.md_step(s, pos, vel, forces, ty, MASS, DT, 1, e, k)
                b.record(stream)
                b.synchronize()
                t += a.elapsed_time(b)
            ctx.sync()
            E1 = ctx.md_edges()
            ctx.close()
            del pos, vel, ty, forces, e, k
            rate = steps / (t / 1e3)
            print(json.dumps({"sweep": "replicas", "kind": kind, "replicas": R, "atoms": s.n_atoms,
                              "edges": {"start": E0, "end": E1}, "precision": args.precision, "steps": steps,
                              "evals_per_s": rate, "md_steps_x_replicas_per_s": rate * R,
                              "edges_per_s": rate * 0.5 * (E0 + E1), "workspace_bytes": workspace}), flush=True)


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
