#!/usr/bin/env python
"""Benchmark of the neighbour-graph hot path: CSR build + block-dense attention.

One step = one ``mlg_forward`` call (on-device cell-list CSR build, then every
attention layer of the workload) over the seeded synthetic system. The metric
is atoms/s (device-timed, CUDA events on the launching stream) with ms/step,
plus the roofline fraction of the dominant kernel, measured live.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica of the whole workload on its own GPU (the path has no exchange step);
the time is the max over ranks and ``value`` counts the atoms of all ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from neighbour_graph_attention_b200 import configs as C  # noqa: E402

METRIC = "atoms/s (build+attention, device-timed)"
DATA = "synthetic (seeded generator)"
DEFAULT_WORKLOAD = 5  # Fe BCC, 524,288 atoms, fp32: the largest system of the list
L2_FLUSH_BYTES = 256 << 20  # > 126 MB of L2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
# Plain-ALU peaks from unit counts and the maximum SM clock: 148 SMs,
# 64 FP64 FMA / 128 FP32 FMA per SM per clock, 2 flops per FMA, 1.965 GHz.
SM_COUNT, SM_MAX_GHZ = 148, 1.965
FP64_PEAK_TFLOPS = SM_COUNT * 64 * 2 * SM_MAX_GHZ / 1e3
FP32_PEAK_TFLOPS = SM_COUNT * 128 * 2 * SM_MAX_GHZ / 1e3
# Special-function unit (ex2): 16 per SM per clock.
SFU_PEAK_TEXP = SM_COUNT * 16 * SM_MAX_GHZ / 1e3

# DRAM traffic per launch of a workload's attention (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture, summarised under profiles/),
# with the kernels it was taken on: used only while the library still
# launches those kernels for the workload.  A change to a kernel removes its
# entry.
ATTN_TRAFFIC = {
    2: ("k_attn_dmma", 5.622e6),   # profiles/k_attn_dmma_f64_diamond512.md
    # profiles/k_attn_tc7_fe_bcc_65536.md: 1,077 MB per launch at 65,536 atoms
    # (4,194,304 edges), scaled by the edges to 33,554,436
    5: ("k_attn_tc7 (tcgen05 logits, mma.sync P.V, rows <= 64) + k_attn_tc (rows <= 128)",
        1.0769e9 * 33554436 / 4194304),
}


def tensor_core_path(kernels: str) -> bool:
    """The logits run on tcgen05 and P.V from registers: the softmax's
    exponentials (special-function unit) are the roofline, not a pipe's FMAs."""
    return "tcgen05 logits" in kernels


def attention_exps(row_ptr, heads):
    """Per layer: one exponential per logit, sum_i n_i^2 * heads."""
    n = np.diff(np.asarray(row_ptr)).astype(np.float64)
    return float(np.sum(n * n)) * heads


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=sorted(C.WORKLOADS))
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--cells", type=int, default=None,
                   help="profiling only: conventional cells per axis of a lattice workload "
                        "(same shapes, fewer atoms)")
    p.add_argument("--impl", choices=["mlg", "reference"], default="mlg")
    p.add_argument("--variant", choices=["block", "smooth", "local"], default="block",
                   help="attention of the step: block-dense (default), block-dense with the "
                        "slot-occupancy softmax in every layer, or local attention (one query "
                        "per centre; the first layer's weights)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="CPU time budget of the oracle baseline sample")
    args = p.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    args.steps = max(args.steps, 1)
    return args


# ------------------------------------------------------------------ metrics

def attention_flops(row_ptr, channels):
    """Per layer: sum_i (6 n_i c^2 + 4 n_i^2 c) (projections, QK^T, PV)."""
    n = np.diff(np.asarray(row_ptr)).astype(np.float64)
    return float(np.sum(6.0 * n * channels * channels + 4.0 * n * n * channels))


def local_attention_flops(row_ptr, channels, heads):
    """Local attention, reassociated: sum_i 2 (3 c^2 + 2 n_i c H)."""
    n = np.diff(np.asarray(row_ptr)).astype(np.float64)
    return float(np.sum(2.0 * (3.0 * channels * channels + 2.0 * n * channels * heads)))


def attention_bytes(n_atoms, n_edges, channels, elem):
    """Per layer: G in + O out + s(r) + row_ptr + three weight matrices."""
    return 2.0 * n_edges * channels * elem + 8.0 * n_edges + 8.0 * (n_atoms + 1) + \
        3.0 * channels * channels * elem


def build_bytes(n_atoms, n_edges):
    """Coordinates in, row_ptr and 56 B per edge out (src, shift, vec, dist, s)."""
    return 24.0 * n_atoms + 8.0 * (n_atoms + 1) + 56.0 * n_edges


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ ranks

def max_over_ranks(x: float, device) -> float:
    """The max of x over the ranks of the default process group (x alone at N = 1)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, n_atoms: int, steps: int, total_ms: float) -> float:
    """Atoms per second of N independent replicas timed by the slowest rank."""
    return world * n_atoms * steps / (total_ms / 1e3)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.samples = []
        self.ok = False
        self.period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = torch_device_index
            if vis:
                ids = [v for v in vis.split(",") if v.strip()]
                if torch_device_index < len(ids) and ids[torch_device_index].strip().isdigit():
                    idx = int(ids[torch_device_index])
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML on this machine
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside = self.samples
            window = "load window ending with the timed region"
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= int(s[2])
        reasons = [name for b, name in self.REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ------------------------------------------------------------------ reference arm

def oracle_step(w, s, W, G, sample_centres=None):
    """One oracle pass: brute-force CSR and every attention layer."""
    import oracle

    if sample_centres is None:
        csr = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        oracle.forward(csr["row_ptr"], csr["sw"], G, W, w.heads, w.dtype)
        return w.n_atoms
    # bounded sample: the CSR rows of the sampled centres (brute force per
    # centre) and their attention layers
    rows, sws, counts = [], [], []
    for i in sample_centres:
        one = oracle.centre(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max, int(i))
        counts.append(one["src"].size)
        sws.append(one["sw"])
    rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    g = G[: int(rp[-1])]
    oracle.forward(rp, np.concatenate(sws) if sws else np.zeros(0), g, W, w.heads, w.dtype)
    return len(sample_centres)


def cpu_sample_plan(w, budget_s):
    """Full system if it is small; otherwise a count of centres sized to the budget."""
    if w.n_atoms <= 6000:
        return None, f"full system ({w.n_atoms} atoms), repeated"
    # brute force per centre is O(N): size the sample to about the time budget
    per_centre_s = 2e-8 * w.n_atoms + 2e-6 * w.nnei_max * w.channels * w.n_layers
    m = int(max(16, min(w.n_atoms, budget_s / per_centre_s / 2)))
    return m, f"{m} of {w.n_atoms} centres (brute-force CSR rows + all layers), repeated"


def run_oracle_timing(w, s, W, budget_s, seed):
    cores = len(os.sched_getaffinity(0))
    count, desc = cpu_sample_plan(w, budget_s)
    rng = np.random.default_rng(seed + 99)
    centres = None if count is None else np.sort(rng.choice(w.n_atoms, count, replace=False))
    e_guess = w.n_atoms * w.nnei_max if count is None else count * w.nnei_max
    G = C.features(w.key, seed, e_guess)
    if count is None:
        import oracle

        csr = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        G = C.features(w.key, seed, int(csr["row_ptr"][-1]))
    done, t0 = 0, time.perf_counter()
    reps = 0
    while True:
        done += oracle_step(w, s, W, G, centres)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    return {"value": done / el, "unit": "atoms/s", "cores": cores, "kind": "oracle",
            "sample": f"{desc}; {reps} pass(es) in {el:.1f} s; OpenMP over centres"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = C.workload(args.workload)
    s = C.system(args.workload, args.seed)
    W = C.weights(args.workload, args.seed)
    cores = len(os.sched_getaffinity(0))
    # each step: a bounded sample sized so that warm-up + steps stay within minutes
    per_step_budget = max(0.05, 150.0 / (args.steps + args.warmup))
    count, desc = cpu_sample_plan(w, per_step_budget)
    rng = np.random.default_rng(args.seed + 7)
    centres = None if count is None else np.sort(rng.choice(w.n_atoms, count, replace=False))
    if count is None:
        import oracle

        csr = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        G = C.features(w.key, args.seed, int(csr["row_ptr"][-1]))
    else:
        G = C.features(w.key, args.seed, count * w.nnei_max)
    for _ in range(args.warmup):
        oracle_step(w, s, W, G, centres)
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += oracle_step(w, s, W, G, centres)
    el = time.perf_counter() - t0
    value = done / el
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "atoms/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": DATA,
            "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": "atoms/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "atoms/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def select_workload(args):
    """The workload, optionally with fewer lattice cells (profiling runs only)."""
    import dataclasses

    w = C.workload(args.workload)
    if args.cells is not None and w.periodic and args.cells != w.cells:
        per_cell = w.n_atoms // w.cells ** 3
        w = dataclasses.replace(w, cells=args.cells, n_atoms=per_cell * args.cells ** 3,
                                name=f"{w.name}-cells{args.cells}")
        C.WORKLOADS[w.key] = w
    return w, C.system(w.key, args.seed)


def workload_config(w, args, extra=None):
    layers = 1 if getattr(args, "variant", "block") == "local" else w.n_layers
    cfg = {"workload": f"{w.name}: {w.n_atoms} atoms, {w.lattice}, rcut {w.rcut} A, "
                       f"nnei_max {w.nnei_max}, c={w.channels}, heads={w.heads}, "
                       f"layers={layers}, {w.dtype}",
           "workload_index": w.key, "seed": args.seed, "n_atoms": w.n_atoms,
           "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU",
           "l2": "flushed between timed steps (256 MiB write)"}
    if getattr(args, "variant", "block") != "block":
        cfg["variant"] = {"smooth": "slot-occupancy softmax in every layer",
                          "local": "local attention (one query per centre)"}[args.variant]
    if extra:
        cfg.update(extra)
    return cfg


# ------------------------------------------------------------------ GPU arm

def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from neighbour_graph_attention_b200 import build as nb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    if rank == 0 or world == 1:
        nb.build()
    if world > 1:
        dist.barrier()
    from neighbour_graph_attention_b200 import mlg as m

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w, s = select_workload(args)
    W = C.weights(args.workload, args.seed)
    dt = torch.float64 if w.dtype == "f64" else torch.float32
    elem = 8 if w.dtype == "f64" else 4
    mdt = m.MLG_F64 if w.dtype == "f64" else m.MLG_F32
    stream = torch.cuda.Stream(device=dev)

    x = torch.as_tensor(s["coords"], device=dev)
    types = torch.as_tensor(s["types"], device=dev)
    sysd = m.make_system(x, s["box"], s["pbc"], types, s["n_types"])
    # first build with the always-sufficient capacity, to learn E
    cap0 = w.n_atoms * w.nnei_max
    csr0 = m.Csr.empty(w.n_atoms, cap0, device=dev)
    ws_b = m.workspace(m.mlg_build_csr_workspace_bytes(w.n_atoms, w.rcut, s["box"], s["pbc"]),
                       device=dev)
    with torch.cuda.stream(stream):
        m.mlg_build_csr(sysd, w.rcut, w.r_on, w.nnei_max, csr0, ws_b, stream=stream)
    stream.synchronize()
    E = int(csr0.n_edges.item())
    row_ptr = csr0.row_ptr.cpu().numpy()
    del csr0
    csr = m.Csr.empty(w.n_atoms, E, device=dev)
    G0 = torch.as_tensor(C.features(args.workload, args.seed, E), dtype=dt, device=dev)
    local = args.variant == "local"
    # local attention writes one row per centre, from the centres' own features
    Gout = torch.empty((w.n_atoms, w.channels), dtype=dt, device=dev) if local \
        else torch.empty_like(G0)
    Hc = torch.as_tensor(C.features(args.workload, args.seed + 1000, w.n_atoms), dtype=dt,
                         device=dev) if local else None
    Wt = [torch.as_tensor(W[l][k], dtype=dt, device=dev) for l in range(w.n_layers)
          for k in range(3)]
    ws = m.workspace(m.mlg_forward_workspace_bytes(w.n_atoms, w.rcut, s["box"], s["pbc"], E,
                                                   w.channels, w.n_layers, mdt), device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    stack_ws = m.workspace(m.mlg_attention_stack_workspace_bytes(E, w.channels, w.n_layers, mdt),
                           device=dev)

    # one step = the two calls mlg_forward makes: the CSR build, then the
    # fused attention stack; an event between them times the attention
    # launch inside the timed region
    def build_call():
        m.mlg_build_csr(sysd, w.rcut, w.r_on, w.nnei_max, csr, ws, stream=stream)

    def attn_call(g_in, g_out):
        if args.variant == "smooth":
            m.mlg_attention_stack_smooth(csr, w.n_atoms, w.nnei_max, w.channels, w.heads,
                                         w.n_layers, mdt, Wt, g_in, g_out, stack_ws, stream=stream)
        elif local:
            m.mlg_local_attention(csr, w.n_atoms, w.nnei_max, w.channels, w.heads, mdt, Hc, g_in,
                                  g_out, Wt[0], Wt[1], Wt[2], stream=stream)
        else:
            m.mlg_attention_stack(csr, w.n_atoms, w.nnei_max, w.channels, w.heads, w.n_layers,
                                  mdt, Wt, g_in, g_out, stack_ws, stream=stream)

    def stack_call():
        attn_call(G0, Gout)

    def timed_steps(k):
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(k)]
        with torch.cuda.stream(stream):
            for e0, e1, e2 in evs:
                flush.fill_(1.0)          # L2 flush, outside the timed events
                e0.record(stream)
                build_call()
                e1.record(stream)
                stack_call()
                e2.record(stream)
        stream.synchronize()
        return [(e0.elapsed_time(e1), e1.elapsed_time(e2)) for e0, e1, e2 in evs]

    def timed_loop(fn, k):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(k)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                flush.fill_(1.0)
                a.record(stream)
                fn()
                b.record(stream)
        stream.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    # warm-up, then a load pre-roll that lets the clock sampler see the GPU busy
    timed_steps(args.warmup)
    sampler = ClockSampler(dev.index)
    sampler.start()
    t_pre = time.perf_counter()
    while time.perf_counter() - t_pre < 1.0:
        timed_steps(20)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    parts = timed_steps(args.steps)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    build_ms_steps = [p[0] for p in parts]
    attn_ms_steps = [p[1] for p in parts]
    total_ms = max_over_ranks(float(sum(build_ms_steps) + sum(attn_ms_steps)), dev)
    ms_per_step = total_ms / args.steps
    value = replica_throughput(world, w.n_atoms, args.steps, total_ms)

    status = int(csr.status.item())
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the timed steps")

    attn_avg = statistics.mean(attn_ms_steps)
    build_avg = statistics.mean(build_ms_steps)
    flops = local_attention_flops(row_ptr, w.channels, w.heads) if local else \
        attention_flops(row_ptr, w.channels) * w.n_layers
    peak_fp = FP64_PEAK_TFLOPS if w.dtype == "f64" else FP32_PEAK_TFLOPS
    achieved_tf = flops / (attn_avg * 1e-3) / 1e12
    hbm_peak, hbm_src = load_peaks()
    bbytes = build_bytes(w.n_atoms, E)
    abytes = attention_bytes(w.n_atoms, E, w.channels, elem) + \
        (w.n_layers - 1) * 3.0 * w.channels * w.channels * elem
    kernels = m.mlg_attention_kernels(w.nnei_max, w.channels, w.heads, w.n_layers, mdt)
    kname = kernels if not local else (
        "k_local_attn_w32" if w.channels == 32 and w.heads in (1, 2, 4, 8) else "k_local_attn")
    rec_k, traffic = ATTN_TRAFFIC.get(w.key, ("", None))
    if rec_k != kname or args.variant != "block":
        traffic = None
    if args.cells is not None:   # a resized system: the stored capture does not apply
        traffic = None
    if tensor_core_path(kernels) and args.variant == "block":
        # products on the tensor cores: the exponentials bound the kernel
        # (special-function unit), ahead of HBM and of the tensor pipe
        exps = attention_exps(row_ptr, w.heads) * w.n_layers
        achieved_ex = exps / (attn_avg * 1e-3) / 1e12
        roofline = {"bound": "alu", "achieved": achieved_ex, "peak": SFU_PEAK_TEXP,
                    "unit": "Texp/s", "frac": achieved_ex / SFU_PEAK_TEXP, "traffic": traffic,
                    "kernel": kname, "algorithmic_exps_per_launch": exps,
                    "algorithmic_flops_per_launch": flops, "achieved_tflops": achieved_tf,
                    "peak_basis": "derived: 148 SMs x 16 ex2/clk x 1.965 GHz (special-function "
                                  "unit; the exponentials' floor exceeds the HBM and "
                                  "tensor-pipe floors)",
                    "hbm_frac_of_" + hbm_src: abytes / (attn_avg * 1e-3) / 1e9 / hbm_peak}
    else:
        roofline = {"bound": "alu", "achieved": achieved_tf, "peak": peak_fp,
                    "unit": "TFLOP/s", "frac": achieved_tf / peak_fp, "traffic": traffic,
                    "kernel": "%s (all %d layer(s) in one launch)" % (kname, w.n_layers),
                    "algorithmic_flops_per_launch": flops,
                    "peak_basis": ("derived: 148 SMs x %d %s FMA/clk x 2 x 1.965 GHz" %
                                   (64 if w.dtype == "f64" else 128, w.dtype.upper())),
                    "hbm_frac_of_" + hbm_src: abytes / (attn_avg * 1e-3) / 1e9 / hbm_peak}
    build_gbs = bbytes / (build_avg * 1e-3) / 1e9
    roofline_build = {"bound": "hbm", "achieved": build_gbs, "peak": hbm_peak, "unit": "GB/s",
                      "frac": build_gbs / hbm_peak, "peak_source": hbm_src,
                      "algorithmic_bytes": bbytes, "ms": build_avg,
                      "note": "whole build stage (several kernels)"}
    layers_share = attn_avg / max(ms_per_step, 1e-9)

    # end to end through the C ABI with host buffers: pinned H2D of the
    # step's inputs (coordinates, edge features), the build and the attention
    # stack, D2H of the result.  The edge features cross PCIe on a second
    # stream while the build (which needs only the coordinates) runs.
    x_h = torch.as_tensor(s["coords"]).pin_memory()
    g_h = G0.cpu().pin_memory()
    out_h = torch.empty(Gout.shape, dtype=dt).pin_memory()
    x_d = torch.empty_like(x)
    g_d = torch.empty_like(G0)
    sys_e = m.make_system(x_d, s["box"], s["pbc"], types, s["n_types"])
    side = torch.cuda.Stream(device=dev)
    ev_start, ev_g = torch.cuda.Event(), torch.cuda.Event()

    def e2e_step():
        ev_start.record(stream)
        side.wait_event(ev_start)
        with torch.cuda.stream(side):
            g_d.copy_(g_h, non_blocking=True)
        ev_g.record(side)
        x_d.copy_(x_h, non_blocking=True)
        m.mlg_build_csr(sys_e, w.rcut, w.r_on, w.nnei_max, csr, ws, stream=stream)
        stream.wait_event(ev_g)
        attn_call(g_d, Gout)
        out_h.copy_(Gout, non_blocking=True)

    timed_loop(e2e_step, 3)
    lat_ms = timed_loop(e2e_step, args.steps)
    lat_total = max_over_ranks(float(sum(lat_ms)), dev)

    # the same steps pipelined, as a stream of independent evaluations is
    # served: copies in, compute and copies out on three streams with two
    # sets of device buffers, so that step k+1's inputs and step k-1's
    # result cross PCIe while step k computes.  Every step still copies its
    # coordinates and edge features from pinned host memory and its whole
    # result back; the timed region runs from before the first copy in to
    # after the last copy out.
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    xs = [x_d, torch.empty_like(x)]
    gs = [g_d, torch.empty_like(G0)]
    ys = [Gout, torch.empty_like(Gout)]
    ys_h = [out_h, torch.empty(Gout.shape, dtype=dt).pin_memory()]
    syss = [sys_e, m.make_system(xs[1], s["box"], s["pbc"], types, s["n_types"])]

    def e2e_pipelined(k):
        ev_in = [torch.cuda.Event() for _ in range(k)]
        ev_done = [torch.cuda.Event() for _ in range(k)]   # step i computed: its inputs are free
        ev_out = [torch.cuda.Event() for _ in range(k)]    # step i read back: its output is free
        t_a = torch.cuda.Event(enable_timing=True)
        t_b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
        t_a.record(stream)
        s_in.wait_event(t_a)
        s_out.wait_event(t_a)
        for i in range(k):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_done[i - 2])
            with torch.cuda.stream(s_in):
                xs[b].copy_(x_h, non_blocking=True)
                gs[b].copy_(g_h, non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])
            m.mlg_build_csr(syss[b], w.rcut, w.r_on, w.nnei_max, csr, ws, stream=stream)
            attn_call(gs[b], ys[b])
            ev_done[i].record(stream)
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                ys_h[b].copy_(ys[b], non_blocking=True)
            ev_out[i].record(s_out)
        stream.wait_event(ev_out[k - 1])
        t_b.record(stream)
        stream.synchronize()
        return t_a.elapsed_time(t_b)

    e2e_pipelined(max(args.warmup, 3))
    e2e_total = max_over_ranks(e2e_pipelined(args.steps), dev)
    e2e_value = replica_throughput(world, w.n_atoms, args.steps, e2e_total)
    # the pipelined result equals the device-resident one
    if args.steps > 1 and not torch.equal(ys[0], ys[1]):
        raise RuntimeError("pipelined end-to-end steps disagree")
    h2d = x_h.numel() * x_h.element_size() + g_h.numel() * g_h.element_size()
    d2h = out_h.numel() * out_h.element_size()

    launches = m.mlg_forward_launch_count(w.n_atoms, w.rcut, s["box"], s["pbc"], w.nnei_max,
                                          w.channels, w.heads, w.n_layers, mdt)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_oracle_timing(w, s, W, args.cpu_seconds, args.seed)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value,
            "unit": "atoms/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": DATA,
            "config": workload_config(w, args), "n_edges": E,
            "roofline": roofline,
            "roofline_build": roofline_build,
            "stages": {"build_ms": build_avg, "attention_ms": attn_avg,
                       "n_layers": w.n_layers, "attention_share_of_step": layers_share},
            "e2e": {"value": e2e_value, "unit": "atoms/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_total / args.steps,
                    "pipelined": True, "latency_ms_per_step": lat_total / args.steps},
            "gpu_launches": launches * args.steps,
            "clocks": sampler.summary(t0, t1),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
