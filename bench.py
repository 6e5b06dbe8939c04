"""Benchmark of the batched Muon update (cubic Newton-Schulz) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b]
                    [--impl ours|reference]

One step = one dmuon_muon_step_batched call over the whole workload (momentum,
Nesterov, normalisation, k Newton-Schulz steps, weight update) with its
inputs resident in HBM.  The metric is useful Newton-Schulz throughput: per
matrix and NS step, m^2 n FLOPs for X X^T plus 2 m^2 n for (X X^T) X, with
m = min(rows, cols), n = max(rows, cols).

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of the
workload (weak scaling, no collective on the data path); the step time is the
maximum over ranks and `value` adds up all ranks' FLOPs.

--impl reference times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload and in the same unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "Muon-step ms & NS TFLOP/s (Llama-8B shapes), % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
NOMINAL_BF16_TFLOPS = 2250.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the GEMM stage: the ncu
# capture of one Llama-8B layer's GEMM on CTA pairs (631.8 MB read + 413.2 MB written for
# 1.735e12 useful FLOPs); a launch of the full workload covers several layers, so its traffic is
# this ratio times the useful FLOPs of that launch.  Valid only for the stage kernels' source it
# was measured on (ns_stage.cuh, gemm_pair.cuh and ptx.cuh).
PROFILED_TRAFFIC = {"kernel_sha256_prefix": "eee49fdfaf9de58a", "workload": "llama8b",
                    "gemm_bytes_per_useful_flop": 1.0450e9 / 1.735e12}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--impl", choices=["ours", "reference", "torch"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-adamw", action="store_true")
    ap.add_argument("--adamw-only", type=int, default=0, metavar="ROWS",
                    help="time only the AdamW leg, with embedding and head of ROWS x 4096 "
                         "(128256 for Llama-8B; smaller for a profiler capture)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' lines (the `configs` key)")
    ap.add_argument("--no-clip", action="store_true")
    ap.add_argument("--no-quintic", action="store_true")
    ap.add_argument("--clip-only", action="store_true",
                    help="time only the per-segment clipping leg (for a profiler capture)")
    return ap.parse_args()


def profiled_traffic(workload: str):
    """The profiled DRAM bytes per useful GEMM FLOP, or None when the stage kernel's source
    changed since."""
    import hashlib
    csrc = os.path.join(HERE, "newton_schulz_09_b200", "csrc")
    try:
        data = b"".join(open(os.path.join(csrc, f), "rb").read()
                        for f in ("ns_stage.cuh", "gemm_pair.cuh", "ptx.cuh"))
    except OSError:
        return None
    sha = hashlib.sha256(data).hexdigest()
    if sha.startswith(PROFILED_TRAFFIC["kernel_sha256_prefix"]) and workload == PROFILED_TRAFFIC["workload"]:
        return PROFILED_TRAFFIC["gemm_bytes_per_useful_flop"]
    return None


def load_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- dist
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def min_over_ranks(x: float, world: int, device) -> float:
    return -max_over_ranks(-x, world, device)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU oracle
def cpu_sample_specs(wl):
    """A bounded sample of the workload for the fp64 oracle: the first layer's
    attention projections for the Llama stack, else the first matrices, up to
    about 2e12 useful FLOPs (10-30 s on a many-core host)."""
    from newton_schulz_09_b200 import synthetic
    budget = 2.2e12
    chosen, fl = [], 0.0
    order = range(len(wl.specs))
    if wl.name == "llama8b":
        order = [0, 1, 2, 3]          # layer 0: q, k, v, o
    for i in order:
        s = wl.specs[i]
        f = 3.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) * wl.ns_steps
        if chosen and fl + f > budget:
            break
        chosen.append(i)
        fl += f
    return chosen, fl


def time_oracle(wl, subset):
    """Runs the oracle's Muon step on host copies of the subset; returns
    (seconds, threads)."""
    import numpy as np
    import oracle
    from newton_schulz_09_b200 import synthetic
    t = synthetic.make_tensors(wl, device="cpu", subset=subset)
    host = [(p.float().numpy(), g.float().numpy(), b.numpy())
            for p, g, b in zip(t.params, t.grads, t.bufs)]
    threads = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        info = [d for d in threadpool_info() if d.get("internal_api") == "openblas"]
        if info:
            threads = int(info[0]["num_threads"])
    except Exception:
        pass
    t0 = time.perf_counter()
    for W, g, b in host:
        oracle.muon_step(W, g, b, lr=wl.lr, momentum=wl.momentum, nesterov=wl.nesterov,
                         weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)
    dt = time.perf_counter() - t0
    del np
    return dt, threads


def cpu_baseline(wl):
    subset, fl = cpu_sample_specs(wl)
    secs, threads = time_oracle(wl, subset)
    names = ",".join(f"{wl.specs[i].name}({wl.specs[i].rows}x{wl.specs[i].cols})" for i in subset)
    return {"value": fl / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"one Muon step (k={wl.ns_steps}) of {names}: {fl:.3e} useful NS FLOPs "
                      f"in {secs:.2f} s, fp64 numpy/OpenBLAS"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from newton_schulz_09_b200 import synthetic
    wl = synthetic.workload(args.workload)
    subset, fl = cpu_sample_specs(wl)
    for _ in range(max(0, args.warmup)):
        pass   # the oracle has no warm-up state; each step is timed as it stands
    secs = []
    threads = 1
    for _ in range(args.steps):
        s, threads = time_oracle(wl, subset)
        secs.append(s)
    tot = sum(secs)
    value = fl * len(secs) / tot / 1e12
    names = ",".join(wl.specs[i].name for i in subset)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / len(secs) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "sample": names, "ns_steps": wl.ns_steps},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"each step: one Muon step of {names} ({fl:.3e} FLOPs)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- ours
def measure_adamw(dm, dev, stream, world, peaks, steps, rows=128256):
    """AdamW over the Llama-8B parameters that are not 2-D projections: token
    embedding and LM head (``rows`` = 128256 x 4096 each) and 65 norm weights
    (4096), bf16 parameters and gradients, fp32 moments; 22 algorithmic bytes
    per element (p read+write 4, g 2, m and v read+write 16)."""
    import torch
    shapes = [(rows * 4096,), (rows * 4096,)] + [(4096,)] * 65
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    ps = [(torch.randn(s, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for s in shapes]
    gs = [(torch.randn(s, generator=gen, device=dev) * 1e-3).to(torch.bfloat16) for s in shapes]
    ms = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
    vs = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
    n = sum(s[0] for s in shapes)
    for t in range(1, 4):
        dm.dmuon_adamw_step_batched(ps, gs, ms, vs, step=t)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(4, 4 + steps):
        dm.dmuon_adamw_step_batched(ps, gs, ms, vs, step=t)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_step = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    gbs = 22.0 * n / (ms_step * 1e-3) / 1e9
    out = {"elements": n, "ms_per_step": ms_step, "achieved": gbs, "unit": "GB/s",
           "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"], "bound": "hbm",
           "bytes_per_element": 22}
    del ps, gs, ms, vs
    torch.cuda.empty_cache()
    return out


QUINTIC = (3.4445, -4.7750, 2.0315)   # a widely used quintic set (not from the pages)


def llama_clip_segments(t, dev, rows=128256):
    """The three gradient groups of a Llama-8B step for the per-segment clip:
    regular (embedding and LM head, rows x 4096 each), Muon (the 224
    projections' gradients) and AdamW (65 norm vectors), bf16."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    regular = [(torch.randn((rows, 4096), generator=gen, device=dev) * 1e-4).to(torch.bfloat16)
               for _ in range(2)]
    norms = [(torch.randn((4096,), generator=gen, device=dev) * 1e-4).to(torch.bfloat16) for _ in range(65)]
    return [regular, list(t.grads), norms]


def measure_clip(dm, dev, stream, world, peaks, steps, segments):
    """Per-segment clipping of the three gradient groups.  Every timed pass
    clips every segment (each step's bound is half the norm the gradients
    had before it, so every coefficient is about 0.5 and the scale pass
    rewrites everything): algorithmic bytes per bf16 element are 2 (norm pass)
    + 2 + 2 (scale pass read and write)."""
    import math
    import torch
    n = sum(g.numel() for seg in segments for g in seg)
    norms, _ = dm.dmuon_clip_grad_norm_buckets(segments, [math.inf] * len(segments))
    torch.cuda.synchronize(dev)
    cur = [float(x) for x in norms.cpu()]
    for _ in range(3):                                         # warm-up passes, also clipping
        dm.dmuon_clip_grad_norm_buckets(segments, [0.5 * c for c in cur])
        cur = [0.5 * c for c in cur]
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        dm.dmuon_clip_grad_norm_buckets(segments, [0.5 * c for c in cur])
        cur = [0.5 * c for c in cur]
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_step = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    gbs = 6.0 * n / (ms_step * 1e-3) / 1e9
    return {"elements": n, "segments": [sum(g.numel() for g in seg) for seg in segments],
            "ms_per_step": ms_step, "achieved": gbs, "unit": "GB/s", "peak": peaks["hbm_gbs"],
            "frac": gbs / peaks["hbm_gbs"], "bound": "hbm", "bytes_per_element": 6,
            "note": "three segments (regular: embedding + head, Muon: 224 projections, AdamW: norms), "
                    "each clipped with its own norm; bf16"}


def measure_quintic(dm, t, wl, dev, stream, world, peaks, steps):
    """The Llama-8B step with quintic coefficients: SYRK, the symmetric square
    P = b A + c A A and the GEMM X <- a X + P X per NS step.  Useful FLOPs per
    matrix and NS step: m^2 n + m^3 + 2 m^2 n."""
    import torch
    fl = wl.ns_steps * sum(3.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) + min(s.rows, s.cols) ** 3
                           for s in wl.specs)

    def step():
        dm.dmuon_muon_step_batched_opts(t.params, t.grads, t.bufs, lr=wl.lr, momentum=wl.momentum,
                                        nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                                        ns_steps=wl.ns_steps, ns_coefficients=QUINTIC)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    dm.dmuon_stage_times(reset=True)
    dm.dmuon_stage_timing(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dm.dmuon_stage_timing(False)
    stages = dm.dmuon_stage_times(reset=True)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    tf = fl / (ms * 1e-3) / 1e12
    return {"coefficients": list(QUINTIC), "ms_per_step": ms, "useful_flops_per_step": fl,
            "tflops": tf, "frac_sustained": tf / peaks["bf16_tflops_sustained"],
            "stage_ms_per_step": {k: v[0] / steps for k, v in stages.items() if v[1]}}


def config_sample(wl, budget):
    """Matrices of a workload for the oracle: all of them when their useful
    FLOPs fit the budget, else the first ones in draw order up to it."""
    chosen, fl = [], 0.0
    for i, s in enumerate(wl.specs):
        f = 3.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) * wl.ns_steps
        if chosen and fl + f > budget:
            break
        chosen.append(i)
        fl += f
    return chosen, fl


def measure_config(name, dm, dev, peaks, steps, cpu):
    """One of the other workloads: Muon-step time on the GPU (inputs resident,
    CUDA events), useful TFLOP/s and the fractions of the peaks, and, when
    ``cpu``, the fp64 oracle's time for the same step on the host cores (in
    full for the small workloads, else on a stated sample).  square4096 adds
    the step-count sweep of the orthogonality error."""
    import torch
    from newton_schulz_09_b200 import synthetic
    wl = synthetic.workload(name)
    t = synthetic.make_tensors(wl, device=dev, flat=True)
    fl = synthetic.ns_flops(wl)
    stream = torch.cuda.current_stream(dev)
    host = None
    if cpu:
        sub, _ = config_sample(wl, 2.2e12)
        host = [(t.params[i].float().cpu().numpy(), t.grads[i].float().cpu().numpy(),
                 t.bufs[i].cpu().numpy()) for i in sub]
        prior = [[g.float().cpu().numpy() for j, g in enumerate(step_g) if j in sub]
                 for step_g in t.prior_grads]
    # the momentum history (R14): prior steps with lr = 0, then the measured step
    for gs in t.prior_grads:
        dm.dmuon_muon_step_batched(t.params, gs, t.bufs, lr=0.0, momentum=wl.momentum,
                                   nesterov=wl.nesterov, weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)

    def step():
        dm.dmuon_muon_step_batched(t.params, t.grads, t.bufs, lr=wl.lr, momentum=wl.momentum,
                                   nesterov=wl.nesterov, weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    tf = fl / (ms * 1e-3) / 1e12
    # per-stage device time, from a few more steps with each launch bracketed
    # by events (kept out of the timed steps above)
    dm.dmuon_stage_times(reset=True)
    dm.dmuon_stage_timing(True)
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    dm.dmuon_stage_timing(False)
    stages = {k: v[0] / 3 for k, v in dm.dmuon_stage_times(reset=True).items() if v[1]}
    out = {"workload": name, "matrices": len(wl.specs), "ns_steps": wl.ns_steps,
           "dtype": "f32 (tf32 operands)" if wl.dtype == torch.float32 else "bf16",
           "useful_flops_per_step": fl, "ms_per_step": ms, "tflops": tf,
           "pct_of_bf16_peak": {"measured_sustained": tf / peaks["bf16_tflops_sustained"],
                                "measured_burst": tf / peaks["bf16_tflops"],
                                "nominal_2250": tf / NOMINAL_BF16_TFLOPS},
           "stage_ms_per_step": stages}
    if name == "mixed1024":
        out["small_matrices"] = measure_small_class(dm, dev, wl, t, peaks, steps)
    sweep = None
    if name == "square4096":
        sweep = []
        G = t.grads[0]
        eye = torch.eye(G.shape[0], dtype=torch.float64, device=dev)
        for k in (3, 5, 7, 10):
            Y = G.clone()
            dm.dmuon_ns_orthogonalize(Y, k)
            Yd = Y.double()
            err = float(torch.linalg.norm(Yd @ Yd.T - eye))
            sweep.append({"k": k, "orthogonality_error_gpu": err})
        out["sweep"] = sweep
    if cpu:
        out["cpu_baseline"] = oracle_config_time(wl, host, prior, sub, sweep, G=t.grads[0] if sweep else None)
    del t
    torch.cuda.empty_cache()
    return out


def measure_small_class(dm, dev, wl, t, peaks, steps, max_side=256):
    """The mixed workload's narrow matrices (short side <= max_side) as a call of
    their own.  Their Newton-Schulz work is too small to bound them by the tensor
    cores, so they are reported against HBM: 16 bytes of unavoidable traffic per
    element (gradient 2, momentum read and write 8, X0 2, weight read and write
    4; the iterates of matrices this small stay in L2)."""
    import torch
    idx = [i for i, s in enumerate(wl.specs) if min(s.rows, s.cols) <= max_side]
    if not idx:
        return None
    ps, gs, bs = [t.params[i] for i in idx], [t.grads[i] for i in idx], [t.bufs[i] for i in idx]

    def step():
        dm.dmuon_muon_step_batched(ps, gs, bs, lr=wl.lr, momentum=wl.momentum, nesterov=wl.nesterov,
                                   weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)

    for _ in range(3):
        step()
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    elems = sum(wl.specs[i].rows * wl.specs[i].cols for i in idx)
    fl = wl.ns_steps * sum(3.0 * min(wl.specs[i].rows, wl.specs[i].cols) ** 2 *
                           max(wl.specs[i].rows, wl.specs[i].cols) for i in idx)
    hbm = 16.0 * elems
    gbs = hbm / (ms * 1e-3) / 1e9
    return {"max_short_side": max_side, "matrices": len(idx), "elements": elems,
            "ms_per_step": ms, "useful_flops_per_step": fl, "tflops": fl / (ms * 1e-3) / 1e12,
            "bound": "hbm", "hbm_bytes_per_step": hbm, "achieved_gbs": gbs,
            "frac_of_hbm": gbs / peaks["hbm_gbs"],
            "note": "one call of these matrices alone; launch and pipeline-fill latency, not HBM "
                    "bandwidth, sets most of the time"}


def oracle_config_time(wl, host, prior, sub, sweep, G=None):
    """The fp64 oracle on the host cores: the same Muon step (after the same
    momentum history) for the sampled matrices; for square4096 also the
    orthogonality error of the oracle's iterate after 3, 5, 7 and 10 steps."""
    import numpy as np
    import oracle
    threads = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        info = [d for d in threadpool_info() if d.get("internal_api") == "openblas"]
        if info:
            threads = int(info[0]["num_threads"])
    except Exception:
        pass
    fl = sum(3.0 * min(wl.specs[i].rows, wl.specs[i].cols) ** 2 * max(wl.specs[i].rows, wl.specs[i].cols)
             * wl.ns_steps for i in sub)
    t0 = time.perf_counter()
    for k, (W, g, b) in enumerate(host):
        for gs in prior:
            b, _, _ = oracle.muon_step(W, gs[k], b, lr=0.0, momentum=wl.momentum, nesterov=wl.nesterov,
                                       weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)
        oracle.muon_step(W, g, b, lr=wl.lr, momentum=wl.momentum, nesterov=wl.nesterov,
                         weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)
    secs = time.perf_counter() - t0
    steps_run = 1 + len(prior)
    res = {"value": fl * steps_run / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
           "seconds": secs,
           "sample": (f"all {len(sub)} matrices" if len(sub) == len(wl.specs) else
                      f"the first {len(sub)} of {len(wl.specs)} matrices in draw order") +
                     f", {steps_run} Muon step(s) of {fl:.3e} useful FLOPs each, fp64 numpy/OpenBLAS"}
    if sweep is not None:
        X = oracle.frobenius_normalize(G.float().cpu().numpy())
        done = 0
        for entry in sweep:
            for _ in range(entry["k"] - done):
                X = oracle.ns_iteration(X)
            done = entry["k"]
            entry["orthogonality_error_oracle"] = oracle.orthogonality_error(X)
    return res


def run_clip_only(args):
    """The per-segment clipping leg alone on the Llama-8B gradients (one
    GPU): its own JSON line, GB/s of algorithmic traffic against the
    measured copy bandwidth."""
    import torch
    import newton_schulz_09_b200 as dm
    from newton_schulz_09_b200 import synthetic
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dm.load_library()
    peaks, peak_src = load_peaks()
    wl = synthetic.workload(args.workload)
    t = synthetic.make_tensors(wl, device=dev, flat=True)
    segs = llama_clip_segments(t, dev, rows=128256 if wl.name == "llama8b" else 8192)
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    c = measure_clip(dm, dev, torch.cuda.current_stream(dev), 1, peaks, args.steps, segs)
    clocks = sampler.stop()
    print(json.dumps({
        "metric": "per-segment gradient clipping GB/s", "value": c["achieved"], "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": 3, "ms_per_step": c["ms_per_step"],
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic", "clocks": clocks,
        "config": {"workload": f"{wl.name} gradients in three segments", "elements": c["elements"],
                   "bytes_per_element": 6},
        "roofline": {"bound": "hbm", "achieved": c["achieved"], "peak": c["peak"], "unit": "GB/s",
                     "frac": c["frac"], "peak_source": f"{peak_src} hbm_gbs"}}))
    return 0


def run_ours(args):
    import torch
    import newton_schulz_09_b200 as dm
    from newton_schulz_09_b200 import synthetic

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    dm.load_library()
    peaks, peak_src = load_peaks()

    wl = synthetic.workload(args.workload)
    t = synthetic.make_tensors(wl, device=dev, flat=True, seed_offset=rank)
    stream = torch.cuda.current_stream(dev)
    fl = synthetic.ns_flops(wl)

    def step():
        dm.dmuon_muon_step_batched(t.params, t.grads, t.bufs, lr=wl.lr, momentum=wl.momentum,
                                   nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                                   ns_steps=wl.ns_steps)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    status = dm.dmuon_device_status()
    if status != 0:
        raise RuntimeError(f"device error word {status} after warm-up")

    # ---- device-timed region (inputs resident in HBM, larger than L2)
    sampler = ClockSampler(dev.index)
    dm.dmuon_stage_times(reset=True)
    dm.dmuon_stage_timing(True)
    launches0 = dm.dmuon_launch_count()
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    launches = dm.dmuon_launch_count() - launches0
    dm.dmuon_stage_timing(False)
    stages = dm.dmuon_stage_times(reset=True)
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, world, dev)
    value = fl * world / (ms * 1e-3) / 1e12

    # ---- roofline of the dominant kernel (the GEMM stage: 2 m^2 n per NS step).
    # The library runs a large call as groups of matrices, so a step has several
    # GEMM launches per NS step; rates use the step's totals (= the launches'
    # FLOP-weighted average), traffic is per average launch.
    gemm_ms, gemm_n = stages["gemm"]
    syrk_ms, syrk_n = stages["syrk"]
    gemm_fl_step = wl.ns_steps * sum(2.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) for s in wl.specs)
    syrk_fl_step = wl.ns_steps * sum(1.0 * min(s.rows, s.cols) ** 2 * max(s.rows, s.cols) for s in wl.specs)
    peak = peaks["bf16_tflops_sustained"]
    gemm_tf = gemm_fl_step / (gemm_ms / args.steps * 1e-3) / 1e12 if gemm_n else None
    syrk_tf = syrk_fl_step / (syrk_ms / args.steps * 1e-3) / 1e12 if syrk_n else None
    gemm_launches_step = gemm_n / args.steps if gemm_n else None
    fl_per_launch = gemm_fl_step / gemm_launches_step if gemm_n else None
    bpf = profiled_traffic(wl.name)
    plan = dm.dmuon_debug_last_plan()
    pair = bool(plan) and all(g["gemm_pair"] for g in plan)
    roofline = {
        "kernel": "gemm_pair_kernel (256 x 256 tiles on CTA pairs, bf16)" if pair
                  else "ns_stage_kernel<GEMM, bf16>",
        "bound": "tensor",
        "achieved": gemm_tf, "peak": peak, "unit": "TFLOP/s",
        "frac": (gemm_tf / peak) if gemm_tf else None,
        "traffic": (bpf * fl_per_launch) if (bpf and fl_per_launch) else None,
        "traffic_unit": "DRAM bytes per average launch (ncu one-layer capture, scaled by useful FLOPs)",
        "launches_per_step": gemm_launches_step, "useful_flop_per_launch": fl_per_launch,
        "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
        "syrk": {"achieved": syrk_tf, "frac": (syrk_tf / peak) if syrk_tf else None},
        "stage_ms_per_step": {k: v[0] / args.steps for k, v in stages.items() if v[1]},
    }
    # The prologue against the HBM roofline: per element it reads the gradient
    # and the fp32 momentum and writes the momentum and the iterate X.
    pro_ms, pro_n = stages["prologue"]
    if pro_n:
        eb = torch.tensor([], dtype=wl.dtype).element_size()
        pro_bytes = wl.numel * (eb + 4 + 4 + eb)
        pro_gbs = pro_bytes / (pro_ms / args.steps * 1e-3) / 1e9
        roofline["prologue"] = {"bound": "hbm", "achieved": pro_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": pro_gbs / peaks["hbm_gbs"], "bytes_per_element": eb + 4 + 4 + eb,
                                "peak_source": f"{peak_src} hbm_gbs"}

    # ---- AdamW of the model's non-orthogonalised parameters (HBM-bound leg)
    adamw = None
    if not args.no_adamw and wl.name == "llama8b":
        adamw = measure_adamw(dm, dev, stream, world, peaks, args.steps)

    # ---- end to end through the public API: pinned host grads in, weights out.
    # dmuon_muon_step_batched_host uploads each group's gradients, updates it
    # and downloads its weights, with the copies overlapped with the kernels.
    e2e = None
    e2e_ok = not args.no_e2e
    if e2e_ok:
        # Every rank of this node pins its own gradient and weight copies; skip
        # the leg (on every rank alike) when the host cannot hold them all.
        import psutil
        pflat, gflat, _ = t.flat
        pin_bytes = pflat.numel() * pflat.element_size() + gflat.numel() * gflat.element_size()
        local_ranks = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
        fits = psutil.virtual_memory().available > 1.3 * pin_bytes * local_ranks
        if min_over_ranks(1.0 if fits else 0.0, world, dev) < 1.0:
            e2e_ok = False
            e2e = {"value": None, "skipped": f"host memory: {local_ranks} ranks x {pin_bytes / 1e9:.0f} GB "
                                             f"pinned exceeds the available RAM"}
    if e2e_ok:
        pflat, gflat, _ = t.flat
        h_g = torch.empty(gflat.shape, dtype=gflat.dtype, pin_memory=True)
        h_g.copy_(gflat)
        h_w = torch.empty(pflat.shape, dtype=pflat.dtype, pin_memory=True)

        def host_view(flat_h, flat_d, views):
            out = []
            for v in views:
                off = (v.data_ptr() - flat_d.data_ptr()) // v.element_size()
                out.append(flat_h[off:off + v.numel()].view(v.shape))
            return out

        hg = host_view(h_g, gflat, t.grads)
        hw = host_view(h_w, pflat, t.params)

        def host_step():
            dm.dmuon_muon_step_batched_host(t.params, t.grads, t.bufs, hg, hw, lr=wl.lr,
                                            momentum=wl.momentum, nesterov=wl.nesterov,
                                            weight_decay=wl.weight_decay, ns_steps=wl.ns_steps)

        host_step()                                  # plans and copy streams
        barrier(world)
        torch.cuda.synchronize(dev)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            host_step()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        if not torch.equal(h_w[:4096], pflat[:4096].cpu()):
            raise RuntimeError("downloaded weights differ from the device weights")
        e2e_ms = max_over_ranks(a0.elapsed_time(a1) / args.e2e_steps, world, dev)
        e2e = {"value": fl * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": gflat.numel() * gflat.element_size(),
               "d2h_bytes_per_step": pflat.numel() * pflat.element_size(),
               "api": "dmuon_muon_step_batched_host (pinned host buffers, copies overlapped)"}
        del h_g, h_w, hg, hw

    # ---- per-segment clipping of the step's three gradient groups (HBM-bound)
    clip = None
    if not args.no_clip and wl.name == "llama8b":
        segs = llama_clip_segments(t, dev)
        clip = measure_clip(dm, dev, stream, world, peaks, args.steps, segs)
        del segs
        torch.cuda.empty_cache()

    # ---- the same stack with quintic coefficients (one more symmetric product)
    quintic = None
    if not args.no_quintic and wl.name in ("llama8b", "llama8b_layer"):
        quintic = measure_quintic(dm, t, wl, dev, stream, world, peaks, 3)

    status = dm.dmuon_device_status()
    if status != 0:
        raise RuntimeError(f"device error word {status}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    # ---- the other workloads, one entry each (single-GPU runs only)
    configs = None
    if world == 1 and not args.no_configs:
        del t
        dm.dmuon_release_cache()
        torch.cuda.empty_cache()
        configs = []
        for name in ("fp32_256x512", "tinymlp", "square4096", "mixed1024"):
            if name == wl.name:
                continue
            configs.append(measure_config(name, dm, dev, peaks, 3 if name == "mixed1024" else 10,
                                          cpu=not args.no_cpu_baseline))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "pct_of_bf16_peak": {
                "measured_sustained": value / world / peaks["bf16_tflops_sustained"],
                "measured_burst": value / world / peaks["bf16_tflops"],
                "nominal_2250": value / world / NOMINAL_BF16_TFLOPS,
                "peak_source": peak_src},
            "config": {"workload": wl.name, "matrices": len(wl.specs), "ns_steps": wl.ns_steps,
                       "useful_ns_flops_per_step_per_gpu": fl,
                       "l2": f"inputs larger than L2 ({wl.numel * 8 / 1e9:.0f} GB per GPU)",
                       "parallelism": f"replicas x{world}"},
            "clocks": clocks, "e2e": e2e, "gpu_launches": launches, "adamw": adamw,
            "roofline": roofline, "cpu_baseline": cpu, "clip": clip, "quintic": quintic,
            "configs": configs,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- torch eager
def run_torch(args):
    """Context arm, not the product: the same step written as plain PyTorch
    eager code, the per-parameter loop of the blog's Vanilla Muon with the
    Newton-Schulz products in bf16 through torch.matmul (cuBLAS).  It forms
    the full X X^T (4 m^2 n FLOPs per step); the rate below still counts the
    3 m^2 n useful FLOPs, as for the product."""
    import torch
    from newton_schulz_09_b200 import synthetic

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    wl = synthetic.workload(args.workload)
    t = synthetic.make_tensors(wl, device=dev, flat=True, seed_offset=rank)
    fl = synthetic.ns_flops(wl)
    mu, lr, wd, k = wl.momentum, wl.lr, wl.weight_decay, wl.ns_steps

    @torch.no_grad()
    def step():
        for p, g, buf in zip(t.params, t.grads, t.bufs):
            buf.mul_(mu).add_(g)
            M = g.float().add(buf, alpha=mu) if wl.nesterov else buf
            X = M.to(torch.bfloat16)
            tall = X.shape[0] > X.shape[1]
            if tall:
                X = X.T
            X = X / (X.norm() + 1e-7)
            for _ in range(k):
                A = X @ X.T
                X = 1.5 * X - 0.5 * (A @ X)
            if tall:
                X = X.T
            p.mul_(1.0 - lr * wd).add_(X.to(p.dtype), alpha=-lr)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    if rank == 0:
        print(json.dumps({
            "impl": "torch-eager", "metric": METRIC, "value": fl * world / (ms * 1e-3) / 1e12,
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "dtype": "bf16",
            "data": "synthetic", "clocks": clocks,
            "config": {"workload": wl.name, "matrices": len(wl.specs), "ns_steps": k,
                       "note": "per-matrix torch eager loop, NS products by torch.matmul (cuBLAS)"}}))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_adamw_only(args):
    """The AdamW leg alone (one GPU): its own JSON line, GB/s of algorithmic
    traffic against the measured copy bandwidth."""
    import torch
    import newton_schulz_09_b200 as dm
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dm.load_library()
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    a = measure_adamw(dm, dev, torch.cuda.current_stream(dev), 1, peaks, args.steps, rows=args.adamw_only)
    clocks = sampler.stop()
    print(json.dumps({
        "metric": "AdamW step GB/s (Llama-8B embedding, head and norms)", "value": a["achieved"],
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": 3, "ms_per_step": a["ms_per_step"],
        "higher_is_better": True, "dtype": "f32", "data": "synthetic", "clocks": clocks,
        "config": {"workload": f"adamw {args.adamw_only}x4096 x2 + 65x4096", "elements": a["elements"],
                   "bytes_per_element": 22, "l2": "inputs larger than L2" if 22 * a["elements"] > 126e6
                   else "inputs within L2"},
        "roofline": {"bound": "hbm", "achieved": a["achieved"], "peak": a["peak"], "unit": "GB/s",
                     "frac": a["frac"], "peak_source": f"{peak_src} hbm_gbs"}}))
    return 0


def main():
    args = parse_args()
    if args.adamw_only > 0:
        return run_adamw_only(args)
    if args.clip_only:
        return run_clip_only(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.impl == "torch":
        return run_torch(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
