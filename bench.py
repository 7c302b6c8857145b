"""MXNorm forward benchmark on B200: GB/s and fraction of HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extras]

One step = one MXNorm forward (block absmax -> p-mean G -> 1/G * gamma ->
E8M0 scales + E4M3 codes, one kernel) over one batch of the workload, default
x bf16 [8192 x 4096] N(0,1) with 1% outlier channels x50, gamma = 1 + 0.1 N,
p = 2, nearest-even, row-major scales.  `value` is whole-job GB/s of algorithmic
bytes (read x 2 B/elem, write codes 1 B/elem and scales 1/32 B/elem, gamma and
G) with inputs resident in HBM; steps rotate over a pool of input/output sets
larger than 3x the L2, so no step reads another's data from L2.

Rank 0 prints one JSON line.  N > 1 runs one process per GPU (torchrun);
every rank processes its own batch (weak scaling, no collective on the data
path) and the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXNorm fwd GB/s & % HBM peak at d=4096, vs RMSNorm+MXCast two-pass"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0          # B200 HBM3e, HGX datasheet figure


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_8192x4096_outliers_p2")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the two-pass comparator, e2e and CPU baseline legs")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the sweep legs (16384 x {2048..16384}, p in {1,2,4,inf}, RNE/SR)")
    ap.add_argument("--soak-s", type=float, default=0.5,
                    help="untimed back-to-back steps before timing, so clocks settle under load")
    ap.add_argument("--profile-only", choices=["fwd", "sr", "mxfp4", "nvfp4", "bwd", "gemm", "sr_sweep"],
                    default=None,
                    help="run only this kernel, 8 launches on the workload with inputs and outputs "
                         "rotating over 4 sets, untimed (for ncu captures); "
                         "sr_sweep: two stochastic-rounding launches per sweep shape (T = 16384, p = 2)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def workload_cfg(name):
    from normalisation_row_bf16_b200 import synthetic
    w = dict(synthetic.WORKLOADS[name])
    w.setdefault("p", 2.0)
    return w


def algorithmic_bytes(T, D):
    # read x (2 B/elem), write E4M3 codes (1 B/elem) and E8M0 scales (1 per 32),
    # read gamma (2 B/column), write G (4 B/row)
    return T * D * 2 + T * D + T * (D // 32) + 2 * D + 4 * T


def two_pass_bytes(T, D):
    # RMSNorm: read x, write y (bf16); MXCast: read y, write codes + scales; gamma
    return T * D * 2 * 2 + T * D * 2 + T * D + T * (D // 32) + 2 * D


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def kernel_source_hash():
    """Hash of the forward kernel's own sources (the profile's traffic figure is
    used only while they are unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "normalisation_row_bf16_b200", "csrc")
    for name in ("device_common.cuh", "row_fwd.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profile_fields(name):
    """The "- key: value" fields of a committed ncu summary under profiles/, if
    it was taken on the current kernel sources (else {})."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return {}
    fields = {}
    for line in open(path):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_hash") != kernel_source_hash():
        return {}
    return fields


def _int_field(fields, key):
    try:
        return int(fields[key])
    except (KeyError, ValueError):
        return None


def profiled_traffic(workload):
    """DRAM bytes per launch (steady state: the mean over captured launches that
    follow other launches) from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    return _int_field(profile_fields(f"mxnorm_fwd_{workload}.md"), "dram_bytes_per_launch")


def profiled_traffic_split(workload):
    f = profile_fields(f"mxnorm_fwd_{workload}.md")
    r, w = _int_field(f, "dram_read_bytes_per_launch"), _int_field(f, "dram_write_bytes_per_launch")
    return None if r is None or w is None else {"read": r, "write": w}


def profiled_instructions(name, key):
    """Thread instructions per element of a kernel from a committed ncu summary
    (current sources only), else None."""
    try:
        return float(profile_fields(name)[key])
    except (KeyError, ValueError):
        return None


def issue_peak(sm_mhz):
    """Lane-instructions per second the SMs can issue: 148 SMs x 4 schedulers x
    one warp-instruction (32 lanes) per clock, at the sampled SM clock."""
    return 148 * 4 * 32 * sm_mhz * 1e6


def alu_roofline(instr_per_elem, elements, ms, sm_mhz):
    """Issue-rate roofline of a launch: thread instructions per element (from
    the committed ncu summary of the same kernel and workload) times the
    elements, over the launch time, against the issue peak at the sampled SM
    clock.  None when either figure is missing."""
    if not instr_per_elem or not sm_mhz:
        return None
    achieved = instr_per_elem * elements / (ms * 1e-3)
    peak = issue_peak(sm_mhz)
    return {"bound": "alu", "instr_per_elem": round(instr_per_elem, 2), "achieved_Tinstr_s": round(achieved / 1e12, 2),
            "peak_Tinstr_s": round(peak / 1e12, 2), "frac": round(achieved / peak, 4), "sm_mhz": sm_mhz}


def compact(leg, extra=None):
    """A graph leg's record as the bench line carries it: time per launch,
    GB/s of algorithmic bytes and the fraction of the HBM peak."""
    out = {"us": round(leg["ms"] * 1e3, 2), "GBps": leg["GBps"], "frac": leg["roofline"]["frac"]}
    if extra:
        out.update(extra)
    return out


def device_hold():
    """Queue a short spin kernel (torch's, about 0.25 ms) ahead of a timed
    region's start event.  The device is then busy while the host enqueues the
    start event and the graph, so the region starts when the device reaches it
    and the first step does not include the host's graph-launch latency."""
    import torch
    torch.cuda._sleep(500_000)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        power = [float(r[3]) for r in self.rows if r[3].replace(".", "").isdigit()]
        reasons = sorted({self.NAMES[i] for r in self.rows for i in range(4) if r[5 + i] == "Active"})
        # samples under load: the upper half by power draw
        loaded = sm
        if power and len(power) == len(sm):
            cut = statistics.median(power)
            loaded = [s for s, p in zip(sm, power) if p >= cut] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from normalisation_row_bf16_b200 import build as nbuild
    from normalisation_row_bf16_b200 import ops, synthetic

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if rank == 0:
        nbuild.build()
    if world > 1:
        dist.barrier()
    ops.lib()
    w = workload_cfg(args.workload)
    T, D, p = w["T"], w["D"], w["p"]
    nbytes = algorithmic_bytes(T, D)
    set_bytes = T * D * 2 + T * D + T * (D // 32) + 4 * T
    n_sets = max(2, math.ceil(3 * L2_BYTES / set_bytes))

    x0 = synthetic.activations(T, D, w["kind"], seed=rank, device=dev)
    g = synthetic.gamma(D, seed=rank, device=dev)
    xs = [x0] + [x0.clone() for _ in range(n_sets - 1)]
    outs = [(torch.empty(T, D, dtype=torch.uint8, device=dev),
             torch.empty(T, D // 32, dtype=torch.uint8, device=dev),
             torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n_sets)]

    def step(i):
        q, s, G = outs[i % n_sets]
        ops.mxnorm_fwd(xs[i % n_sets], g, p, q=q, scales=s, G=G)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}") if rank == 0 else None

    for i in range(args.warmup):
        step(i)
    # untimed soak so that the sampled clocks reflect the loaded state
    barrier()
    t_end = time.time() + args.soak_s
    i = 0
    while time.time() < t_end:
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize()

    # The K timed steps are captured once into a CUDA graph and replayed: every
    # kernel of every step runs, without the host's per-call dispatch between
    # them.  The per-launch time of the kernel is the region over K.
    K = args.steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(K):
            step(i)
    graph.replay()                     # untimed: first replay uploads the graph
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    device_hold()
    t0.record()
    graph.replay()
    t1.record()
    barrier()
    clocks = sampler.stop() if sampler else None
    region_ms = t0.elapsed_time(t1)
    kern_ms = [region_ms / K]
    del graph
    times = torch.tensor([region_ms, statistics.mean(kern_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    region_ms, mean_kern_ms = float(times[0]), float(times[1])
    ms_per_step = region_ms / K
    value = world * nbytes / (ms_per_step * 1e-3) / 1e9

    extras = {}
    if not args.no_extras:
        sm_mhz = (clocks or {}).get("sm_mhz") if rank == 0 else None
        extras = run_extras(args, w, rank, world, dev, xs, g, n_sets, barrier, ms_per_step, sm_mhz)

    if rank != 0:
        return None
    peaks, peak_src = measured_peaks()
    achieved = nbytes / (mean_kern_ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic(args.workload),
            "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json hbm_gbs' if peak_src == 'measured' else 'recipe fallback'})",
            "algorithmic_bytes_per_launch": nbytes,
            "kernel": "row_fwd_kernel<MXNorm>", "mean_launch_ms": round(mean_kern_ms, 6)}
    split = profiled_traffic_split(args.workload)
    if split:
        roof["traffic_read"], roof["traffic_write"] = split["read"], split["write"]
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": args.workload, "T": T, "D": D, "block": 32, "p": p, "rounding": "rne",
            "timing": "K steps captured in one CUDA graph, replayed between CUDA events "
                      "(a spin kernel queued ahead of the start event keeps the graph-launch latency out)",
            "gamma": True, "scale_layout": "rowmajor", "x": w["kind"],
            "l2": f"inputs rotate over {n_sets} sets of {set_bytes / 2**20:.0f} MiB "
                  f"({n_sets * set_bytes / 2**20:.0f} MiB > 3x the 126 MB L2)",
            "parallelism": f"replicas x{world}: each rank its own {T}-row batch, no collective",
            "clock_soak_s": args.soak_s,
        },
        "roofline": roof,
        "gpu_launches": K,
        "clocks": clocks,
    }
    # Bulky context first, the figures the summary reads last (a reader of the
    # line's tail sees them).
    order = ["cpu_baseline", "e2e", "stream_context", "gemm", "fold_weight", "pipeline_mxnorm_gemm",
             "pipeline_rmsnorm_mxcast_gemm", "pipeline_speedup", "mxfp4_fwd", "nvfp4_fwd", "scale_reuse_fwd",
             "sweep", "tiny", "bwd", "sr_fwd", "parity"]
    for k in order:
        if k in extras:
            line[k] = extras.pop(k)
    line.update(extras)
    line["tokens_per_s"] = round(world * T / (ms_per_step * 1e-3), 1)
    line["pct_hbm_nominal"] = round(100.0 * value / (world * NOMINAL_HBM_GBS), 2)
    line["pct_hbm_peak"] = round(100.0 * value / (world * peak), 2)
    for k in ("two_pass", "speedup_vs_two_pass"):
        if k in line:
            line[k] = line.pop(k)
    return line


def run_extras(args, w, rank, world, dev, xs, g, n_sets, barrier, ms_per_step, sm_mhz):
    """Two-pass comparator, end-to-end through host buffers, CPU oracle."""
    import torch
    import torch.distributed as dist
    from normalisation_row_bf16_b200 import ops, synthetic

    T, D, p = w["T"], w["D"], w["p"]
    out = {}
    # two-pass RMSNorm -> bf16 -> MXCast, same rotation
    n2 = max(2, math.ceil(3 * L2_BYTES / (T * D * 5)))
    tmp = [(torch.empty(T, D, dtype=torch.bfloat16, device=dev),
            torch.empty(T, D, dtype=torch.uint8, device=dev),
            torch.empty(T, D // 32, dtype=torch.uint8, device=dev)) for _ in range(n2)]
    xs2 = [xs[i % n_sets] for i in range(n2)]
    K2 = args.steps

    def step2(i):
        y, q, s = tmp[i % n2]
        ops.rmsnorm_then_mxcast(xs2[i % n2], g, 1e-5, y_tmp=y, q=q, scales=s)

    for i in range(args.warmup):
        step2(i)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        for i in range(K2):
            step2(i)
    g2.replay()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    device_hold()
    t0.record()
    g2.replay()
    t1.record()
    barrier()
    del g2
    tp = torch.tensor([t0.elapsed_time(t1) / K2], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tp, op=dist.ReduceOp.MAX)
    tp_ms = float(tp[0])
    out["two_pass"] = {"ms_per_step": round(tp_ms, 6), "timing": "same graph replay",
                       "GBps_own_bytes": round(world * two_pass_bytes(T, D) / (tp_ms * 1e-3) / 1e9, 1),
                       "kernels_per_step": 2}
    out["speedup_vs_two_pass"] = round(tp_ms / ms_per_step, 3)
    del tmp

    # end to end through the C ABI with pinned host buffers: the batch in row
    # chunks through three streams, so each chunk's host -> device copy, the
    # MXNorm call and its device -> host copies overlap the neighbours' (rows
    # are independent; nearest-even results do not depend on the chunking).
    # Consecutive steps overlap too: a chunk's copy in waits only for the
    # previous step's kernel on that chunk (its input buffer), and the kernel
    # only for the previous step's copies out of that chunk (its outputs), so
    # one step's copies out share the link's time with the next step's copies in.
    xh = xs[0].cpu().pin_memory()
    qh = torch.empty(T, D, dtype=torch.uint8).pin_memory()
    sh = torch.empty(T, D // 32, dtype=torch.uint8).pin_memory()
    Gh = torch.empty(T, dtype=torch.float32).pin_memory()
    xd = torch.empty_like(xs[0])
    qd = torch.empty(T, D, dtype=torch.uint8, device=dev)
    sd = torch.empty(T, D // 32, dtype=torch.uint8, device=dev)
    Gd = torch.empty(T, dtype=torch.float32, device=dev)
    n_chunks = 8 if T % 8 == 0 else 1
    rows = T // n_chunks
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_chunks)]
    ev_run = [torch.cuda.Event() for _ in range(n_chunks)]
    ev_out = [torch.cuda.Event() for _ in range(n_chunks)]
    main = torch.cuda.current_stream()

    def step_e2e(first):
        if first:                      # start after everything queued on the main stream
            for st in (s_in, s_run, s_out):
                st.wait_stream(main)
        for c in range(n_chunks):
            r0, r1 = c * rows, (c + 1) * rows
            if not first:
                s_in.wait_event(ev_run[c])      # the previous step's kernel has read xd[c]
            with torch.cuda.stream(s_in):
                xd[r0:r1].copy_(xh[r0:r1], non_blocking=True)
                ev_in[c].record(s_in)
            s_run.wait_event(ev_in[c])
            if not first:
                s_run.wait_event(ev_out[c])     # the previous step's outputs of chunk c are on the host
            with torch.cuda.stream(s_run):
                ops.mxnorm_fwd(xd[r0:r1], g, p, q=qd[r0:r1], scales=sd[r0:r1], G=Gd[r0:r1], stream=s_run)
                ev_run[c].record(s_run)
            s_out.wait_event(ev_run[c])
            with torch.cuda.stream(s_out):
                qh[r0:r1].copy_(qd[r0:r1], non_blocking=True)
                sh[r0:r1].copy_(sd[r0:r1], non_blocking=True)
                Gh[r0:r1].copy_(Gd[r0:r1], non_blocking=True)
                ev_out[c].record(s_out)

    def join():
        for st in (s_in, s_run, s_out):
            main.wait_stream(st)

    Ke = min(args.steps, 100)
    for i in range(3):
        step_e2e(i == 0)
    join()
    barrier()
    t0.record()
    for i in range(Ke):
        step_e2e(i == 0)
    join()
    t1.record()
    barrier()
    te = torch.tensor([t0.elapsed_time(t1) / Ke], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    te_ms = float(te[0])
    out["e2e"] = {"value": round(world * algorithmic_bytes(T, D) / (te_ms * 1e-3) / 1e9, 2),
                  "unit": "GB/s", "h2d_bytes_per_step": T * D * 2,
                  "d2h_bytes_per_step": T * D + T * (D // 32) + 4 * T,
                  "steps": Ke, "ms_per_step": round(te_ms, 4),
                  "pipeline": f"{n_chunks} row chunks over 3 streams (copy in, MXNorm, copy out), consecutive steps overlapped"}
    # the check a user would make: the pipelined host results equal one device call's
    torch.cuda.synchronize()
    q_ref, s_ref, G_ref = ops.mxnorm_fwd(xd, g, p)
    torch.cuda.synchronize()
    out["e2e"]["matches_single_call"] = bool(torch.equal(qh, q_ref.cpu()) and torch.equal(sh, s_ref.cpu())
                                             and torch.equal(Gh, G_ref.cpu()))

    # Every leg rotates whole input and output sets (> 3x L2), like the headline.
    outs = [(torch.empty(T, D, dtype=torch.uint8, device=dev), torch.empty(T, D // 32, dtype=torch.uint8, device=dev),
             torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n_sets)]
    sr = run_graph_leg(args, world, dev, barrier,
                       lambda i: ops.mxnorm_fwd(xs[i % n_sets], g, p, rounding=ops.SR, seed=i,
                                                q=outs[i % n_sets][0], scales=outs[i % n_sets][1],
                                                G=outs[i % n_sets][2]),
                       algorithmic_bytes(T, D), "row_fwd_kernel<MXNorm, SR>")
    out["sr_fwd"] = compact(sr, {"alu": alu_roofline(
        profiled_instructions(f"mxnorm_fwd_sr_{args.workload}.md", "thread_instructions_per_element"),
        T * D, sr["ms"], sm_mhz)})
    del outs
    dys = [synthetic.upstream_grad(T, D, seed=j, device=dev) for j in range(n_sets)]
    dxs = [torch.empty_like(xs[0]) for _ in range(n_sets)]
    Gbs = [ops.mxnorm_fwd(xs[j], g, p)[2] for j in range(n_sets)]
    dgb = torch.empty(D, dtype=torch.bfloat16, device=dev)
    wsb = torch.empty(max(16, ops.bwd_workspace_bytes(T, D)), dtype=torch.uint8, device=dev)
    bw = run_graph_leg(args, world, dev, barrier,
                       lambda i: ops.mxnorm_bwd(xs[i % n_sets], dys[i % n_sets], g, Gbs[i % n_sets],
                                                dx=dxs[i % n_sets], dgamma=dgb, workspace=wsb),
                       bwd_bytes(T, D, 0), "row_bwd_kernel + dgamma_reduce_kernel")
    # frac counts the algorithmic bytes (x, dy, dx, G, gamma, dgamma); the dgamma
    # partial rows written and read back are traffic on top, shown apart
    ws = ops.bwd_workspace_bytes(T, D)
    out["bwd"] = compact(bw, {"workspace_bytes": 2 * ws,
                              "GBps_with_workspace": round(world * bwd_bytes(T, D, ws) / (bw["ms"] * 1e-3) / 1e9, 1)})
    del dys, dxs, Gbs

    # Size context for the headline's roofline fraction: the measured HBM peak
    # is torch's copy_ over 4 GiB moved; the same copy_ moving only the
    # forward's algorithmic bytes (half read, half written), and torch's
    # elementwise bf16 -> float8_e4m3fn cast of x (reads 2 B, writes 1 B per
    # element: the forward's byte pattern with no statistic and no block
    # scales), show what a plain streaming kernel reaches at this size.  Sets
    # rotate as above.
    half = algorithmic_bytes(T, D) // 2 // 16 * 16
    srcs = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(n_sets)]
    dsts = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(n_sets)]
    ctx = {"copy_same_bytes": run_graph_leg(args, world, dev, barrier,
                                            lambda i: dsts[i % n_sets].copy_(srcs[i % n_sets]), 2 * half,
                                            "torch copy_ (uint8), read + write bytes")}
    del srcs, dsts
    f8s = [torch.empty(T, D, dtype=torch.float8_e4m3fn, device=dev) for _ in range(n_sets)]
    ctx["cast_bf16_to_e4m3"] = run_graph_leg(args, world, dev, barrier,
                                             lambda i: f8s[i % n_sets].copy_(xs[i % n_sets]), 3 * T * D,
                                             "torch elementwise cast bf16 -> float8_e4m3fn of x (no scales)")
    del f8s
    out["stream_context"] = {
        k: compact(v, {"headline_over_this": round(v["ms"] / ms_per_step * algorithmic_bytes(T, D) /
                                                   v["roofline"]["algorithmic_bytes_per_launch"], 3)})
        for k, v in ctx.items()}

    # Variants on the same batch: MXFP4 codes, the scale-reuse statistic.
    outs4 = [(torch.empty(T, D // 2, dtype=torch.uint8, device=dev),
              torch.empty(T, D // 32, dtype=torch.uint8, device=dev),
              torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n_sets)]
    out["mxfp4_fwd"] = compact_leg(args, world, dev, barrier,
                                     lambda i: ops.mxnorm_fwd_ex(xs[i % n_sets], g, p, elem="e2m1",
                                                                 q=outs4[i % n_sets][0], scales=outs4[i % n_sets][1],
                                                                 G=outs4[i % n_sets][2]),
                                     fp4_bytes(T, D), "row_fwd_kernel<MXNorm, E2M1>")
    del outs4
    outsn = [(torch.empty(T, D // 2, dtype=torch.uint8, device=dev),
              torch.empty(T, D // 16, dtype=torch.uint8, device=dev),
              torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n_sets)]
    out["nvfp4_fwd"] = compact_leg(args, world, dev, barrier,
                                     lambda i: ops.mxnorm_fwd_ex(xs[i % n_sets], g, p, elem="nvfp4",
                                                                 q=outsn[i % n_sets][0], scales=outsn[i % n_sets][1],
                                                                 G=outsn[i % n_sets][2]),
                                     nvfp4_bytes(T, D), "row_fwd_kernel<MXNorm, NVFP4>")
    del outsn
    outs = [(torch.empty(T, D, dtype=torch.uint8, device=dev), torch.empty(T, D // 32, dtype=torch.uint8, device=dev),
             torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n_sets)]
    out["scale_reuse_fwd"] = compact_leg(args, world, dev, barrier,
                                           lambda i: ops.mxnorm_fwd_ex(xs[i % n_sets], g, p, stat="scale_exp",
                                                                       q=outs[i % n_sets][0], scales=outs[i % n_sets][1],
                                                                       G=outs[i % n_sets][2]),
                                           algorithmic_bytes(T, D), "row_fwd_kernel<MXNorm>, scale-exponent statistic")
    del outs

    # Downstream block-scaled MXFP8 GEMM (MXNormLinear): the MXNorm output of
    # an 8192 x 4096 N(0,1) batch times the fused QKV weight [4096 x 6144];
    # the weight folding (gamma into W) and the norm -> GEMM pipeline.
    if D == 4096 and T % 128 == 0:
        out["gemm"] = run_gemm_leg(args, w, rank, world, dev, barrier)
        out.update(run_linear_legs(args, w, rank, world, dev, barrier))

    if not args.no_sweep:
        out["sweep"] = run_sweep(args, world, dev, barrier, sm_mhz)
    out["tiny"] = run_tiny(args, world, dev, barrier)

    # CPU oracle on the host cores: rank 0, one GPU only
    if rank == 0 and world == 1:
        import oracle
        x_cpu = xs[0].cpu()
        g_cpu = g.cpu()
        oracle.mxnorm_fwd(x_cpu[:64], g_cpu, p)             # load + warm
        # whole passes over the workload until about 10 s of CPU work
        passes, t = 0, time.time()
        first = None
        while True:
            res = oracle.mxnorm_fwd(x_cpu, g_cpu, p)
            first = res if first is None else first
            passes += 1
            if time.time() - t >= 10.0:
                break
        dt = (time.time() - t) / passes
        # The oracle's pass above is the reference for the GPU's result on the
        # same batch (one more launch, after every timed region): counts of G
        # bits, E8M0 scales and E4M3 codes that differ from the oracle's own.
        q_o, s_o, G_o = first
        q_g, s_g, G_g = ops.mxnorm_fwd(xs[0], g, p)
        torch.cuda.synchronize()
        q_g = q_g.cpu().numpy()
        s_g = s_g.cpu().numpy()
        G_g = G_g.cpu().numpy()
        import numpy as np
        rel = np.abs(G_g.astype(np.float64) - G_o.astype(np.float64)) / np.maximum(G_o.astype(np.float64), 1e-300)
        out["parity"] = {"vs": "oracle's own result, every row of the batch", "rows": int(T),
                         "G_bit_mismatch_rows": int(np.count_nonzero(G_g.view(np.uint32) != G_o.view(np.uint32))),
                         "G_max_rel": float(rel.max()),
                         "scale_mismatch": int(np.count_nonzero(s_g != s_o)),
                         "code_mismatch": int(np.count_nonzero(q_g != q_o))}
        out["cpu_baseline"] = {"value": round(algorithmic_bytes(T, D) / dt / 1e9, 3), "unit": "GB/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"all {T} rows of the workload, {passes} passes "
                                         f"({passes * dt:.1f} s, {dt * 1e3:.1f} ms per pass)"}
        # and on one core: every (T / 256)-th row, repeated for about 2 s
        rows1 = list(range(0, T, max(1, T // 256)))[:256]
        passes1, t = 0, time.time()
        while True:
            oracle.mxnorm_fwd(x_cpu, g_cpu, p, rows=rows1, nthreads=1)
            passes1 += 1
            if time.time() - t >= 2.0:
                break
        dt1 = (time.time() - t) / passes1
        out["cpu_baseline"]["value_1core"] = round(algorithmic_bytes(len(rows1), D) / dt1 / 1e9, 4)
        out["cpu_baseline"]["sample_1core"] = (f"{len(rows1)} rows (one in {max(1, T // 256)}), 1 thread, "
                                               f"{passes1} passes ({passes1 * dt1:.1f} s)")
    return out


def compact_leg(args, world, dev, barrier, fn, nbytes, kernel):
    return compact(run_graph_leg(args, world, dev, barrier, fn, nbytes, kernel))


def run_tiny(args, world, dev, barrier):
    """The small configuration (x bf16 [256 x 1024] N(0,1), gamma, p = 2,
    nearest-even): one launch moves 0.79 MB, so it is launch-bound; reported
    for completeness."""
    import torch
    from normalisation_row_bf16_b200 import ops, synthetic
    w = workload_cfg("tiny_256x1024_normal_p2")
    T, D, p = w["T"], w["D"], w["p"]
    x = synthetic.activations(T, D, w["kind"], seed=0, device=dev)
    g = synthetic.gamma(D, seed=0, device=dev)
    n = 8
    xs = [x] + [x.clone() for _ in range(n - 1)]
    outs = [(torch.empty(T, D, dtype=torch.uint8, device=dev), torch.empty(T, D // 32, dtype=torch.uint8, device=dev),
             torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(n)]
    leg = run_graph_leg(args, world, dev, barrier,
                        lambda i: ops.mxnorm_fwd(xs[i % n], g, p, q=outs[i % n][0], scales=outs[i % n][1],
                                                 G=outs[i % n][2]),
                        algorithmic_bytes(T, D), "row_fwd_kernel<MXNorm>")
    return compact(leg, {"workload": "tiny_256x1024_normal_p2", "note": "launch-bound (0.79 MB per launch), L2-resident"})


def bwd_bytes(T, D, ws_bytes):
    # read x, dy (2 B/elem each), write dx (2 B/elem); G, gamma; partial sums
    # written and read once; dgamma written
    return 6 * T * D + 4 * T + 2 * D + 2 * ws_bytes + 2 * D


def run_graph_leg(args, world, dev, barrier, fn, nbytes, kernel):
    """Time fn(i) for K steps as one replayed CUDA graph; GB/s vs the HBM peak."""
    import torch
    import torch.distributed as dist
    for i in range(max(3, args.warmup)):
        fn(i)
    K = max(1, min(args.steps, 500))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(K):
            fn(i)
    graph.replay()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    device_hold()
    t0.record()
    graph.replay()
    t1.record()
    barrier()
    del graph
    tm = torch.tensor([t0.elapsed_time(t1) / K], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    ms = float(tm[0])
    peaks, src = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 5), "steps": K, "GBps": round(world * gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "algorithmic_bytes_per_launch": int(nbytes)},
            "kernel": kernel}


def run_sweep(args, world, dev, barrier, sm_mhz):
    """T = 16384, D in {2048, 4096, 8192, 16384}, x = 0.5 t(3), no gamma, p in
    {1, 2, 4, inf}, nearest-even and stochastic rounding.  One compact record
    per case: [D, p, rounding, us, GB/s, fraction of HBM, fraction of the issue
    rate (stochastic rounding at p = 2, where a committed instruction count
    exists)]."""
    import math as _m
    import torch
    from normalisation_row_bf16_b200 import ops, synthetic
    res = []
    for D in (2048, 4096, 8192, 16384):
        T = 16384
        x = synthetic.activations(T, D, "student_t", seed=1, device=dev)
        # Whole input + output sets rotate, at least 3x L2 in all, so neither
        # the reads nor the code writes of one step are served by L2 in the next.
        per_set = T * D * 3 + T * (D // 32) + 4 * T
        n_rot = max(2, math.ceil(3 * L2_BYTES / per_set))
        xs2 = [x] + [x.clone() for _ in range(n_rot - 1)]
        qs = [torch.empty(T, D, dtype=torch.uint8, device=dev) for _ in range(n_rot)]
        scs = [torch.empty(T, D // 32, dtype=torch.uint8, device=dev) for _ in range(n_rot)]
        Gs = [torch.empty(T, dtype=torch.float32, device=dev) for _ in range(n_rot)]
        ipe = profiled_instructions("mxnorm_fwd_sr_sweep_16384.md", f"thread_instructions_per_element_D{D}")
        for p in (1.0, 2.0, 4.0, _m.inf):
            for rnd in (ops.RNE, ops.SR):
                r = run_graph_leg(args, world, dev, barrier,
                                  lambda i: ops.mxnorm_fwd(xs2[i % n_rot], None, p, rounding=rnd, seed=0,
                                                           q=qs[i % n_rot], scales=scs[i % n_rot],
                                                           G=Gs[i % n_rot]),
                                  algorithmic_bytes(T, D) - 2 * D, "row_fwd_kernel<MXNorm>")
                rec = [D, "inf" if _m.isinf(p) else int(p), "sr" if rnd == ops.SR else "rne",
                       round(r["ms"] * 1e3, 1), round(r["GBps"]), round(r["roofline"]["frac"], 3)]
                if rnd == ops.SR and p == 2.0:
                    alu = alu_roofline(ipe, T * D, r["ms"], sm_mhz)
                    rec.append(alu["frac"] if alu else None)
                res.append(rec)
        del x, xs2, qs, scs, Gs
        torch.cuda.empty_cache()
    return {"T": 16384, "x": "0.5 t(3)", "gamma": False,
            "fields": ["D", "p", "rounding", "us", "GBps", "frac_hbm", "frac_issue (sr, p=2)"], "cases": res}


def run_gemm_leg(args, w, rank, world, dev, barrier):
    import torch
    import torch.distributed as dist
    from normalisation_row_bf16_b200 import ops, synthetic

    T, K, N = w["T"], w["D"], 6144
    x = synthetic.activations(T, K, "normal", seed=rank, device=dev)
    g = synthetic.gamma(K, seed=rank, device=dev)
    wt = synthetic.gemm_weight(N, K, seed=rank, device=dev)
    aq, a_s, _ = ops.mxnorm_fwd(x, g, 2.0, scale_layout=ops.SCALES_MMA)
    bq, b_s = ops.mxfp8_cast(wt, scale_layout=ops.SCALES_MMA)
    c = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    for _ in range(max(3, args.warmup)):
        ops.mxfp8_gemm(aq, a_s, bq, b_s, T, N, K, c=c)
    Kg = max(1, min(args.steps, 200))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(Kg):
            ops.mxfp8_gemm(aq, a_s, bq, b_s, T, N, K, c=c)
    graph.replay()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    device_hold()
    t0.record()
    graph.replay()
    t1.record()
    barrier()
    del graph
    ms = t0.elapsed_time(t1) / Kg
    tm = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    ms = float(tm[0])
    flops = 2.0 * T * N * K
    peaks, src = measured_peaks()
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    fp8_peak = 2.0 * bf16        # nominal dense fp8 : bf16 ratio is 2 (4.5 vs 2.25 PFLOP/s)
    tflops = world * flops / (ms * 1e-3) / 1e12
    return {"shape_MNK": [T, N, K], "ms": round(ms, 5), "steps": Kg, "TFLOPs": round(tflops, 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops / world, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(tflops / world / fp8_peak, 4),
                         "peak_source": f"{src} bf16 x 2 (nominal fp8/bf16 ratio)"},
            "kernel": ("gemm_mxfp8_wide_kernel (tcgen05 mxf8f6f4 block_scale, 256x192 tiles)"
                       if T % 256 == 0 and N % 384 == 0 else
                       "gemm_mxfp8_kernel (tcgen05 mxf8f6f4 block_scale, 128x256 tiles)")}


def nvfp4_bytes(T, D):
    # read x (2 B/elem), write E2M1 codes (1/2 B/elem) and E4M3 scales (1 per 16); gamma, G
    return int(T * D * 2 + T * D // 2 + T * (D // 16) + 2 * D + 4 * T)


def fp4_bytes(T, D):
    # read x (2 B/elem), write E2M1 codes (1/2 B/elem) and scales (1/32); gamma, G
    return int(T * D * 2 + T * D // 2 + T * (D // 32) + 2 * D + 4 * T)


def run_linear_legs(args, w, rank, world, dev, barrier):
    """MXNormLinear: folding gamma into the QKV weight, and one linear layer's
    input path + GEMM as a pipeline (MXNorm -> GEMM vs RMSNorm -> MXCast -> GEMM)."""
    import torch
    import torch.distributed as dist
    from normalisation_row_bf16_b200 import ops, synthetic

    T, K, N, p = w["T"], w["D"], 6144, w["p"]
    res = {}
    wt = synthetic.gemm_weight(N, K, seed=rank, device=dev)
    g = synthetic.gamma(K, seed=rank, device=dev)
    n_w = max(2, math.ceil(3 * L2_BYTES / (N * K * 3)))
    wts = [wt] + [wt.clone() for _ in range(n_w - 1)]
    bqs = [torch.empty(N, K, dtype=torch.uint8, device=dev) for _ in range(n_w)]
    bss = [torch.zeros(ops.scales_bytes(N, K, ops.SCALES_MMA), dtype=torch.uint8, device=dev) for _ in range(n_w)]
    res["fold_weight"] = run_graph_leg(args, world, dev, barrier,
                                       lambda i: ops.fold_weight(wts[i % n_w], g, q=bqs[i % n_w], scales=bss[i % n_w]),
                                       N * K * 3 + N * (K // 32) + 2 * K, "row_fwd_kernel<Cast, gain>")
    bq, bs = bqs[0], bss[0]
    del wts, bqs[1:], bss[1:]

    # pipeline: per step one batch x -> codes -> C, inputs and outputs rotating
    n_s = 3
    xs = [synthetic.activations(T, K, "normal", seed=rank + j, device=dev) for j in range(n_s)]
    aqs = [torch.empty(T, K, dtype=torch.uint8, device=dev) for _ in range(n_s)]
    ass = [torch.zeros(ops.scales_bytes(T, K, ops.SCALES_MMA), dtype=torch.uint8, device=dev) for _ in range(n_s)]
    Gs = [torch.empty(T, dtype=torch.float32, device=dev) for _ in range(n_s)]
    cs = [torch.empty(T, N, dtype=torch.bfloat16, device=dev) for _ in range(n_s)]
    ytmp = torch.empty(T, K, dtype=torch.bfloat16, device=dev)
    bq_u, bs_u = ops.mxfp8_cast(wt, scale_layout=ops.SCALES_MMA)

    def mxnorm_step(i):
        j = i % n_s
        ops.mxnorm_fwd(xs[j], None, p, scale_layout=ops.SCALES_MMA, q=aqs[j], scales=ass[j], G=Gs[j])
        ops.mxfp8_gemm(aqs[j], ass[j], bq, bs, T, N, K, c=cs[j])

    def two_pass_step(i):
        j = i % n_s
        ops.rmsnorm_then_mxcast(xs[j], g, 1e-5, scale_layout=ops.SCALES_MMA, y_tmp=ytmp, q=aqs[j], scales=ass[j])
        ops.mxfp8_gemm(aqs[j], ass[j], bq_u, bs_u, T, N, K, c=cs[j])

    flops = 2.0 * T * N * K
    for name, fn in (("pipeline_mxnorm_gemm", mxnorm_step), ("pipeline_rmsnorm_mxcast_gemm", two_pass_step)):
        r = run_graph_leg(args, world, dev, barrier, fn, 0, name)
        res[name] = {"ms": r["ms"], "steps": r["steps"],
                     "TFLOPs_gemm_equiv": round(world * flops / (r["ms"] * 1e-3) / 1e12, 1),
                     "kernels_per_step": 2 if name.startswith("pipeline_mxnorm") else 3}
    res["pipeline_speedup"] = round(res["pipeline_rmsnorm_mxcast_gemm"]["ms"] /
                                    res["pipeline_mxnorm_gemm"]["ms"], 4)
    return res


# ---------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm, on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    import torch
    import oracle
    from normalisation_row_bf16_b200 import synthetic

    w = workload_cfg(args.workload)
    T, D, p = w["T"], w["D"], w["p"]
    x = synthetic.activations(T, D, w["kind"], seed=0)
    g = synthetic.gamma(D, seed=0)
    # size each step's sample so that warm-up + steps take about a minute
    probe = min(T, 256)
    t = time.time()
    oracle.mxnorm_fwd(x[:probe], g, p)
    per_row = (time.time() - t) / probe
    total = args.steps + args.warmup
    rows = int(max(1, min(T, 60.0 / max(total, 1) / max(per_row, 1e-9))))
    xs = x[:rows].contiguous()
    for _ in range(args.warmup):
        oracle.mxnorm_fwd(xs, g, p)
    t = time.time()
    for _ in range(args.steps):
        oracle.mxnorm_fwd(xs, g, p)
    dt = (time.time() - t) / max(args.steps, 1)
    value = algorithmic_bytes(rows, D) / dt / 1e9
    cores = oracle.num_threads()
    sample = f"rows 0..{rows - 1} of the {T}-row workload per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "T": T, "D": D, "block": 32, "p": p, "rounding": "rne",
                   "gamma": True, "scale_layout": "rowmajor", "x": w["kind"]},
        "cpu_baseline": {"kind": "oracle", "value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_profile_only(args):
    """Four untimed launches of one kernel on the workload (the 8192 x 4096
    batch; the GEMM on the fused QKV weight), for a profiler to capture."""
    import torch
    from normalisation_row_bf16_b200 import ops, synthetic
    leg = args.profile_only
    if leg == "sr_sweep":
        for Ds in (2048, 4096, 8192, 16384):
            xs = synthetic.activations(16384, Ds, "student_t", seed=1, device="cuda")
            for i in range(2):
                ops.mxnorm_fwd(xs, None, 2.0, rounding=ops.SR, seed=i)
            torch.cuda.synchronize()
            del xs
            torch.cuda.empty_cache()
        if ops.device_status() != ops.MXN_OK:
            raise SystemExit("device status not clean")
        print(json.dumps({"profile_only": leg, "launches": 8}), flush=True)
        return
    w = workload_cfg(args.workload)
    T, D, p = w["T"], w["D"], w["p"]
    x = synthetic.activations(T, D, w.get("kind", "outliers"), seed=0, device="cuda")
    g = synthetic.gamma(D, seed=0, device="cuda")
    # Inputs and outputs rotate over 4 sets (> 3x L2) as in the timed legs, so
    # a captured launch sees the steady state's DRAM traffic: its inputs come
    # from DRAM and the write-backs of earlier launches' outputs land in it.
    n = 4
    xs = [x] + [x.clone() for _ in range(n - 1)]
    if leg == "bwd":
        dys = [synthetic.upstream_grad(T, D, seed=j, device="cuda") for j in range(n)]
        Gs = [ops.mxnorm_fwd(xs[j], g, p)[2] for j in range(n)]
        dxs = [torch.empty_like(x) for _ in range(n)]
    if leg == "gemm":
        wt = synthetic.gemm_weight(6144, D, seed=0, device="cuda")
        aq, a_s, _ = ops.mxnorm_fwd(x, None, p, scale_layout=ops.SCALES_MMA)
        bq, b_s = ops.fold_weight(wt, g)
    cw = D // 2 if leg in ("mxfp4", "nvfp4") else D
    sw = D // 16 if leg == "nvfp4" else D // 32
    outs = [(torch.empty(T, cw, dtype=torch.uint8, device="cuda"), torch.empty(T, sw, dtype=torch.uint8, device="cuda"),
             torch.empty(T, dtype=torch.float32, device="cuda")) for _ in range(n)]
    for i in range(8):
        j = i % n
        q, s, Gq = outs[j]
        if leg == "fwd":
            ops.mxnorm_fwd(xs[j], g, p, q=q, scales=s, G=Gq)
        elif leg == "sr":
            ops.mxnorm_fwd(xs[j], g, p, rounding=ops.SR, seed=i, q=q, scales=s, G=Gq)
        elif leg == "mxfp4":
            ops.mxnorm_fwd_ex(xs[j], g, p, elem="e2m1", q=q, scales=s, G=Gq)
        elif leg == "nvfp4":
            ops.mxnorm_fwd_ex(xs[j], g, p, elem="nvfp4", q=q, scales=s, G=Gq)
        elif leg == "bwd":
            ops.mxnorm_bwd(xs[j], dys[j], g, Gs[j], dx=dxs[j])
        elif leg == "gemm":
            ops.mxfp8_gemm(aq, a_s, bq, b_s, T, 6144, D)
    torch.cuda.synchronize()
    if ops.device_status() != ops.MXN_OK:
        raise SystemExit("device status not clean")
    print(json.dumps({"profile_only": leg, "launches": 8}), flush=True)


def main():
    args = parse_args()
    if args.profile_only:
        run_profile_only(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    import datetime
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
