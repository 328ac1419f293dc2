#!/usr/bin/env python
"""Benchmark of the B200 gated delta-net scan (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one pass of the whole scan over one batch of synthetic inputs that
are already resident in HBM: for the default workload, skewed (B=4, H=32,
T=16,384, d_k=d_v=128, bf16 q/k/v, fp32 gates, fp32 output and state; the
largest single-call workload), one gdn_scan_causal call.  Its inputs
(~1.6 GB) are larger than the 126 MB L2, so no flush is needed between steps;
for workloads smaller than L2 a 256 MB buffer is written between timed steps,
outside the events.  After the headline workload the other bf16 workloads
(--others) are timed the same way and reported under `others`.

Metric: Mtokens/s = B*H*T per step / step time.  Time is measured with CUDA
events on the launching stream after W warm-up steps, bracketed by a barrier
and a device synchronise; with N > 1 (torchrun, one rank per GPU) every rank
runs the same workload as an independent problem (weak scaling, no data-path
collective) and the max over ranks is used.

Extra keys: `roofline` (the dominant kernel's algorithmic bytes or FLOPs per
launch over its mean CUDA-event duration, from a second pass of the same
steps with an event pair around every launch, against the measured peak), `cpu_baseline` (the FP64 oracle on a bounded sample, on
the host cores; rank 0 at N = 1), `e2e` (the same metric through the Python
API with the inputs copied from pinned host memory and the output and state
read back inside the timed region, successive steps pipelined so that one's
upload overlaps the previous one's download), `clocks` (nvidia-smi samples taken during
the timed region), `gpu_launches` (kernels the library launched in the
timed region, from its own launch counter) and, for the rollout workload,
`graph` (the same step captured once in a CUDA graph and replayed),
`device_timeouts` (bounded device-side waits that gave up during the run,
read from the library; a non-zero count marks the line invalid).

`--impl reference` times the FP64 oracle (the reference implementation of
this build) on the host cores instead: each step is a bounded sample of the
same workload.
"""
import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-delta scan Mtokens/s (B·H·T) on 1 B200; % of roofline"
UNIT = "Mtokens/s"
L2_BYTES = 126 * 1024 * 1024

# Roofline denominators: measured on this machine's B200s (MEASURED_PEAKS.json)
# when present, else the earlier pool measurement.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# algorithmic traffic and work (per token-head)
# ---------------------------------------------------------------------------
def bytes_per_token_head(w, out_bytes=4):
    ib = 4 if w.dtype == "f32" else 2
    return ib * (2 * w.dk + w.dv) + out_bytes * w.dv + 8   # q,k,v read; o written; alpha,beta


def state_bytes_per_call(w):
    return w.B * w.H * w.dk * w.dv * 4


def flops_per_token_head(w, C=64):
    dk, dv = w.dk, w.dv
    if w.mode == "vda":
        return sum(vda_kernel_flops(w).values())
    causal = C * (6 * dk + 4 * dv) + 6 * dk * dv + C * C / 3.0
    if w.mode == "bidir":
        return causal + C * (2 * dk + 4 * dv) + 6 * dk * dv + C * C / 3.0
    return causal


def vda_kernel_flops(w):
    """FLOPs per token-head of the frame-wise operator's kernels (bidirectional):
    the frame's key Gram and key-value products (2 dk (dk + dv) per token);
    per frame the Cholesky of I + A (dk^3/3) and the solves for P = (I + A)^-1
    (2 dk^3); per frame and direction S <- P (a S + B) (2 dk^2 dv); the
    readout of the two summed states (2 dk dv per token)."""
    dk, dv, U = w.dk, w.dv, w.frame
    f = {"vda_gram": 2.0 * dk * (dk + dv),
         "vda_factor": (dk ** 3 / 3.0 + 2.0 * dk ** 3) / U,
         "vda_chain": 2 * 2.0 * dk * dk * dv / U,
         "vda_readout": 2.0 * dk * dv}
    f["vda_gram_tc"], f["vda_readout_tc"] = f["vda_gram"], f["vda_readout"]
    return f


def vda_kernel_bytes(name, w, out_bytes=4):
    """Algorithmic HBM bytes per token-head of the frame-wise operator's
    streaming kernels: the Gram reads k, v and beta; the readout reads q and
    the two directions' states of its frame (fp32-sized, per frame of U
    tokens) and writes o."""
    ib = 4 if w.dtype == "f32" else 2
    if "gram" in name:
        return ib * (w.dk + w.dv) + 4
    return ib * w.dk + out_bytes * w.dv + 2 * 4 * w.dk * w.dv / w.frame


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 FMA/clk x 2 FLOP x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def algorithmic_bytes_per_step(w, out_bytes=4):
    b = w.token_heads * bytes_per_token_head(w, out_bytes)
    if w.mode == "rollout":
        b += w.calls * 2 * state_bytes_per_call(w)       # state read + written per call
    elif w.mode == "causal":
        b += state_bytes_per_call(w)                     # final state written
    return b


# Per kernel: which algorithmic bytes (per token-head) it moves.  The prep
# kernel reads q, k, v and the gates; the chain kernel writes o (and the
# state).  A fused kernel moves all of them.  out_bytes: element size of o.
def kernel_algorithmic_bytes(name, w, out_bytes=4):
    ib = 4 if w.dtype == "f32" else 2
    reads = ib * (2 * w.dk + w.dv) + 8
    writes = out_bytes * w.dv
    if "prep" in name:
        return reads
    if "chain" in name:
        return writes
    return reads + writes


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per token-head
# of a kernel, from one ncu capture of a smaller case of the same launch
# configuration (profiles/ holds the summaries), scaled by the token-heads a
# launch processes.  Keyed by (kernel, workload); absent means not captured
# for this kernel as it stands.
MEASURED_TRAFFIC_PER_TOKEN_HEAD = {
    ("tc_prep", "skewed"): (203.651072e6 + 248.647424e6) / (4 * 32 * 2048),   # prep_kernel<128>, T = 2048
    ("tc_chain", "skewed"): (302.596608e6 + 105.210368e6) / (4 * 32 * 2048),   # chain_kernel<128, float>, T = 2048
}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_indices):
        self.idx = set(gpu_indices)
        self.proc = None
        self.path = os.path.join("/tmp", "gdn_bench_clocks_%d.csv" % os.getpid())

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + SMI_FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    if int(parts[0]) not in self.idx:
                        continue
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the workload's step on the GPU
# ---------------------------------------------------------------------------
class GPUStep:
    def __init__(self, w, device):
        import torch
        import gated_delta_rule_72_b200 as gdn
        from gated_delta_rule_72_b200 import inputs
        self.torch, self.gdn, self.w, self.dev = torch, gdn, w, device
        host = inputs.workload_inputs(w)          # drawn on the CPU, seeded
        self.host = host
        self.d = {n: t.to(device) for n, t in host.items()}
        torch.cuda.synchronize(device)
        self.o = torch.empty(w.B, w.total_T, w.H, w.dv, dtype=torch.float32, device=device)
        self.state = torch.zeros(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=device)
        td = self.d["q"].dtype
        if w.mode == "vda":
            from gated_delta_rule_72_b200 import inputs as I
            self.d["alpha_frame"] = I.frame_alpha(self.d["alpha"], w.frame)
            nb = gdn.gdn_vda_workspace_size(w.B, w.T // w.frame, w.frame, w.H, w.dk, w.dv, 1)
        elif w.mode == "rollout":
            nb = gdn.workspace_size(w.B, w.T, w.H, w.dk, w.dv, td)
            self.slices = []
            for i in range(w.calls):
                sl = slice(i * w.T, (i + 1) * w.T)
                self.slices.append(({n: t[:, sl] for n, t in self.d.items()}, self.o[:, sl]))
        else:
            nb = gdn.workspace_size(w.B, w.T, w.H, w.dk, w.dv, td, bidir=(w.mode == "bidir"))
        self.ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=device)
        self.flush = None
        in_bytes = sum(t.numel() * t.element_size() for t in self.d.values())
        if in_bytes < 2 * L2_BYTES:
            self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def run(self):
        gdn, d, w = self.gdn, self.d, self.w
        if w.mode == "causal":
            gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], None, out=self.o,
                            state_out=self.state, workspace=self.ws)
        elif w.mode == "bidir":
            gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out=self.o,
                           workspace=self.ws)
        elif w.mode == "vda":
            gdn.vda_scan(d["q"], d["k"], d["v"], d["alpha_frame"], d["beta"], w.frame, bidir=True, out=self.o,
                         workspace=self.ws)
        else:
            self.state.zero_()
            for part, o in self.slices:
                gdn.step(part["q"], part["k"], part["v"], part["alpha"], part["beta"], self.state,
                         out=o, workspace=self.ws)

    def between(self):
        if self.flush is not None:
            self.flush.fill_(1)

    def scan_with(self, d, o, state):
        """The step's scan through the public API on inputs `d` (device
        tensors, the layout of the host copies), into `o` and `state`."""
        gdn, w = self.gdn, self.w
        if w.mode == "causal":
            gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], None, out=o,
                            state_out=state, workspace=self.ws)
        elif w.mode == "bidir":
            gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out=o, workspace=self.ws)
        elif w.mode == "vda":
            from gated_delta_rule_72_b200 import inputs as I
            gdn.vda_scan(d["q"], d["k"], d["v"], I.frame_alpha(d["alpha"], w.frame), d["beta"], w.frame,
                         bidir=True, out=o, workspace=self.ws)
        else:
            state.zero_()
            for i in range(w.calls):
                sl = slice(i * w.T, (i + 1) * w.T)
                gdn.step(d["q"][:, sl], d["k"][:, sl], d["v"][:, sl], d["alpha"][:, sl],
                         d["beta"][:, sl], state, out=o[:, sl], workspace=self.ws)


def timed(torch, fn, between, steps, dist=None):
    """Mean device ms per step over `steps` steps, CUDA events on the current stream."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for s, e in ev:
        between()
        s.record()
        fn()
        e.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return sum(s.elapsed_time(e) for s, e in ev) / steps


def graph_replay_ms(torch, step, steps, dist=None):
    """The rollout's calls captured once in a CUDA graph, then `steps` replays
    timed like the eager steps (mean device ms per replay)."""
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        step.run()
    for _ in range(3):
        step.between()
        g.replay()
    ms = timed(torch, g.replay, step.between, steps, dist)
    del g
    return ms


def max_over_ranks(torch, dist, x, device):
    """The slowest rank's time (every rank takes part; gloo on the CPU, NCCL on GPUs)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(n_gpus, units_per_gpu, ms_max):
    """Whole-job Mtokens/s: the token-heads all ranks processed over the slowest rank's time."""
    return n_gpus * units_per_gpu / (ms_max * 1e-3) / 1e6


# ---------------------------------------------------------------------------
# the FP64 oracle on the host cores (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def oracle_run(w, x, threads):
    """One oracle pass over the inputs x of workload w (a sample of it)."""
    import oracle
    from gated_delta_rule_72_b200 import inputs
    if w.mode == "vda":
        oracle.vda_scan(x["q"], x["k"], x["v"], inputs.frame_alpha(x["alpha"], w.frame), x["beta"], w.frame,
                        mode="bidir")
    else:
        oracle.scan(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                    mode="bidir" if w.mode == "bidir" else "causal", threads=threads)


def oracle_sample(w, target_s):
    """Time the oracle on the first T_s tokens of every head (whole frames for
    the frame-wise operator), T_s sized so the run takes about target_s
    seconds.  Returns (Mtok/s, threads, description, T_s)."""
    from gated_delta_rule_72_b200 import inputs
    threads = max(1, min(os.cpu_count() or 1, w.B * w.H))
    mode = {"bidir": "bidir", "vda": "frame-wise, bidir"}.get(w.mode, "causal")
    full_T = w.total_T
    step = w.frame if w.mode == "vda" else 1

    def run(Ts):
        x = inputs.generate(w.B, Ts, w.H, w.dk, w.dv, w.dtype, w.seed, w.gates)
        t0 = time.perf_counter()
        oracle_run(w, x, threads)
        return time.perf_counter() - t0

    Tc = min(full_T, max(128, step))
    tc = run(Tc)
    Ts = int(min(full_T, max(Tc, Tc * target_s / max(tc, 1e-6))))
    Ts = max(step, Ts // step * step)
    ts = run(Ts)
    units = w.B * w.H * Ts
    desc = "%s: all %d heads x first %d of %d tokens (%s), float64, %d threads" % (
        w.name, w.B * w.H, Ts, full_T, mode, threads)
    return units / ts / 1e6, threads, desc, Ts


def device_timeouts(gdn):
    """Bounded device-side waits of the library that gave up so far (the
    library's own counter; a timed result is valid only while it stays 0)."""
    try:
        return int(gdn.gdn_device_timeouts())
    except Exception:   # noqa: BLE001  (reported as unknown, never as zero)
        return -1


def roofline_of(w, ktimes, steps, units, peaks, peak_src):
    """The dominant kernel's achieved rate against its roofline, from the
    per-kernel CUDA-event times of the timed region."""
    if not ktimes:
        return None
    name, (tot_ms, n) = max(ktimes.items(), key=lambda kv: kv[1][0])
    per_launch_ms = tot_ms / n
    launches_per_step = n / steps
    units_per_launch = units / launches_per_step
    bound = "tensor" if w.mode == "bidir" and "chain" not in name else "hbm"
    if w.mode == "vda":
        # the factor and the chain are fp32 on the CUDA cores; the Gram and
        # the readout stream their operands from HBM
        bound = "hbm" if ("gram" in name or "readout" in name) else "alu"
    nbytes = (lambda ob=4: vda_kernel_bytes(name, w, ob)) if w.mode == "vda" else \
        (lambda ob=4: kernel_algorithmic_bytes(name, w, out_bytes=ob))
    extra = {}
    if bound == "alu":
        alg = vda_kernel_flops(w).get(name, 0.0) * units_per_launch
        achieved = alg / (per_launch_ms * 1e-3) / 1e12
        peak = FP32_ALU_TFLOPS
        unit = "TFLOP/s"
    elif bound == "hbm":
        alg = nbytes() * units_per_launch
        achieved = alg / (per_launch_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        # the same kernel against the byte count with o in bf16 (the inputs' dtype)
        alg16 = nbytes(2) * units_per_launch
        extra = {"frac_bf16_out_bytes": alg16 / (per_launch_ms * 1e-3) / 1e9 / peak,
                 "bytes_per_token_head": nbytes(),
                 "bytes_per_token_head_bf16_out": nbytes(2)}
    else:
        alg = flops_per_token_head(w) * units_per_launch
        achieved = alg / (per_launch_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    total_ms = sum(t for t, _ in ktimes.values())
    tph = MEASURED_TRAFFIC_PER_TOKEN_HEAD.get((name, w.name))
    traffic = tph * units_per_launch if tph is not None else None
    roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic, "kernel": name,
            "peak_source": ("derived: 148 SMs x 128 fp32 FMA/clk x 2 x 1.965 GHz" if bound == "alu" else
                            "%s (%s)" % (peak_src, "MEASURED_PEAKS.json" if peak_src == "measured"
                                         else "pool fallback")),
            "kernel_ms_per_launch": per_launch_ms,
            "kernel_share": tot_ms / total_ms if total_ms else None,
            "kernels": {k: {"ms_per_step": t / steps, "launches_per_step": c / steps}
                        for k, (t, c) in ktimes.items()}}
    roof.update(extra)
    return roof


def step_roofline(w, ms, peaks):
    """The whole step against its roofline: bytes at HBM bandwidth vs FLOPs at
    the tensor peak; bytes with o in fp32 (as written here) and in bf16 (o in
    the inputs' dtype)."""
    t_flop = w.token_heads * flops_per_token_head(w) / (peaks["bf16_tflops"] * 1e12)
    out = {}
    for key, ob in (("", 4), ("_bf16_out", 2)):
        t_mem = algorithmic_bytes_per_step(w, ob) / (peaks["hbm_gbs"] * 1e9)
        t = max(t_mem, t_flop)
        out["t_roofline_ms" + key] = t * 1e3
        out["bound" + key] = "hbm" if t_mem >= t_flop else "tensor"
        out["frac" + key] = t / (ms * 1e-3)
    return out


def measure(torch, gdn, w, device, args, dist, rank, clocks=True):
    """Warm up, then time args.steps steps of workload w with per-kernel
    events on; the clocks are sampled during the timed region."""
    step = GPUStep(w, device)
    for _ in range(max(3, args.warmup)):
        step.between()
        step.run()
    torch.cuda.synchronize()
    sampler = ClockSampler(range(args.gpus)) if clocks else None
    if sampler:
        # nvidia-smi takes a moment to start sampling: keep the GPU busy with
        # extra untimed steps for ~1 s so samples cover the load up to the
        # timed region, which follows immediately
        sampler.start()
        t_end = time.time() + 1.0
        while time.time() < t_end:
            step.run()
            torch.cuda.synchronize()
    n0 = gdn.gdn_launch_count()
    ms = timed(torch, step.run, step.between, args.steps, dist)
    launches = gdn.gdn_launch_count() - n0
    clk = sampler.stop() if sampler else None
    ms = max_over_ranks(torch, dist, ms, device)
    # the per-kernel breakdown comes from a second pass of the same steps with
    # an event pair around every launch (kept out of the timed pass above:
    # the events add host work per launch)
    gdn.gdn_read_kernel_timing()                  # drop anything recorded so far
    gdn.gdn_set_kernel_timing(1)
    timed(torch, step.run, step.between, args.steps, dist)
    gdn.gdn_set_kernel_timing(0)
    ktimes = gdn.gdn_read_kernel_timing()
    units = w.token_heads                          # per GPU per step
    peaks, peak_src = load_peaks()
    return {"step": step, "ms": ms, "value": whole_job_value(args.gpus, units, ms),
            "roof": roofline_of(w, ktimes, args.steps, units, peaks, peak_src),
            "step_roof": step_roofline(w, ms, peaks), "clocks": clk, "launches": launches}


def workload_config(w, gpus):
    return {"workload": "%s (%s B=%d H=%d T=%d%s d_k=%d d_v=%d, %s in, fp32 out/state, %s gates)"
            % (w.name, w.mode, w.B, w.H, w.T, (" x %d calls" % w.calls) if w.calls > 1 else "",
               w.dk, w.dv, w.dtype, w.gates),
            "B": w.B, "H": w.H, "T": w.total_T, "d_k": w.dk, "d_v": w.dv,
            **({"frame": w.frame} if w.mode == "vda" else {"chunk": 64}),
            "parallelism": "replicas%d (independent (b,h) problems per GPU)" % gpus}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="skewed",
                    choices=["stream480", "bidir720", "rollout", "skewed", "tiny", "vda480"])
    ap.add_argument("--others", default="stream480,bidir720,rollout",
                    help="comma-separated workloads timed after the headline one (device time only); "
                         "empty: none")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target length of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling aid: shorten T to this many tokens (not a benchmark result)")
    args = ap.parse_args()

    import dataclasses
    from gated_delta_rule_72_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    if args.tokens:
        w = dataclasses.replace(w, T=min(w.T, args.tokens), name=w.name + "-T%d" % args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    config = workload_config(w, args.gpus)

    if args.impl == "reference":
        if rank != 0:
            return 0
        per_step_s = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
        import oracle  # noqa: F401  (the reference arm of this build is the oracle)
        rate, threads, desc, Ts = oracle_sample(w, per_step_s)
        # W warm-up + K timed steps, each the same bounded sample
        from gated_delta_rule_72_b200 import inputs as I
        x = I.generate(w.B, Ts, w.H, w.dk, w.dv, w.dtype, w.seed, w.gates)
        for _ in range(args.warmup):
            oracle_run(w, x, threads)
        times = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            oracle_run(w, x, threads)
            times.append(time.perf_counter() - t0)
        step_s = sum(times) / len(times)
        value = w.B * w.H * Ts / step_s / 1e6
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": dict(config, sample_tokens_per_head=Ts),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import gated_delta_rule_72_b200 as gdn
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    gdn.load()

    timeouts0 = device_timeouts(gdn)
    m = measure(torch, gdn, w, device, args, dist, rank, clocks=(rank == 0))
    step, ms, value, roof, step_roof, clocks, launches = (m[k] for k in (
        "step", "ms", "value", "roof", "step_roof", "clocks", "launches"))
    units = w.token_heads
    l2_note = ("inputs larger than L2, no flush" if step.flush is None
               else "L2 flushed between steps (256 MB write)")

    # ---- the streaming rollout replayed from a CUDA graph (device-timed like value)
    graph = None
    if w.mode == "rollout":
        gms = max_over_ranks(torch, dist, graph_replay_ms(torch, step, args.steps, dist), device)
        graph = {"value": whole_job_value(args.gpus, units, gms), "unit": UNIT, "ms_per_step": gms,
                 "calls_per_step": w.calls}

    # ---- end to end through the public API, host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, step, device, args, dist, units)

    # ---- oracle baseline on the host cores (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, desc, _ = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    # ---- the other workloads, device time only (every rank, same order)
    others = {}
    del step, m
    torch.cuda.empty_cache()
    for name in [x for x in args.others.split(",") if x and x != w.name]:
        wo = inputs.WORKLOADS[name]
        mo = measure(torch, gdn, wo, device, args, dist, rank, clocks=(rank == 0))
        rec = {"value": mo["value"], "unit": UNIT, "ms_per_step": mo["ms"],
               "config": workload_config(wo, args.gpus), "roofline": mo["roof"],
               "step_roofline": mo["step_roof"], "clocks": mo["clocks"], "gpu_launches": mo["launches"]}
        if wo.mode == "rollout":
            gms = max_over_ranks(torch, dist, graph_replay_ms(torch, mo["step"], args.steps, dist), device)
            rec["graph"] = {"value": whole_job_value(args.gpus, wo.token_heads, gms), "unit": UNIT,
                            "ms_per_step": gms, "calls_per_step": wo.calls}
        others[name] = rec
        del mo
        torch.cuda.empty_cache()
    timeouts1 = device_timeouts(gdn)
    n_timeouts = timeouts1 - timeouts0 if min(timeouts0, timeouts1) >= 0 else None

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": dict(config, l2=l2_note),
                "roofline": roof, "step_roofline": step_roof,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": launches}
        if graph is not None:
            line["graph"] = graph
        if others:
            line["others"] = others
        line["device_timeouts"] = n_timeouts
        if n_timeouts != 0:
            line["valid"] = False
            line["note"] = "a bounded device-side wait gave up (or the count is unknown): not a result"
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(torch, step, device, args, dist, units):
    """Same metric end to end through the Python API: every step copies its
    inputs from pinned host memory, runs the scan and reads back the output
    and the final state.  The steps are pipelined over three streams (inputs
    in, the scan, results out) with two sets of buffers, so that one step's
    upload overlaps the previous step's download (PCIe carries both
    directions at once); the timed region runs from the first step's upload
    to the last step's download."""
    pinned = {n: t.pin_memory() for n, t in step.host.items()}
    dev = [{n: torch.empty_like(t, device=device) for n, t in step.host.items()} for _ in range(2)]
    outs = [step.o, torch.empty_like(step.o)]
    states = [step.state, torch.empty_like(step.state)]
    out_host = [torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory() for _ in range(2)]
    state_host = [torch.empty(step.state.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_run = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def pipeline(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_run = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        start.record(s_in)
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_run[i - 2])      # the scan of step i-2 is done with buffer set b
            with torch.cuda.stream(s_in):
                for name, t in pinned.items():
                    dev[b][name].copy_(t, non_blocking=True)
            ev_in[i].record(s_in)
            s_run.wait_event(ev_in[i])
            if i >= 2:
                s_run.wait_event(ev_out[i - 2])     # step i-2's results have left buffer set b
            step.scan_with(dev[b], outs[b], states[b])
            ev_run[i].record(s_run)
            s_out.wait_event(ev_run[i])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(outs[b], non_blocking=True)
                state_host[b].copy_(states[b], non_blocking=True)
            ev_out[i].record(s_out)
        end.record(s_out)                           # after every step's download (and so all else)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return start.elapsed_time(end) / n

    pipeline(2)
    e2e_ms = pipeline(args.steps)
    e2e_ms = max_over_ranks(torch, dist, e2e_ms, device)
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host[0].numel() * out_host[0].element_size() + state_host[0].numel() * 4
    return {"value": args.gpus * units / (e2e_ms * 1e-3) / 1e6, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "pipelining": "uploads, scans and downloads on three streams, two buffer sets"}


if __name__ == "__main__":
    sys.exit(main())
