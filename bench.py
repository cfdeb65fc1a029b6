"""Benchmark of the DiG GLA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (N=1): DiG-XL/2 at 1792 resolution -- B=2, H=16, a 112x112 token grid
(T=12544), dk=dv=72, bf16 q/k/v, fp32 log_alpha with g ~ N(0,1).  One step is one
pass of the whole path over the four-direction cycle: for layer l = 0..3,
gla_fwd(dir = l) -> dwconv3x3 on the output viewed as the [B,112,112,1152] grid
-> srem_reorient into the next layer's scan order (dir = (l+1) % 4).  Each layer
has its own seeded inputs (347 MB, larger than the 126 MB L2), so no L2 flush is
needed between iterations.

The metric is token-heads per second (B*T*H per layer) over the whole step;
`roofline` reports the GLA forward (the dominant op) against measured HBM
bandwidth; `cpu_baseline` times the fp64 CPU oracle on a bounded sample of the
same workload (all host threads, and one thread beside it).  `value` is the step
throughput; `gla_only` gives the GLA forward alone, the op the metric names.

Beside the headline (rank 0, unless --no-extras): a long window of c4 GLA launches
(at least one second of device time, its own clock samples, median per direction),
and the 28-layer DiG-XL/2 stack at 2048 resolution (gla_fwd -> dwconv3x3 ->
srem_reorient per layer, fresh inputs per layer, dir = layer % 4), timed with and
without the reorientation; the GLA backward (gla_bwd) on c4 and c2; the c4 GLA forward
along the eight zigzag orders; the draft's normalised variant on c4 and c2;
and the c4 forward with bf16 gate logits (gla_fwd_glogit).  Under torchrun (N > 1) every rank runs its own replica of the
workload (no data exchange: heads and batches are independent), and rank 0
prints the aggregate.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "GLA fwd tokens·heads/s and % of roofline at T=12544, dk=dv=72, bf16"
UNIT = "tokens·heads/s"
WORKLOAD = workloads.WORKLOADS["c4"]
LAYERS = 4
# Algorithmic bytes of one GLA forward per token-head: q, k, v (bf16) + log_alpha
# (fp32) read once, out (bf16) written once.
GLA_BYTES_PER_TOKEN_HEAD = 2 * (2 * WORKLOAD.dk + WORKLOAD.dv) + 4 * WORKLOAD.dk + 2 * WORKLOAD.dv
GLA_FLOP_PER_TOKEN_HEAD = 65 * (WORKLOAD.dk + WORKLOAD.dv) + 4 * WORKLOAD.dk * WORKLOAD.dv
FALLBACK_HBM_GBS = 6650.0


def config_dict(extra=None):
    w = WORKLOAD
    d = {"workload": w.name, "B": w.B, "H": w.H, "grid": f"{w.Hgrid}x{w.Wgrid}", "T": w.T, "dk": w.dk, "dv": w.dv,
         "layers_per_step": LAYERS, "dirs": "layer % 4", "conv_channels": w.C,
         "step": "4 x (gla_fwd + dwconv3x3 + srem_reorient)", "qkv_scale": "1/sqrt(72)",
         "log_alpha": "logsigmoid(g)/16, g~N(0,1)", "l2": "inputs larger than L2 (347 MB per layer), no flush"}
    if extra:
        d.update(extra)
    return d


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# The sources of the GLA forward kernel (gla_ws_fwd): a recorded DRAM traffic figure
# is reported only while these are unchanged.
GLA_KERNEL_SOURCES = ("gla_ws.cu", "dev_common.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_linear_attention_chunkwise_b200", "csrc")
    for name in GLA_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per GLA forward from the committed ncu summary, if it was taken
    on the current kernel sources; otherwise None."""
    path = os.path.join(ROOT, "profiles", "gla_fwd_c4_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except OSError:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_gla_fwd")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for name, bit in self.REASONS.items():
                    if bits & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- CPU oracle timing
def oracle_sample(seconds_target: float = 12.0):
    """Times the fp64 oracle on a bounded sample of the workload: whole heads of the
    GLA scan (all four directions) plus the matching conv channels.  Returns
    (token_heads, seconds, threads, description)."""
    import oracle
    w = WORKLOAD
    cores = oracle.hardware_threads()
    q, k, v, la = (t.double().numpy() for t in workloads.gla_inputs(w, seed=0))  # widened once
    conv_w = workloads.conv_weight(w.C, seed=0).double().numpy()
    # probe: one head, one direction, one thread
    t0 = time.perf_counter()
    oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 0, nthreads=1, heads=(0, 1))
    per_head = time.perf_counter() - t0
    nh = max(1, min(w.B * w.H, int(seconds_target * cores / (LAYERS * per_head * 1.1))))
    nh = min(w.B * w.H, max(nh, min(cores, w.B * w.H)))
    t0 = time.perf_counter()
    threads = 1
    for layer in range(LAYERS):
        out, threads = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, layer, nthreads=cores, heads=(0, nh),
                                      return_threads=True)
        # conv over the channels of the sampled heads of batch 0 (whole grid)
        hb = min(nh, w.H)
        grid = out[:1, :, :hb, :].reshape(1, w.Hgrid, w.Wgrid, hb * w.dv)
        oracle.dwconv3x3(grid, conv_w[: hb * w.dv], nthreads=cores)
        oracle.reorient(grid.reshape(1, w.T, hb * w.dv), (layer + 1) % 4, 0, w.Hgrid, w.Wgrid)
    secs = time.perf_counter() - t0
    desc = (f"fp64 C oracle on heads 0..{nh - 1} of {w.B * w.H} (whole 12544-token scans) x 4 directions, "
            f"plus dwconv3x3 + reorient on the sampled heads' channels")
    return nh * w.T * LAYERS, secs, threads, desc


def oracle_sample_one_core():
    """The oracle on one host thread: one head of the c4 workload through the four
    directions (whole 12544-token scans) plus dwconv3x3 and the reorientation on that
    head's 72 channels.  Returns (token_heads, seconds, description)."""
    import oracle
    w = WORKLOAD
    q, k, v, la = (t.double().numpy() for t in workloads.gla_inputs(w, seed=0))
    conv_w = workloads.conv_weight(w.C, seed=0).double().numpy()
    t0 = time.perf_counter()
    for layer in range(LAYERS):
        out = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, layer, nthreads=1, heads=(0, 1))
        grid = out[:1, :, :1, :].reshape(1, w.Hgrid, w.Wgrid, w.dv)
        oracle.dwconv3x3(grid, conv_w[: w.dv], nthreads=1)
        oracle.reorient(grid.reshape(1, w.T, w.dv), (layer + 1) % 4, 0, w.Hgrid, w.Wgrid)
    secs = time.perf_counter() - t0
    return w.T * LAYERS, secs, "fp64 C oracle, 1 thread: head 0 of 32 x 4 directions, conv + reorient on its channels"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = WORKLOAD
    cores = oracle.hardware_threads()
    q, k, v, la = (t.double().numpy() for t in workloads.gla_inputs(w, seed=0))  # widened once
    conv_w = workloads.conv_weight(w.C, seed=0).double().numpy()
    nh = min(w.B * w.H, cores)

    def step():
        for layer in range(LAYERS):
            out = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, layer, nthreads=cores, heads=(0, nh))
            hb = min(nh, w.H)
            grid = out[:1, :, :hb, :].reshape(1, w.Hgrid, w.Wgrid, hb * w.dv)
            oracle.dwconv3x3(grid, conv_w[: hb * w.dv], nthreads=cores)
            oracle.reorient(grid.reshape(1, w.T, hb * w.dv), (layer + 1) % 4, 0, w.Hgrid, w.Wgrid)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = time.perf_counter() - t0
    th_per_step = nh * w.T * LAYERS
    value = th_per_step * args.steps / secs
    desc = f"fp64 C oracle, heads 0..{nh - 1} of {w.B * w.H} per step, 4 directions, conv + reorient on their channels"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict({"sample": desc}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks of the process group (x itself on a single rank):
    every multi-rank time is the slowest rank's."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_gpu(args):
    import torch.distributed as dist

    import gated_linear_attention_chunkwise_b200 as dig

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOAD

    # Inputs: one seeded set per layer, generated on the host, resident in HBM.
    host = [workloads.gla_inputs(w, seed=layer + 97 * rank) for layer in range(LAYERS)]
    dev_in = [[t.to(dev) for t in layer] for layer in host]
    conv_w = workloads.conv_weight(w.C, seed=rank).to(dev)
    outs = [torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
    convs = [torch.empty((w.B, w.Hgrid, w.Wgrid, w.C), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
    reor = [torch.empty((w.B, w.T, w.C), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
    stream = torch.cuda.current_stream(dev)
    launches_per_layer = 1 + 1 + 1  # gla_ws_fwd + dwconv3x3 + srem_reorient (the flag reset is a memset)

    def layer(l, ev=None):
        q, k, v, la = dev_in[l]
        if ev is not None:
            ev[0].record(stream)
        dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, l % 4, out=outs[l])
        if ev is not None:
            ev[1].record(stream)
        dig.dwconv3x3(outs[l].view(w.B, w.Hgrid, w.Wgrid, w.C), conv_w, out=convs[l])
        if ev is not None:
            ev[2].record(stream)
        dig.srem_reorient(convs[l].view(w.B, w.T, w.C), (l + 1) % 4, 0, w.Hgrid, w.Wgrid, out=reor[l])
        if ev is not None:
            ev[3].record(stream)

    def step(evs=None):
        for l in range(LAYERS):
            layer(l, None if evs is None else evs[l])

    for _ in range(args.warmup):
        step()
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {dig.status_string(status)}")

    # Timed region: exactly K steps, per-op events inside.
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(LAYERS)]
           for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(stop)
    gla_ms = [e[l][0].elapsed_time(e[l][1]) for e in evs for l in range(LAYERS)]
    conv_ms = [e[l][1].elapsed_time(e[l][2]) for e in evs for l in range(LAYERS)]
    reor_ms = [e[l][2].elapsed_time(e[l][3]) for e in evs for l in range(LAYERS)]
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {dig.status_string(status)}")

    max_ms = max_over_ranks(elapsed_ms, world, dev)
    th_per_step = w.token_heads * LAYERS
    value = th_per_step * args.steps * world / (max_ms / 1e3)

    # End to end through the public API: pinned host inputs -> device -> path -> host result.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    pinned = [[t.pin_memory() for t in layer] for layer in host]
    host_out = [torch.empty((w.B, w.T, w.C), dtype=torch.bfloat16).pin_memory() for _ in range(LAYERS)]
    h2d = sum(t.numel() * t.element_size() for layer in pinned for t in layer)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    # Inputs stream in on one copy stream and results out on another, layer by layer, so
    # that the PCIe transfers of one layer overlap the kernels of the others; events keep
    # a buffer from being overwritten before its previous use is done.
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(LAYERS)]
    in_free = [torch.cuda.Event() for _ in range(LAYERS)]
    out_ready = [torch.cuda.Event() for _ in range(LAYERS)]
    out_free = [torch.cuda.Event() for _ in range(LAYERS)]

    def e2e_step():
        for l in range(LAYERS):
            h2d_stream.wait_event(in_free[l])  # the previous step's layer l has read its inputs
            with torch.cuda.stream(h2d_stream):
                for dst, src in zip(dev_in[l], pinned[l]):
                    dst.copy_(src, non_blocking=True)
            in_ready[l].record(h2d_stream)
        for l in range(LAYERS):
            stream.wait_event(in_ready[l])
            stream.wait_event(out_free[l])  # the previous step's copy of reor[l] is done
            layer(l)
            in_free[l].record(stream)
            out_ready[l].record(stream)
            d2h_stream.wait_event(out_ready[l])
            with torch.cuda.stream(d2h_stream):
                host_out[l].copy_(reor[l], non_blocking=True)
            out_free[l].record(d2h_stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)  # the first input copy starts inside the timed region
    for _ in range(e2e_steps):
        e2e_step()
    for l in range(LAYERS):
        stream.wait_event(out_free[l])  # every result is on the host
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = th_per_step * e2e_steps * world / (max_over_ranks(e0.elapsed_time(e1), world, dev) / 1e3)

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    extra = other_configs(dig, dev, stream, hbm) if (rank == 0 and not args.no_other_configs) else None
    gla_avg_s = statistics.mean(gla_ms) / 1e3
    window = stack = bwd = zig = nrm = glg = None
    if rank == 0 and not args.no_extras:
        window = long_window(dig, dev, stream, dev_in, outs, hbm, gla_us_hint=gla_avg_s * 1e6)
        stack = stack_c5(dig, dev, stream, hbm)
        bwd = bwd_configs(dig, dev, stream, hbm)
        zig = zigzag_c4(dig, dev, stream, dev_in, outs, hbm)
        nrm = norm_configs(dig, dev, stream, hbm)
        glg = glogit_c4(dig, dev, stream, hbm)
    gla_bytes = GLA_BYTES_PER_TOKEN_HEAD * w.token_heads
    achieved = gla_bytes / gla_avg_s / 1e9
    traffic = recorded_traffic()

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            th, secs, threads, desc = oracle_sample(args.cpu_seconds)
            cpu = {"value": th / secs, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                   "seconds": secs}
            th1, secs1, desc1 = oracle_sample_one_core()
            cpu["one_core"] = {"value": th1 / secs1, "unit": UNIT, "cores": 1, "sample": desc1, "seconds": secs1}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT,
            "value_is": ("step throughput: token-heads per second through 4 x (gla_fwd + dwconv3x3 + "
                         "srem_reorient) on c4; the GLA forward alone is gla_only.tokens_heads_per_s"), "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict({"parallelism": f"replicas x{world}" if world > 1 else "single GPU"}),
            "roofline": {
                "bound": "hbm", "kernel": "gla_ws_fwd (persistent warp-specialised GLA forward)",
                "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": f"{peak_kind} hbm_gbs", "traffic": traffic,
                "algorithmic_bytes_per_launch": gla_bytes, "avg_launch_us": gla_avg_s * 1e6,
            },
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gpu_launches": launches_per_layer * LAYERS * args.steps,
            "clocks": clk.summary(),
            "breakdown_us_per_layer": {"gla_fwd": statistics.mean(gla_ms) * 1e3,
                                       "dwconv3x3": statistics.mean(conv_ms) * 1e3,
                                       "srem_reorient": statistics.mean(reor_ms) * 1e3},
            "gla_only": {"tokens_heads_per_s": w.token_heads / gla_avg_s,
                         "tflops": GLA_FLOP_PER_TOKEN_HEAD * w.token_heads / gla_avg_s / 1e12,
                         "median_us": statistics.median(gla_ms) * 1e3,
                         "median_us_by_dir": [statistics.median(gla_ms[l::LAYERS]) * 1e3 for l in range(LAYERS)]},
            "per_kernel": per_kernel(w, gla_ms, conv_ms, reor_ms, hbm),
            "other_configs_gla_fwd": extra,
            "gla_long_window_c4": window,
            "stack_c5_28_layers": stack,
            "gla_bwd": bwd,
            "gla_fwd_zigzag_c4": zig,
            "gla_norm_fwd": nrm,
            "gla_fwd_glogit_c4": glg,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def device_us(fn, stream, reps):
    """Median device time in microseconds of one of `reps` back-to-back calls of fn.
    The stream first spins on the GPU (about 1 ms) while the host enqueues every call,
    so the calls run back to back and the host's own work per call (argument checks,
    the binding, the launches) falls between no pair of events."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    torch.cuda.synchronize()
    torch.cuda._sleep(2_000_000)
    evs[0].record(stream)
    for i in range(reps):
        fn()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(evs[i].elapsed_time(evs[i + 1]) * 1e3 for i in range(reps))


def other_configs(dig, dev, stream, hbm, reps=10):
    """GLA forward alone on the other bf16 configurations (median of `reps` calls per
    scan direction, event-timed, inputs resident in HBM; c2 and c3 fit in L2, so their
    numbers are L2-warm), with the fraction of the HBM roofline on their algorithmic
    bytes.  Supplementary to the headline line."""
    res = {}
    for name in ("c2", "c3", "c5"):
        cw = workloads.WORKLOADS[name]
        q, k, v, la = [t.to(dev) for t in workloads.gla_inputs(cw, seed=7)]
        out = torch.empty((cw.B, cw.T, cw.H, cw.dv), dtype=torch.bfloat16, device=dev)
        nbytes = (2 * (2 * cw.dk + cw.dv) + 4 * cw.dk + 2 * cw.dv) * cw.token_heads
        per_dir = []
        for d in range(4):
            for _ in range(3):
                dig.gla_fwd(q, k, v, la, cw.Hgrid, cw.Wgrid, d, out=out)
            per_dir.append(device_us(lambda: dig.gla_fwd(q, k, v, la, cw.Hgrid, cw.Wgrid, d, out=out), stream, reps))
        us = statistics.mean(per_dir)
        res[name] = {"workload": cw.name, "us_per_dir": per_dir, "bytes": nbytes,
                     "tokens_heads_per_s": cw.token_heads / (us / 1e6),
                     "frac_of_hbm": nbytes / (us / 1e6) / 1e9 / hbm}
        del q, k, v, la, out
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the other configurations: {dig.status_string(status)}")
    return res


def oracle_beside(fn, token_heads, sample):
    """The fp64 oracle timed on the host's threads on a bounded sample of an extra
    entry point's workload: {value (token-heads/s), unit, cores, kind, sample}."""
    import oracle
    t0 = time.perf_counter()
    fn()
    secs = time.perf_counter() - t0
    return {"value": token_heads / secs, "unit": UNIT, "cores": oracle.hardware_threads(), "kind": "oracle",
            "sample": sample, "seconds": secs}


def stack_c5(dig, dev, stream, hbm, reps=5):
    """The 28-layer DiG-XL/2 stack at 2048 resolution (128x128 grid, B=1, H=16, d=72):
    layer l runs gla_fwd(dir = l % 4) -> dwconv3x3 -> srem_reorient(dir = (l+1) % 4)
    on its own seeded inputs (drawn on the device, 189 MB per layer, 5.3 GB in all)
    and writes its own output buffers.  Timed with CUDA events around the whole stack,
    median of `reps` stacks, with and without the reorientation (whose result feeds
    nothing, since every layer's q/k/v are fresh)."""
    w = workloads.WORKLOADS["c5"]
    L = w.layers
    ins = [workloads.gla_inputs_device(w, seed=l, device=dev) for l in range(L)]
    cws = [workloads.conv_weight_device(w.C, seed=l, device=dev) for l in range(L)]
    outs = [torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev) for _ in range(L)]
    convs = [torch.empty((w.B, w.Hgrid, w.Wgrid, w.C), dtype=torch.bfloat16, device=dev) for _ in range(L)]
    reor = [torch.empty((w.B, w.T, w.C), dtype=torch.bfloat16, device=dev) for _ in range(L)]

    def run(with_reorient, ev=None):
        for l in range(L):
            q, k, v, la = ins[l]
            if ev is not None:
                ev[l][0].record(stream)
            dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, l % 4, out=outs[l])
            if ev is not None:
                ev[l][1].record(stream)
            dig.dwconv3x3(outs[l].view(w.B, w.Hgrid, w.Wgrid, w.C), cws[l], out=convs[l])
            if ev is not None:
                ev[l][2].record(stream)
            if with_reorient:
                dig.srem_reorient(convs[l].view(w.B, w.T, w.C), (l + 1) % 4, 0, w.Hgrid, w.Wgrid, out=reor[l])
            if ev is not None:
                ev[l][3].record(stream)

    res = {"workload": w.name, "layers": L, "dirs": "layer % 4", "inputs": "fresh per layer, seed = layer",
           "reps": reps}
    for with_reorient in (True, False):
        run(with_reorient)
        totals, gla, conv, reo = [], [], [], []
        for _ in range(reps):
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(L)]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            run(with_reorient, ev)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            totals.append(e0.elapsed_time(e1) * 1e3)
            gla += [e[0].elapsed_time(e[1]) * 1e3 for e in ev]
            conv += [e[1].elapsed_time(e[2]) * 1e3 for e in ev]
            if with_reorient:
                reo += [e[2].elapsed_time(e[3]) * 1e3 for e in ev]
        us = statistics.median(totals)
        key = "with_reorient" if with_reorient else "without_reorient"
        res[key] = {"stack_us": us, "tokens_heads_per_s": w.token_heads * L / (us / 1e6),
                    "gla_fwd_us_per_layer": statistics.mean(gla), "dwconv3x3_us_per_layer": statistics.mean(conv)}
        if with_reorient:
            res[key]["srem_reorient_us_per_layer"] = statistics.mean(reo)
    gla_bytes = (2 * (2 * w.dk + w.dv) + 4 * w.dk + 2 * w.dv) * w.token_heads
    res["gla_fwd_frac_of_hbm"] = gla_bytes / (res["with_reorient"]["gla_fwd_us_per_layer"] / 1e6) / 1e9 / hbm
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the c5 stack: {dig.status_string(status)}")
    del ins, outs, convs, reor
    return res


def long_window(dig, dev, stream, dev_in, outs, hbm, seconds=1.0, gla_us_hint=220.0):
    """c4 GLA forward alone, back to back over the four directions for at least
    `seconds` of device time (each launch on its own layer's inputs, 347 MB > L2), with
    its own clock samples: median per direction and the mean."""
    w = WORKLOAD
    rounds = int(seconds * 1e6 / (4 * gla_us_hint)) + 1
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(4)]
          for _ in range(rounds)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index or 0) as clk:
        e0.record(stream)
        for r in range(rounds):
            for l in range(4):
                q, k, v, la = dev_in[l]
                ev[r][l][0].record(stream)
                dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, l, out=outs[l])
                ev[r][l][1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    per_dir = [[ev[r][l][0].elapsed_time(ev[r][l][1]) * 1e3 for r in range(rounds)] for l in range(4)]
    allv = [x for d in per_dir for x in d]
    mean_us = statistics.mean(allv)
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the long window: {dig.status_string(status)}")
    return {"launches": 4 * rounds, "window_s": e0.elapsed_time(e1) / 1e3,
            "median_us_by_dir": [statistics.median(d) for d in per_dir], "mean_us": mean_us,
            "p90_us": sorted(allv)[int(0.9 * len(allv))],
            "tokens_heads_per_s": w.token_heads / (mean_us / 1e6),
            "frac_of_hbm": GLA_BYTES_PER_TOKEN_HEAD * w.token_heads / (mean_us / 1e6) / 1e9 / hbm,
            "clocks": clk.summary()}


def bwd_configs(dig, dev, stream, hbm, reps=5):
    """The GLA backward (gla_bwd, bf16) on c4 and c2: median of `reps` calls per
    direction, event-timed, inputs resident in HBM, against the HBM roofline of its
    algorithmic bytes: q, k, v, dout, log_alpha read once, dq, dk, dv, dlog_alpha
    written once."""
    res = {}
    for name in ("c4", "c2"):
        cw = workloads.WORKLOADS[name]
        q, k, v, la = [t.to(dev) for t in workloads.gla_inputs(cw, seed=11)]
        do = workloads.gla_dout(cw, seed=11).to(dev)
        per_th = 2 * (2 * cw.dk + 2 * cw.dv) + 4 * cw.dk + 2 * (2 * cw.dk + cw.dv) + 4 * cw.dk
        nbytes = per_th * cw.token_heads
        per_dir = []
        for d in range(4):
            dig.gla_bwd(q, k, v, la, do, cw.Hgrid, cw.Wgrid, d)
            per_dir.append(device_us(lambda: dig.gla_bwd(q, k, v, la, do, cw.Hgrid, cw.Wgrid, d), stream, reps))
        us = statistics.mean(per_dir)
        if name == "c2":
            import oracle
            hq, hk, hv, hla = workloads.gla_inputs(cw, seed=11)
            hdo = workloads.gla_dout(cw, seed=11)
            res["cpu_baseline"] = oracle_beside(
                lambda: oracle.gla_bwd(hq, hk, hv, hla, hdo, cw.Hgrid, cw.Wgrid, 0), cw.token_heads,
                "fp64 oracle reverse sweep, c2 whole (48 heads), direction 0, all host threads")
        res[name] = {"workload": cw.name, "kernel": "gla_bwd (3 launches: local terms, chunk scans, gradients)",
                     "us_per_dir": per_dir, "bytes": nbytes, "bytes_per_token_head": per_th,
                     "tokens_heads_per_s": cw.token_heads / (us / 1e6),
                     "frac_of_hbm": nbytes / (us / 1e6) / 1e9 / hbm}
        del q, k, v, la, do
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the backward: {dig.status_string(status)}")
    return res


def zigzag_c4(dig, dev, stream, dev_in, outs, hbm, reps=5):
    """The c4 GLA forward along the eight zigzag orders (codes 4..11): each call gathers
    q, k, v, log_alpha into the scan order, scans, and scatters the output back.  Median
    of `reps` calls per scheme; the fraction is on the GLA's own algorithmic bytes (the
    arranged copies are extra traffic)."""
    w = WORKLOAD
    q, k, v, la = dev_in[0]
    per = []
    for j in range(8):
        dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j, out=outs[0])
        per.append(device_us(lambda: dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j, out=outs[0]), stream, reps))
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the zigzag orders: {dig.status_string(status)}")
    import oracle
    hq, hk, hv, hla = (t.double().numpy() for t in workloads.gla_inputs(w, seed=0))
    cpu = oracle_beside(lambda: oracle.gla_fwd(hq, hk, hv, hla, w.Hgrid, w.Wgrid, 4, heads=(0, 16)),
                        16 * w.T, "fp64 oracle, c4 heads 0..15 of 32 along zigzag scheme 0, all host threads")
    us = statistics.mean(per)
    gla_bytes = GLA_BYTES_PER_TOKEN_HEAD * w.token_heads
    copy_bytes = 2 * (2 * (2 * w.dk + w.dv) + 4 * w.dk + 2 * w.dv) * w.token_heads  # gathers + scatter
    return {"us_per_scheme": per, "tokens_heads_per_s": w.token_heads / (us / 1e6),
            "frac_of_hbm": gla_bytes / (us / 1e6) / 1e9 / hbm,
            "bytes_moved_incl_arranging": gla_bytes + copy_bytes, "cpu_baseline": cpu}


def norm_configs(dig, dev, stream, hbm, reps=5):
    """The normalised variant (gla_norm_fwd, bf16) on c4 and c2: median of `reps` calls
    per direction; the fraction is on its algorithmic bytes (q, k, v read once, out
    written once, bf16)."""
    res = {}
    for name in ("c4", "c2"):
        cw = workloads.WORKLOADS[name]
        q, k, v, _ = [t.to(dev) for t in workloads.gla_inputs(cw, seed=13)]
        per_th = 2 * (2 * cw.dk + cw.dv) + 2 * cw.dv
        per_dir = []
        for d in range(4):
            dig.gla_norm_fwd(q, k, v, cw.Hgrid, cw.Wgrid, d)
            per_dir.append(device_us(lambda: dig.gla_norm_fwd(q, k, v, cw.Hgrid, cw.Wgrid, d), stream, reps))
        us = statistics.mean(per_dir)
        if name == "c2":
            import oracle
            hq, hk, hv, _ = workloads.gla_inputs(cw, seed=13)
            res["cpu_baseline"] = oracle_beside(
                lambda: oracle.gla_norm_fwd(hq, hk, hv, cw.Hgrid, cw.Wgrid, 0), cw.token_heads,
                "fp64 oracle of the normalised variant, c2 whole (48 heads), direction 0, all host threads")
        res[name] = {"workload": cw.name, "kernels": "prep + fp32 chunk-wise GLA (3) + post",
                     "us_per_dir": per_dir, "bytes_per_token_head": per_th,
                     "tokens_heads_per_s": cw.token_heads / (us / 1e6),
                     "frac_of_hbm": per_th * cw.token_heads / (us / 1e6) / 1e9 / hbm}
        del q, k, v
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the normalised variant: {dig.status_string(status)}")
    return res


def glogit_c4(dig, dev, stream, hbm, reps=10):
    """The c4 GLA forward with bf16 gate logits (gla_fwd_glogit: log_alpha =
    logsigmoid(g)/16 inside the kernel), median of `reps` calls per direction; its
    algorithmic bytes are q, k, v, g and out in bf16 (720 B per token-head at d = 72)."""
    w = WORKLOAD
    q, k, v, g = [t.to(dev) for t in workloads.gla_inputs_glogit(w, seed=17)]
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    per_th = 2 * (2 * w.dk + w.dv) + 2 * w.dk + 2 * w.dv
    per_dir = []
    for d in range(4):
        for _ in range(2):
            dig.gla_fwd_glogit(q, k, v, g, w.Hgrid, w.Wgrid, d, out=out)
        per_dir.append(device_us(lambda: dig.gla_fwd_glogit(q, k, v, g, w.Hgrid, w.Wgrid, d, out=out), stream, reps))
    status = dig.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the gate-logit forward: {dig.status_string(status)}")
    import oracle
    hq, hk, hv, hg = workloads.gla_inputs_glogit(w, seed=17)
    cpu = oracle_beside(lambda: oracle.gla_fwd_glogit(hq, hk, hv, hg, w.Hgrid, w.Wgrid, 0, 16.0), w.token_heads,
                        "fp64 oracle with gate logits, c4 whole (32 heads), direction 0, all host threads")
    us = statistics.mean(per_dir)
    return {"cpu_baseline": cpu, "us_per_dir": per_dir, "bytes_per_token_head": per_th,
            "tokens_heads_per_s": w.token_heads / (us / 1e6),
            "frac_of_hbm": per_th * w.token_heads / (us / 1e6) / 1e9 / hbm}


def per_kernel(w, gla_ms, conv_ms, reor_ms, hbm):
    """Achieved algorithmic GB/s (and TFLOP/s for the GLA) of each op of a layer and of
    the layer as a whole, from the event-timed means, with the fraction of the HBM peak."""
    grid_bytes = 2 * w.B * w.T * w.C * 2  # bf16 in + out, dwconv and reorient alike
    rows = {"gla_fwd": (statistics.mean(gla_ms), GLA_BYTES_PER_TOKEN_HEAD * w.token_heads,
                        GLA_FLOP_PER_TOKEN_HEAD * w.token_heads),
            "dwconv3x3": (statistics.mean(conv_ms), grid_bytes, 18 * w.B * w.T * w.C),
            "srem_reorient": (statistics.mean(reor_ms), grid_bytes, 0)}
    out = {}
    tot_ms = tot_b = 0.0
    for name, (ms, nbytes, flops) in rows.items():
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"us": ms * 1e3, "bytes": nbytes, "GB_per_s": gbs, "frac_of_hbm": gbs / hbm,
                     "TFLOP_per_s": flops / (ms / 1e3) / 1e12}
        tot_ms += ms
        tot_b += nbytes
    out["layer"] = {"us": tot_ms * 1e3, "bytes": tot_b, "GB_per_s": tot_b / (tot_ms / 1e3) / 1e9,
                    "frac_of_hbm": tot_b / (tot_ms / 1e3) / 1e9 / hbm}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the supplementary GLA timings on the c2, c3 and c5 shapes")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the long c4 GLA window and the 28-layer c5 stack")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
