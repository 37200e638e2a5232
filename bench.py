#!/usr/bin/env python
"""Benchmark: U-Net denoiser steps/s (batch 1, BF16) and TFLOP/s on B200.

One step = one whole SD2.1-base-shaped denoiser timestep (latent 4x96x96,
context 77x1024, t = 500) through ``sd_unet_step``, captured once in a CUDA
graph and replayed. Weights are random-init BF16 (N(0, 1/fan_in)), inputs
N(0, 1) BF16, all seeded and synthetic. The 1.73 GB of weights streamed by
every step exceed the 126 MB L2, so no flush is needed between steps.

Multi-GPU: the step does not shard (a spatial split would need a halo
exchange per convolution and global GroupNorm statistics), so N GPUs run N
independent replicas with no collective on the data path ("replicas",
weak scaling); the value is the sum over ranks of steps/s, taken from the
slowest rank's device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "U-Net denoiser steps/sec (batch 1, BF16) and TFLOP/s as % of B200 BF16 peak"
UNIT = "steps/s"
WORKLOAD_ID = 5
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CPU_SAMPLE = "mid block of the step: ResnetBlock2D + Transformer2DModel + ResnetBlock2D at 1280x12x12"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--launch-records", default=None, help="write the per-launch records (JSON) to this path")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:  # noqa: BLE001
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id is not None:
            cmd += ["-i", str(self.gpu_id)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:  # noqa: BLE001
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- oracle sample (CPU)

MID_PREFIXES = ("mid.", "time.")


def measured_traffic(kernel):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary, or None
    when there is none or the kernel's source changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_dram_traffic_unet_step_sd21_96.md")
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":", 1)[0] in ("traffic_bytes_per_launch", "source", "source_sha256"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    try:
        src = os.path.join(ROOT, fields["source"])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if digest != fields["source_sha256"]:
            return None
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, OSError, ValueError):
        return None


def mid_params(seed=4, canonical_unet=None):
    """Oracle parameters of the time MLP and the mid block of the SD2.1-base
    U-Net: sliced from the canonical buffer when given, else drawn from the
    generator (the same values)."""
    import numpy as np

    from oracle import model
    from latent_diffusion_net_b200 import synth

    params = {}
    off = 0
    for k, (name, shape, kind, fan) in enumerate(model.enumerate_unet_params(model.SD21_BASE)):
        n = int(np.prod(shape))
        if name.startswith(MID_PREFIXES):
            if canonical_unet is not None:
                params[name] = synth.bf16_bits_to_f32(canonical_unet[off:off + n]).reshape(shape)
            else:
                params[name] = synth.param_value(seed, k, shape, kind, fan)
        off += n
    return params


MID_PARTS = ("mid.res.0", "mid.attn.0", "mid.res.1")


def mid_part_flops(part):
    hw, C = 144, 1280
    if part.startswith("mid.res"):
        return 2 * (2.0 * hw * C * C * 9) + 2.0 * 1280 * C
    return 2 * (2.0 * hw * C * C) + (2.0 * hw * C * 3 * C + 4.0 * hw * hw * C + 2.0 * hw * C * C) \
        + (2.0 * hw * C * C + 2.0 * 77 * 1024 * 2 * C + 4.0 * hw * 77 * C + 2.0 * hw * C * C) \
        + (2.0 * hw * C * 8 * C + 2.0 * hw * 4 * C * C)


class OracleSample:
    """The oracle on the three parts of the step's mid block (ResnetBlock2D,
    Transformer2DModel, ResnetBlock2D at 1280x12x12), one part per call."""

    def __init__(self, params):
        import numpy as np

        import oracle
        from latent_diffusion_net_b200 import synth
        self.oracle = oracle
        self.p = params
        self.x = synth.normal_bf16(99, 0, (1280, 12, 12)).astype(np.float64)
        self.ctx = synth.normal_bf16(99, 1, (77, 1024)).astype(np.float64)
        self.temb = oracle.time_mlp(params, 500.0)
        self.i = 0

    def run_one(self):
        part = MID_PARTS[self.i % 3]
        self.i += 1
        if part.startswith("mid.res"):
            self.oracle.resblock(self.x, self.temb, self.p, part)
        else:
            self.oracle.transformer(self.x, self.ctx, self.p, part, 1)
        return mid_part_flops(part)


def oracle_mid_block_sample(params, target_seconds, max_parts=300):
    """Oracle FLOP rate on the mid block, parts run in order until about
    ``target_seconds`` of CPU work (whole mid blocks only); returns
    (seconds, FLOPs, parts run)."""
    s = OracleSample(params)
    fl = 0.0
    t0 = time.perf_counter()
    while True:
        fl += s.run_one()
        el = time.perf_counter() - t0
        if (s.i % 3 == 0 and el >= target_seconds) or s.i >= max_parts:
            break
    return el, fl, s.i


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- reference arm

def slowest_rank_ms(ms, world, device=None):
    """Per-step time of the slowest rank (max over ranks); the local value for one rank.
    Every rank must call it at the same point (it is a collective for world > 1)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_steps_per_s(ms_step, world):
    """Whole-job throughput of `world` independent replicas, each timed by the slowest rank."""
    return world * 1e3 / ms_step


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step is the bounded mid-block
    sample, and the value is the oracle's FLOP rate over that sample converted
    to whole denoiser steps per second."""
    if rank != 0:
        return 0
    from latent_diffusion_net_b200.harness import flops

    params = mid_params(seed=4)
    step_flops = flops(WORKLOAD_ID)
    sample = OracleSample(params)
    for _ in range(args.warmup):
        sample.run_one()
    sample.i = 0
    t0 = time.perf_counter()
    fl = 0.0
    for _ in range(args.steps):
        fl += sample.run_one()
    el = time.perf_counter() - t0
    steps_per_s = (fl / el) / step_flops
    line = {"metric": METRIC, "value": steps_per_s, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 / steps_per_s, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "sd21_base_unet_step_96", "latent": [1, 4, 96, 96], "context": [1, 77, 1024],
                       "timestep": 500},
            "cpu_baseline": {"value": steps_per_s, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": f"{CPU_SAMPLE}: one of its three blocks per step, in turn ({args.steps} steps, "
                                       f"{fl / 1e9:.1f} GFLOP in {el:.1f} s), converted to whole steps by FLOPs "
                                       f"({step_flops / 1e9:.1f} GFLOP per step)"},
            "e2e": {"value": steps_per_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    from latent_diffusion_net_b200 import binding as B
    from latent_diffusion_net_b200 import build as _build
    from latent_diffusion_net_b200.harness import Workload, flops
    from latent_diffusion_net_b200.workloads import WORKLOADS

    if not os.path.exists(B.LIB_PATH):
        _build.build()
    peaks, peak_src = load_peaks()
    spec = WORKLOADS[WORKLOAD_ID]
    step_flops = flops(WORKLOAD_ID)
    torch.cuda.reset_peak_memory_stats(dev)
    wl = Workload(WORKLOAD_ID, device=dev)
    stream = torch.cuda.Stream(device=dev)

    # eager warm-up; the first one records launch events so that capture can reuse them
    with torch.cuda.stream(stream):
        B.sd_profile_begin()
        wl.step(stream)
        n_launch = B.sd_profile_end()
        for _ in range(max(args.warmup, 3)):
            wl.step(stream)
    stream.synchronize()
    st = B.sd_query_device_status(wl.modules[0].ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # graph of one step (headline) and the same step with per-launch event nodes
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        wl.step(torch.cuda.current_stream())
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=stream):
        B.sd_profile_begin()
        wl.step(torch.cuda.current_stream())
        n_graph = B.sd_profile_end()
    assert n_graph == n_launch, (n_graph, n_launch)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        pgraph.replay()
    stream.synchronize()

    # ------------------------------------------------------------- timed region
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        gpu_id = None
    clocks = ClockSampler(gpu_id)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches_before = B.sd_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms_total = ev0.elapsed_time(ev1)
    ms_step = ms_total / args.steps
    # graph replays do not pass through the host library: every replay launches the captured kernels
    gpu_launches = n_graph * args.steps + (B.sd_launch_count() - launches_before)
    ms_step = slowest_rank_ms(ms_step, world, dev)
    value = aggregate_steps_per_s(ms_step, world)
    tflops = step_flops / (ms_step * 1e-3) / 1e12

    # second timed region: the same step with an event pair around every launch
    # (the event nodes add a few microseconds each, so this region is not the headline)
    prof_steps = max(1, min(args.steps, 20))
    with torch.cuda.stream(stream):
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for _ in range(prof_steps):
            pgraph.replay()
        p1.record(stream)
    torch.cuda.synchronize(dev)
    ms_profiled = p0.elapsed_time(p1) / prof_steps

    # per-launch device times of the last profiled replay (events inside the graph)
    recs = B.sd_profile_read()
    if args.launch_records and rank == 0:
        with open(args.launch_records, "w") as f:
            json.dump(recs, f)
    fam = {}
    for r in recs:
        f = fam.setdefault(r["kernel"], {"ms": 0.0, "flops": 0.0, "bytes": 0.0, "launches": 0})
        f["ms"] += max(r["ms"], 0.0)
        f["flops"] += r["flops"]
        f["bytes"] += r["bytes"]
        f["launches"] += 1
    if not any(f["ms"] > 0 for f in fam.values()):
        raise RuntimeError("per-launch event times unavailable")
    dom_name = max(fam, key=lambda k: fam[k]["ms"])
    dom = fam[dom_name]
    avg_ms = dom["ms"] / dom["launches"]
    if dom["flops"] > 0:
        achieved = dom["flops"] / dom["launches"] / (avg_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"kernel": dom_name, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": measured_traffic(dom_name),
                "traffic_unit": "bytes per launch (ncu dram read + write, committed summary)",
                "algorithmic_bytes_per_launch": dom["bytes"] / dom["launches"],
                "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
                "launches_per_step": dom["launches"], "avg_launch_us": avg_ms * 1e3,
                "algorithmic_flops_per_launch": dom["flops"] / dom["launches"],
                "measured": "last replay of the profiled step graph (per-launch CUDA event pairs)"}
    else:
        achieved = dom["bytes"] / dom["launches"] / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": dom_name, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None, "peak_source": f"{peak_src} HBM copy",
                "launches_per_step": dom["launches"], "avg_launch_us": avg_ms * 1e3}
    step_kernel_ms = sum(f["ms"] for f in fam.values())
    breakdown = {k: {"ms": round(v["ms"], 4), "share": round(v["ms"] / step_kernel_ms, 4), "launches": v["launches"],
                     "tflops": round(v["flops"] / (v["ms"] * 1e-3) / 1e12, 1) if v["flops"] and v["ms"] > 0 else None,
                     "gbs": round(v["bytes"] / (v["ms"] * 1e-3) / 1e9, 1) if v["ms"] > 0 else None}
                 for k, v in sorted(fam.items(), key=lambda kv: -kv[1]["ms"])}

    # ------------------------------------------------------------- end to end through the ABI
    lat_h = wl.dev_inputs["x"].cpu().pin_memory()
    ctx_h = wl.dev_inputs["ctx"].cpu().pin_memory()
    eps_h = torch.empty(wl.out.shape, dtype=torch.bfloat16).pin_memory()
    lat_d = torch.empty_like(wl.dev_inputs["x"])
    ctx_d = torch.empty_like(wl.dev_inputs["ctx"])
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(e2e_steps + 2):
            if i == 2:
                torch.cuda.synchronize(dev)
                t_wall = time.perf_counter()
                e0.record(stream)
            lat_d.copy_(lat_h, non_blocking=True)
            ctx_d.copy_(ctx_h, non_blocking=True)
            out = wl.step(stream, latent=lat_d, context=ctx_d)
            eps_h.copy_(out, non_blocking=True)
            stream.synchronize()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t_wall
    e2e_ms = max(e0.elapsed_time(e1), wall * 1e3) / e2e_steps
    e2e_ms = slowest_rank_ms(e2e_ms, world, dev)
    e2e = {"value": aggregate_steps_per_s(e2e_ms, world), "unit": UNIT, "h2d_bytes_per_step": lat_h.numel() * 2 + ctx_h.numel() * 2,
           "d2h_bytes_per_step": eps_h.numel() * 2, "ms_per_step": e2e_ms,
           "path": "pinned host latent+context -> device, sd_unet_step (eager ABI call), eps -> pinned host, "
                   "stream synchronised every step"}
    st = B.sd_query_device_status(wl.modules[0].ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")
    peak_mem = torch.cuda.max_memory_allocated(dev) / 2 ** 30

    # ------------------------------------------------------------- CPU baseline (oracle)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, fl, parts = oracle_mid_block_sample(mid_params(canonical_unet=wl.canonical[0]), args.cpu_seconds)
        cpu_steps = (fl / sec) / step_flops
        cpu = {"value": cpu_steps, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{CPU_SAMPLE}: {parts // 3} mid block(s), {fl / 1e9:.1f} GFLOP in {sec:.1f} s, "
                         f"converted to whole steps by FLOPs ({step_flops / 1e9:.1f} GFLOP per step)"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec["name"], "latent": [1, 4, spec["H"], spec["W"]],
                       "context": [1, 77, spec["ctx_dim"]], "timestep": 500, "params": 865910724,
                       "global_batch": world, "parallelism": f"replicas x{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2: 1.73 GB of BF16 weights streamed per step (L2 126 MB)",
                       "timing": "CUDA graph of one step replayed K times, CUDA events on the launching stream; "
                                 "per-kernel times from a second region replaying the same step with an event "
                                 "pair around every launch"},
            "ms_per_step_with_launch_events": ms_profiled,
            "tflops": tflops, "tflops_frac_of_peak": tflops / peaks["bf16_tflops_sustained"],
            "peak_source": peak_src, "roofline": roof, "kernel_breakdown": breakdown,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches, "launches_per_step": n_graph,
            "clocks": clk, "max_memory_allocated_gib": round(peak_mem, 3)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, pgraph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
