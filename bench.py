"""Benchmark of the group-wise fully quantized int8 Winograd convolution on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload resnet18] [--impl reference]

One step = one pass of the whole hot path over one batch: the input
transform with its group-wise int8 quantisation, the Hadamard int8 GEMM(s)
with per-K-group dequantisation and Y absmax, Y requantisation and the output
transform (wino_conv2d_int8).  The weight transform is offline (once per
layer) and is not part of a step.

Metric: direct-convolution-equivalent TFLOP/s, 2 N H W Cin Cout 9 / time,
whole job (all ranks).  Default workload: the ResNet-18-like layer, F(6,3),
N32 C64 56x56 bf16, seeded synthetic inputs.  L2 is flushed (a 256 MiB write)
before every timed step; each step is timed with CUDA events on the stream
the kernels run on, and the run's time is the sum of the step times (max over
ranks).  Multi-GPU: each rank runs its own batch (weak scaling, no
collective on the data path).

--impl reference times the CPU oracle (the plain C++ restatement of the
method in oracle/) on the host cores for the same workload and metric, each
step a bounded sample of tile rows of the layer.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_wise_int8_b200 import synth  # noqa: E402

METRIC = "direct-conv-equiv TFLOP/s per layer; % of int8 tensor-core / HBM roofline"
UNIT = "TFLOP/s"

# DRAM bytes per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum); the summary with its command
# line is the named file under profiles/.  None until a capture of the
# current kernel exists.
NCU_TRAFFIC = {
    # (workload, layer, kernel) -> dram read+write bytes per launch from one ncu capture of the
    # CURRENT kernel (summarised under profiles/); entries are removed whenever that kernel changes.
    ("resnet18", 0, "input_transform"): 12912896,
    ("resnet18", 0, "hadamard_absmax"): 15109632,
    ("resnet18", 0, "hadamard_quant"): 15120128,
    ("resnet18", 0, "output_transform"): 13168896,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="resnet18",
                    help="resnet18 (default) | resnet34:<i> | sd15:<i> | sd15_stack:<i> | probe:<i>")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--y-groups", default="tile", choices=["tile", "tap"],
                    help="Y quantisation groups: tile (default reading) or tap (the per-tap option)")
    ap.add_argument("--x-int8", action="store_true",
                    help="alternative reading: x group-quantised per pixel before the input transform")
    ap.add_argument("--int8-transforms", action="store_true",
                    help="alternative reading: B^T and A^T held as int8 with one scale per matrix")
    return ap.parse_args()


def pick_layer(name: str) -> synth.Layer:
    if ":" in name:
        w, i = name.split(":")
        return synth.workload(w)[int(i)]
    return synth.workload(name)[0]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs"), "bf16_tflops": d.get("bf16_tflops"),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------- byte model
def stage_model(layer: synth.Layer, y_path: int, x_int8: bool = False):
    """Algorithmic bytes and int8 ops of each launch of one call, by launch index."""
    from group_wise_int8_b200 import wino
    n2 = layer.n * layer.n
    T = layer.tiles
    G = layer.group
    xs = 2 if layer.dtype == "bf16" else 4
    x = layer.N * layer.H * layer.W * layer.Cin * xs
    out = layer.N * layer.H * layer.W * layer.Cout * 2
    v = T * n2 * layer.Cin + 4 * T * n2 * (layer.Cin // G)
    u = n2 * layer.Cout * layer.Cin + 4 * n2 * (layer.Cin // G) * layer.Cout
    amax = 4 * T * (layer.Cout // G)
    yq = T * n2 * layer.Cout
    ops = 2.0 * T * n2 * layer.Cin * layer.Cout
    stages = []
    if x_int8:   # reads x, writes its fp32 round trip, which the input transform then reads
        xq = layer.N * layer.H * layer.W * layer.Cin * 4
        stages.append(("input_quant", x + xq, 0.0))
        x = xq
    stages.append(("input_transform", x + v + amax, 0.0))
    if y_path == wino.YPATH_RECOMPUTE:
        stages.append(("hadamard_absmax", v + u + amax, ops))
        stages.append(("hadamard_quant", v + u + amax + yq, ops))
        stages.append(("output_transform", yq + amax + out, 0.0))
    else:
        stages.append(("hadamard_y32", v + u + amax + 4 * yq, ops))
        stages.append(("output_transform", 4 * yq + amax + out, 0.0))
    return stages


# ---------------------------------------------------------------- clock sampler
class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = str(bus_id or "").lower()
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader",
                                          "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        if self.bus_id:
            mine = [r for r in rows if r and r[0].lower().endswith(self.bus_id[-12:])]
            rows = mine or rows
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1].split()[0]))
                smax = float(r[2].split()[0])
                for nm, val in zip(names, r[5:9]):
                    if val.strip() == "Active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        under_load = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(under_load), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- multi-rank
def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (all ranks call it, in the same order)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job rate (weak scaling: every rank processes its own batch)."""
    return world * units_per_rank / (max_ms * 1e-3)


# --------------------------------------------------------------- our CUDA path
def run_ours(args, layer, rank, world):
    import torch
    import torch.distributed as dist
    from group_wise_int8_b200 import build, wino

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    build.build()
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    y_groups = wino.YGROUPS_TAP if getattr(args, "y_groups", "tile") == "tap" else wino.YGROUPS_TILE
    plan = wino.Plan(layer.m, layer.points, sb, sg, layer.group, y_groups=y_groups, x_int8=args.x_int8,
                     int8_transforms=args.int8_transforms)
    N, H, W, Cin, Cout = layer.N, layer.H, layer.W, layer.Cin, layer.Cout
    if x_bits is not None:
        x = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(x_f32).to(dev)
    wt = plan.transform_weights(torch.from_numpy(w).to(dev))
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device=dev)
    y = torch.empty((N, H, W, Cout), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    y_path, gemm = plan.resolved_config(N, H, W, Cin, Cout)
    launches = plan.launches_per_call(N, H, W, Cin, Cout)

    for _ in range(args.warmup):
        flush.fill_(1)
        plan.conv2d(x, wt, Cout, out=y, workspace=ws)
    torch.cuda.synchronize()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    bus = None
    try:
        pr = torch.cuda.get_device_properties(dev)
        bus = "%08X:%02X:%02X.0" % (int(pr.pci_domain_id), int(pr.pci_bus_id), int(pr.pci_device_id))
    except Exception:
        pass
    sampler = ClockSampler(bus)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xff)
        starts[i].record(stream)
        plan.conv2d(x, wt, Cout, out=y, workspace=ws)
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    # Per-kernel breakdown: a second pass of the same steps with an event between every two
    # kernels (events between kernels stop the next kernel's launch from overlapping the
    # previous one's tail, so this pass is kept out of the timed region above).
    prof_steps = min(args.steps, 500)
    plan.profile_begin(prof_steps)
    for i in range(prof_steps):
        flush.fill_(i & 0xff)
        plan.conv2d(x, wt, Cout, out=y, workspace=ws)
    torch.cuda.synchronize()
    stage_ms, calls = plan.profile_end()
    assert calls == prof_steps
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), world, dev)

    # end to end through the host-buffer entry point (H2D of x, conv, D2H of y per step)
    e2e = None
    if args.e2e_steps > 0:
        xs = x.element_size()
        x_host = x.cpu().pin_memory()
        y_host = torch.empty((N, H, W, Cout), dtype=torch.bfloat16).pin_memory()
        ws_h = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) +
                           plan.host_staging_bytes(N, H, W, Cin, Cout, x.dtype, torch.bfloat16),
                           dtype=torch.uint8, device=dev)
        for _ in range(3):
            plan.conv2d_host(x_host, wt, Cout, y_host, ws_h)
        torch.cuda.synchronize()
        k = args.e2e_steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(k):
            plan.conv2d_host(x_host, wt, Cout, y_host, ws_h)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_throughput(k * layer.direct_flops, world, e_ms) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(N * H * W * Cin * xs), "d2h_bytes_per_step": int(N * H * W * Cout * 2),
               "steps": k, "ms_per_step": e_ms / k}

    # roofline of the dominant kernel
    peaks = load_peaks()
    model = stage_model(layer, y_path, args.x_int8)
    avg_ms = [t / calls for t in stage_ms]
    dom = int(np.argmax(avg_ms))
    name, nbytes, ops = model[dom]
    achieved_gbs = nbytes / (avg_ms[dom] * 1e-3) / 1e9
    traffic = NCU_TRAFFIC.get((layer.workload, layer.index, name))
    roofline = {"kernel": name, "bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
                "traffic": traffic, "algorithmic_bytes": int(nbytes), "avg_launch_us": round(avg_ms[dom] * 1e3, 2),
                "peak_source": peaks["source"] + " (hbm_gbs, copy test)",
                "launch_timing": "CUDA events between kernels on the launching stream, second pass of %d steps "
                                 "right after the timed region" % calls}
    per_kernel = [{"kernel": m[0], "avg_us": round(a * 1e3, 2), "algorithmic_bytes": int(m[1]),
                   "gbs": round(m[1] / (a * 1e-3) / 1e9, 1),
                   "int8_tops": round(m[2] / (a * 1e-3) / 1e12, 2) if m[2] else None}
                  for m, a in zip(model, avg_ms)]
    ms_step = total_ms / args.steps
    value = job_throughput(args.steps * layer.direct_flops, world, total_ms) / 1e12
    return {
        "value": value, "ms_per_step": ms_step, "e2e": e2e, "roofline": roofline, "clocks": clocks,
        "gpu_launches": args.steps * launches, "per_kernel": per_kernel, "wall_s": t_wall,
        "y_path": {1: "recompute", 2: "y32"}.get(y_path), "gemm": {1: "tcgen05", 2: "simt"}.get(gemm),
    }


# ------------------------------------------------------------- CPU oracle timing
def oracle_sample(layer: synth.Layer, rows: int, images: int, int8_transforms: bool = False):
    """The layer cropped to `rows` tile rows of `images` images (same weights)."""
    import oracle
    x_f32, _ = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    H = min(layer.H, rows * layer.m)
    xs = np.ascontiguousarray(x_f32[:images, :H])
    plan = oracle.Plan(layer.m, layer.points, sb, sg, int8_transforms=int8_transforms)
    Uq, sU, _ = oracle.weight_transform(plan, w, layer.group)
    flops = 2.0 * images * H * layer.W * layer.Cin * layer.Cout * 9
    return plan, xs, Uq, sU, flops


def oracle_step(plan, xs, Uq, sU, G, per_tap=False, x_int8=False):
    import oracle
    n2 = plan.n * plan.n
    N, H, W, _ = xs.shape
    if x_int8:
        xs = oracle.quantize_input(xs, G)
    Vq, sV, _ = oracle.input_transform(plan, xs, G)
    Y, _ = oracle.hadamard(n2, Vq, sV, Uq, sU, G)
    Yq, sY = oracle.y_requant(n2, Y, G, per_tap)
    oracle.output_transform(plan, Yq, sY, N, H, W, G, per_tap)


def cpu_baseline(layer: synth.Layer, budget_s: float = 12.0, per_tap: bool = False, x_int8: bool = False,
                 int8_transforms: bool = False):
    import oracle
    threads = oracle.set_threads(0)
    rows, images = 1, 1
    plan, xs, Uq, sU, flops = oracle_sample(layer, rows, images, int8_transforms)
    t0 = time.perf_counter()
    oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
    dt = time.perf_counter() - t0
    # grow the sample (whole images first) while it stays within the budget
    TH = -(-layer.H // layer.m)
    while dt * 2 < budget_s / 2 and (rows < TH or images < layer.N):
        if rows < TH:
            rows = min(TH, rows * 2)
        else:
            images = min(layer.N, images * 2)
        plan, xs, Uq, sU, flops = oracle_sample(layer, rows, images, int8_transforms)
        t0 = time.perf_counter()
        oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
        dt = time.perf_counter() - t0
    reps = max(1, int(budget_s / 2 / max(dt, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
    dt = (time.perf_counter() - t0) / reps
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": "%d image(s) x %d of %d tile rows of %s; input transform, Hadamard, Y requant, output "
                      "transform (weights pre-transformed); %d rep(s)" % (images, rows, TH, layer.describe(), reps)}


def run_reference(args, layer):
    per_tap = args.y_groups == "tap"
    x_int8 = args.x_int8
    import oracle
    threads = oracle.set_threads(0)
    TH = -(-layer.H // layer.m)
    budget = 150.0 / max(1, args.steps + args.warmup)   # seconds per step: whole run within a few minutes
    rows = 1
    plan, xs, Uq, sU, flops = oracle_sample(layer, rows, 1, args.int8_transforms)
    t0 = time.perf_counter()
    oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
    dt = time.perf_counter() - t0
    while dt * 2 <= budget and rows < TH:
        rows = min(TH, rows * 2)
        plan, xs, Uq, sU, flops = oracle_sample(layer, rows, 1, args.int8_transforms)
        t0 = time.perf_counter()
        oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
        dt = time.perf_counter() - t0
    for _ in range(args.warmup):
        oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
    total = time.perf_counter() - t0
    value = args.steps * flops / total / 1e12
    sample = "1 image x %d of %d tile rows of %s per step" % (rows, TH, layer.describe())
    return {"value": value, "ms_per_step": total / args.steps * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample}}


def main():
    args = parse()
    layer = pick_layer(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    config = {"workload": "%s[%d]: %s" % (layer.workload, layer.index, layer.describe()), "model": layer.workload,
              "global_batch": layer.N * world, "seq_len": None, "H": layer.H, "W": layer.W, "Cin": layer.Cin,
              "Cout": layer.Cout, "m": layer.m, "group": layer.group, "parallelism": "dp%d" % world,
              "l2": "flushed before every timed step (256 MiB write)", "output": "bf16 NHWC",
              "y_groups": args.y_groups, "x_int8": args.x_int8, "int8_transforms": args.int8_transforms}
    line = {"metric": METRIC, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8 (fp32 transforms)",
            "data": "synthetic (seeded)", "config": config}

    if args.impl == "reference":
        if rank != 0:
            return
        r = run_reference(args, layer)
        line.update(impl="reference", value=r["value"], ms_per_step=r["ms_per_step"], n_gpus=args.gpus,
                    cpu_baseline=r["cpu_baseline"],
                    e2e={"value": r["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
        print(json.dumps(line))
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        r = run_ours(args, layer, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(layer, per_tap=args.y_groups == "tap", x_int8=args.x_int8,
                           int8_transforms=args.int8_transforms)
    line.update(value=r["value"], ms_per_step=r["ms_per_step"], e2e=r["e2e"], roofline=r["roofline"],
                cpu_baseline=cpu, clocks=r["clocks"], gpu_launches=r["gpu_launches"],
                kernels=r["per_kernel"], y_path=r["y_path"], gemm=r["gemm"], impl="ours")
    print(json.dumps(line))


if __name__ == "__main__":
    main()
