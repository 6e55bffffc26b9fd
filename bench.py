"""Benchmark of the group-wise fully quantized int8 Winograd convolution on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload sd15_stack] [--impl reference]

One step = one pass of the whole hot path over one batch of every conv of the
workload: per conv the input transform with its group-wise int8 quantisation,
the Hadamard int8 GEMM(s) with per-K-group dequantisation and Y absmax, Y
requantisation and the output transform (wino_conv2d_int8).  The weight
transform is offline (once per layer, "pre-transformed once") and is not part
of a step.

Default workload: the back-to-back stack of the 44 3x3 ResNet-block convs of
an SD-v1.5-shaped UNet (channels 320/640/1280/1280 on the down and up paths,
latent 64x64, concatenated-skip widths Cin = 960/1920/2560 included), batch
8, F(6,3), G = 64, bf16 Student-t(3) activations with 1 % outlier channels,
seeded scales; every conv has its own seeded input and weights.  L2 is
flushed (a 256 MiB write) once before every step and the 44 convs then run
back to back on one stream, as they would inside a model.  Metric:
direct-convolution-equivalent TFLOP/s = sum over convs of 2 N H W Cin Cout 9
/ step time, whole job (all ranks).  Each step is timed with CUDA events on
the stream the kernels run on; the run's time is the sum of the step times
(max over ranks).  Multi-GPU: each rank runs its own batch (weak scaling, no
collective on the data path).

The same JSON line carries, beside the headline: the ResNet-18-like layer
(F(6,3) N32 C64 56x56 G32) timed the same way with an L2 flush before every
call; a per-layer table of the ResNet-34-shaped and SD-shaped layers; cuDNN
bf16 channels-last convolution of the same shapes for context; the int8
tensor-core peak measured in-run (a large torch._int_mm); and the CPU oracle
on the host cores (all of them, and one thread).

--impl reference times the CPU oracle (the plain C++ restatement of the
method in oracle/) on the host cores for the same workload and metric, each
step a bounded sample of tile rows of the workload's convs.
"""
from __future__ import annotations

import argparse
import collections
import concurrent.futures
import json
import multiprocessing
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

# DRAM bytes per launch of a kernel from one ncu capture of the CURRENT kernel
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by (layer shape, kernel);
# the summary with its command line is the named file under profiles/.  An
# entry is removed whenever its kernel changes.
NCU_TRAFFIC = {
    # profiles/hadamard_y32_swapped_sd15_1280x1280_8x8_full.md: 114,457,344 + 4,860,160 B
    ("F(6,3) N8 1280->1280 8x8 G64", "hadamard_y32"): 119317504,
    # profiles/hadamard_y32_swapped_n80_sd15_1280x1280_16x16_full.md: 120,098,048 + 10,921,472 B
    ("F(6,3) N8 1280->1280 16x16 G64", "hadamard_y32"): 131019520,
    # profiles/hadamard_y32_a_resident_sd15_320x320_64x64_full.md: 32,512,256 + 29,470,208 B
    ("F(6,3) N8 320->320 64x64 G64", "hadamard_y32"): 61982464,
    # profiles/output_transform_y32_sd15_320x320_64x64_full.md: 79,385,600 + 3,409,920 B
    ("F(6,3) N8 320->320 64x64 G64", "output_transform"): 82795520,
    # profiles/input_transform_sd15_320x320_64x64_full.md: 21,031,168 + 85,760 B
    ("F(6,3) N8 320->320 64x64 G64", "input_transform"): 21116928,
    # profiles/hadamard_y32_probe_T2048_C2560_full.md: 6.022703 GB + 1.330437 GB (ncu rounds to 1 kB)
    ("F(6,3) N2 2560->2560 192x192 G64", "hadamard_y32"): 7353140000,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="sd15_stack",
                    help="sd15_stack (default: all 44 convs) | resnet18[:i] | resnet34[:i] | sd15[:i] | "
                         "sd15_stack:<i> | probe:<i>")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the ResNet-18 line, the per-layer table, cuDNN and the int8 peak")
    ap.add_argument("--layer-steps", type=int, default=30, help="timed calls per layer in the per-layer table")
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the host-buffer leg (default: --steps)")
    ap.add_argument("--y-groups", default="tile", choices=["tile", "tap"],
                    help="Y quantisation groups: tile (default reading) or tap (the per-tap option)")
    ap.add_argument("--x-int8", action="store_true",
                    help="alternative reading: x group-quantised per pixel before the input transform")
    ap.add_argument("--int8-transforms", action="store_true",
                    help="alternative reading: B^T and A^T held as int8 with one scale per matrix")
    ap.add_argument("--fused", action="store_true",
                    help="the one-kernel path for small channel counts where it applies (off by default)")
    return ap.parse_args()


def pick_layers(name: str):
    """(label, layers): a whole workload, or one layer of it with 'workload:i'."""
    if ":" in name:
        w, i = name.split(":")
        layer = synth.workload(w)[int(i)]
        return "%s[%d]: %s" % (w, layer.index, layer.describe()), [layer]
    layers = synth.workload(name)
    if name == "resnet18":
        layers = layers[:1]
    if len(layers) == 1:
        return "%s[0]: %s" % (name, layers[0].describe()), layers
    if name == "sd15_stack":
        l0 = layers[0]
        return ("sd15_stack: the 44 3x3 ResNet-block convs of an SD-v1.5-shaped UNet back to back, "
                "F(%d,3) N%d G%d %s, Cin 320-2560, Cout 320-1280, 64x64..8x8" % (l0.m, l0.N, l0.group, l0.dtype),
                layers)
    return "%s: %d layers" % (name, len(layers)), layers


def shape_key(layer: synth.Layer) -> str:
    return "F(%d,3) N%d %d->%d %dx%d G%d" % (layer.m, layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.group)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs"), "bf16_tflops": d.get("bf16_tflops"),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------- byte model
def stage_model(layer: synth.Layer, y_path: int, x_int8: bool = False, fused: bool = False):
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
    if fused:   # one kernel: x in, the transformed weights, the output out; both GEMM passes
        return [("fused_layer", x + u + out, 2 * ops)]
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


# ------------------------------------------------------ synthetic data (host)
def _gen_layer(layer: synth.Layer):
    """Seeded input (bf16 bits or fp32) and weights of one layer; runs in the spawn pool."""
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    return (x_bits if x_bits is not None else x_f32), w


def generate(layers):
    """Inputs and weights of every layer, in layer order, drawn by a pool of spawned worker
    processes (spawn, so the workers inherit no CUDA state of this process)."""
    if len(layers) == 1:
        return iter([_gen_layer(layers[0])])
    ctx = multiprocessing.get_context("spawn")
    workers = max(1, min(len(layers), (os.cpu_count() or 2) - 1, 16))
    ex = concurrent.futures.ProcessPoolExecutor(max_workers=workers, mp_context=ctx)
    futs = [ex.submit(_gen_layer, l) for l in layers]

    def it():
        try:
            for f in futs:
                yield f.result()
        finally:
            ex.shutdown(wait=True)
    return it()


# --------------------------------------------------------------- our CUDA path
class DevLayer:
    pass


def plan_key(layer: synth.Layer):
    return (layer.m, layer.points, layer.group, layer.workload if layer.scales != "identity" else "identity")


def make_plan(layer: synth.Layer, args, fused=None, y_path=None):
    from group_wise_int8_b200 import wino
    sb, sg = synth.make_scales(layer)
    y_groups = wino.YGROUPS_TAP if getattr(args, "y_groups", "tile") == "tap" else wino.YGROUPS_TILE
    if fused is None:
        fused = wino.FUSED_ON if getattr(args, "fused", False) else wino.FUSED_AUTO
    return wino.Plan(layer.m, layer.points, sb, sg, layer.group, y_groups=y_groups,
                     x_int8=getattr(args, "x_int8", False), int8_transforms=getattr(args, "int8_transforms", False),
                     fused=fused, y_path=wino.YPATH_AUTO if y_path is None else y_path)


def prepare(layers, args, dev, keep_bf16_weights=False):
    """Device copies of every layer: input, transformed weights, output buffer, and the plans
    (one per distinct plan key, shared by the layers that use it)."""
    import torch
    plans = {}
    dls = []
    for layer, (xh, w) in zip(layers, generate(layers)):
        k = plan_key(layer)
        if k not in plans:
            plans[k] = make_plan(layer, args)
        d = DevLayer()
        d.layer, d.plan = layer, plans[k]
        if xh.dtype == np.uint16:
            d.x = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            d.x = torch.from_numpy(xh).to(dev)
        wd = torch.from_numpy(w).to(dev)
        d.wt = d.plan.transform_weights(wd)
        d.w_bf16 = wd.to(torch.bfloat16).permute(0, 3, 1, 2) if keep_bf16_weights else None
        del wd
        d.y = torch.empty((layer.N, layer.H, layer.W, layer.Cout), dtype=torch.bfloat16, device=dev)
        d.shape = (layer.N, layer.H, layer.W, layer.Cin, layer.Cout)
        d.y_path, d.gemm = d.plan.resolved_config(*d.shape)
        d.variants = d.plan.resolved_variants(*d.shape)
        d.launches = d.plan.launches_per_call(*d.shape)
        dls.append(d)
    torch.cuda.synchronize()
    return dls


def run_step(dls, ws, plan_of=None):
    for d in dls:
        p = plan_of(d) if plan_of else d.plan
        p.conv2d(d.x, d.wt, d.layer.Cout, out=d.y, workspace=ws)


def bus_id(dev):
    import torch
    try:
        pr = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (int(pr.pci_domain_id), int(pr.pci_bus_id), int(pr.pci_device_id))
    except Exception:
        return None


def time_steps(dls, ws, flush, stream, steps, warmup):
    """Per-step CUDA-event times (ms) with one L2 flush before each step (outside the events)."""
    import torch
    for i in range(warmup):
        flush.fill_(i & 0xff)
        run_step(dls, ws)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xff)
        starts[i].record(stream)
        run_step(dls, ws)
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def profile_kernels(dls, ws, flush, steps, args):
    """Average duration of every launch of every layer: a pass of `steps` steps with per-layer
    plans whose calls record a CUDA event between kernels (kept out of the timed region: events
    between kernels stop the next kernel's launch from overlapping the previous one's tail)."""
    import torch
    from group_wise_int8_b200 import wino
    pplans = [make_plan(d.layer, args) for d in dls]
    for p in pplans:
        p.profile_begin(steps)
    idx = {id(d): i for i, d in enumerate(dls)}
    for i in range(steps):
        flush.fill_(i & 0xff)
        run_step(dls, ws, plan_of=lambda d: pplans[idx[id(d)]])
    torch.cuda.synchronize()
    out = []
    for d, p in zip(dls, pplans):
        ms, calls = p.profile_end()
        assert calls == steps
        model = stage_model(d.layer, d.y_path, getattr(args, "x_int8", False),
                            bool(d.variants & wino.VARIANT_FUSED))
        assert len(model) == len(ms), (len(model), len(ms))
        out.append([(mk[0], mk[1], mk[2], t / calls) for mk, t in zip(model, ms)])
    return out


def roofline_of(dls, prof, peaks, int8_peak=None):
    """Dominant (layer shape, kernel): the largest summed launch time over the step."""
    tot = collections.defaultdict(float)
    info = {}
    for d, kernels in zip(dls, prof):
        for name, nbytes, ops, ms in kernels:
            key = (shape_key(d.layer), name)
            tot[key] += ms
            info.setdefault(key, []).append((nbytes, ops, ms))
    key = max(tot, key=tot.get)
    runs = info[key]
    nbytes, ops = runs[0][0], runs[0][1]
    avg_ms = sum(r[2] for r in runs) / len(runs)
    achieved = nbytes / (avg_ms * 1e-3) / 1e9
    step_ms = sum(tot.values())
    r = {"kernel": "%s (%s)" % (key[1], key[0]), "bound": "hbm", "achieved": round(achieved, 1),
         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
         "traffic": NCU_TRAFFIC.get(key), "algorithmic_bytes": int(nbytes), "avg_launch_us": round(avg_ms * 1e3, 2),
         "launches_per_step": len(runs), "share_of_kernel_time": round(tot[key] / step_ms, 3),
         "peak_source": peaks["source"] + " (hbm_gbs, copy test)",
         "launch_timing": "CUDA events between kernels on the launching stream, in a second pass right after "
                          "the timed region"}
    if ops and int8_peak:
        r["int8_tops"] = round(ops / (avg_ms * 1e-3) / 1e12, 1)
        r["int8_frac"] = round(ops / (avg_ms * 1e-3) / 1e12 / int8_peak, 4)
    return r


def kernel_table(dls, prof, int8_peak=None, peaks=None):
    """Per distinct layer shape: count, and per kernel the average us, GB/s and fractions."""
    rows = collections.OrderedDict()
    for d, kernels in zip(dls, prof):
        k = shape_key(d.layer)
        row = rows.setdefault(k, {"layer": k, "count": 0, "y_path": {1: "recompute", 2: "y32"}.get(d.y_path),
                                  "variants": d.variants, "acc": collections.defaultdict(list)})
        row["count"] += 1
        for name, nbytes, ops, ms in kernels:
            row["acc"][name].append((nbytes, ops, ms))
    out = []
    for row in rows.values():
        ks = []
        for name, runs in row.pop("acc").items():
            ms = sum(r[2] for r in runs) / len(runs)
            e = {"kernel": name, "avg_us": round(ms * 1e3, 2), "gbs": round(runs[0][0] / (ms * 1e-3) / 1e9, 1)}
            if peaks:
                e["hbm_frac"] = round(runs[0][0] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)
            if runs[0][1]:
                e["int8_tops"] = round(runs[0][1] / (ms * 1e-3) / 1e12, 1)
                if int8_peak:
                    e["int8_frac"] = round(runs[0][1] / (ms * 1e-3) / 1e12 / int8_peak, 4)
            ks.append(e)
        row["kernels"] = ks
        out.append(row)
    return out


def time_e2e(dls, steps, world, dev, stream):
    """The host-buffer entry point: every step copies each conv's input from pinned host memory,
    runs it and copies its output back (wino_conv2d_int8_host)."""
    import torch
    import torch.distributed as dist
    hx = [d.x.cpu().pin_memory() for d in dls]
    hy = [torch.empty(d.y.shape, dtype=torch.bfloat16).pin_memory() for d in dls]
    # the largest convolution workspace plus two stagings: every call finds staging clear of the
    # previous call's, so its input copies overlap the previous call's convolution and output copies
    need = max(d.plan.workspace_bytes(*d.shape) for d in dls) + \
        max(d.plan.host_staging_bytes(*d.shape, d.x.dtype, torch.bfloat16) for d in dls)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def step():
        for d, x_h, y_h in zip(dls, hx, hy):
            d.plan.conv2d_host(x_h, d.wt, d.layer.Cout, y_h, ws)
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    flops = sum(d.layer.direct_flops for d in dls)
    h2d = sum(x.numel() * x.element_size() for x in hx)
    d2h = sum(y.numel() * y.element_size() for y in hy)
    del ws
    return {"value": job_throughput(steps * flops, world, e_ms) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": e_ms / steps, "api": "wino_conv2d_int8_host (pinned host buffers, copies in the call)"}


def time_cudnn(dls, flush, stream, steps, warmup=3):
    """cuDNN bf16 convolution of the same shapes (channels-last), for context."""
    import torch
    import torch.nn.functional as F
    torch.backends.cudnn.benchmark = True
    xs = [d.x.permute(0, 3, 1, 2) if d.x.dtype == torch.bfloat16 else d.x.to(torch.bfloat16).permute(0, 3, 1, 2)
          for d in dls]
    ws_ = [d.w_bf16 for d in dls]

    def step():
        for x, w in zip(xs, ws_):
            F.conv2d(x, w, padding=1)
    for i in range(warmup):
        flush.fill_(i & 0xff)
        step()
    torch.cuda.synchronize()
    times = []
    for i in range(steps):
        flush.fill_(i & 0xff)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        step()
        e.record(stream)
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    ms = sum(times) / len(times)
    flops = sum(d.layer.direct_flops for d in dls)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "what": "torch.nn.functional.conv2d, bf16 NHWC (channels_last), cudnn.benchmark, same shapes"}


def int8_peak_tops(dev, size=8192, reps=10):
    """Dense int8 tensor-core throughput measured in-run: torch._int_mm (cuBLASLt) on size^3."""
    import torch
    try:
        a = torch.randint(-127, 128, (size, size), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (size, size), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            torch._int_mm(a, b)
            e.record()
            torch.cuda.synchronize()
            best = min(best, s.elapsed_time(e))
        return {"int8_tops": round(2.0 * size ** 3 / (best * 1e-3) / 1e12, 1), "how":
                "torch._int_mm int8 %d^3, best of %d (CUDA events)" % (size, reps)}
    except Exception as ex:   # report, do not fail the benchmark
        return {"int8_tops": None, "how": "torch._int_mm unavailable: %s" % str(ex).splitlines()[0][:120]}


def run_ours(args, label, layers, rank, world):
    import torch
    import torch.distributed as dist
    from group_wise_int8_b200 import build, wino

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    build.build(debug=False)
    extras = not args.no_extras and world == 1
    dls = prepare(layers, args, dev, keep_bf16_weights=extras)
    ws = torch.empty(max(d.plan.workspace_bytes(*d.shape) for d in dls), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    for i in range(args.warmup):
        flush.fill_(i & 0xff)
        run_step(dls, ws)
    torch.cuda.synchronize()
    last = dls[-1]   # the error word of the last call on the shared workspace
    assert last.plan.check_device_error(ws, *last.shape) == wino.OK
    sampler = ClockSampler(bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    step_ms = time_steps(dls, ws, flush, stream, args.steps, 0)
    if world > 1:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    assert last.plan.check_device_error(ws, *last.shape) == wino.OK
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    prof = profile_kernels(dls, ws, flush, min(args.steps, 200), args)
    e2e = time_e2e(dls, args.e2e_steps or args.steps, world, dev, stream)

    peaks = load_peaks()
    i8 = int8_peak_tops(dev) if extras else {"int8_tops": None, "how": "not measured (--no-extras)"}
    flops = sum(d.layer.direct_flops for d in dls)
    res = {
        "value": job_throughput(args.steps * flops, world, total_ms) / 1e12, "ms_per_step": total_ms / args.steps,
        "e2e": e2e, "roofline": roofline_of(dls, prof, peaks, i8["int8_tops"]), "clocks": clocks,
        "gpu_launches": args.steps * sum(d.launches for d in dls), "wall_s": t_wall,
        "kernels": kernel_table(dls, prof, i8["int8_tops"], peaks), "int8_peak": i8,
    }
    if extras:
        res["cudnn_bf16"] = time_cudnn(dls, flush, stream, args.steps)
    del dls, ws
    torch.cuda.empty_cache()
    if extras and len(layers) > 1:
        res["y_path_check"] = y_path_check(layers, args, dev, flush, stream, args.layer_steps)
    torch.cuda.empty_cache()
    if extras:
        res["beside"] = layer_line("resnet18", synth.workload("resnet18")[0], args, dev, flush, stream, peaks, i8)
        res["layers"] = [layer_line(w, l, args, dev, flush, stream, peaks, i8)
                         for w in ("resnet34", "sd15") for l in synth.workload(w)]
    return res


def layer_line(wname, layer, args, dev, flush, stream, peaks, i8):
    """One layer timed on its own: L2 flushed before every call."""
    import torch
    dls = prepare([layer], args, dev, keep_bf16_weights=True)
    d = dls[0]
    ws = torch.empty(d.plan.workspace_bytes(*d.shape), dtype=torch.uint8, device=dev)
    steps = args.layer_steps
    ms = time_steps(dls, ws, flush, stream, steps, 3)
    prof = profile_kernels(dls, ws, flush, steps, args)
    cd = time_cudnn(dls, flush, stream, steps)
    avg = sum(ms) / len(ms)
    out = {"layer": "%s[%d]: %s" % (wname, layer.index, layer.describe()), "value": round(layer.direct_flops /
           (avg * 1e-3) / 1e12, 1), "us": round(avg * 1e3, 1),
           "y_path": {1: "recompute", 2: "y32"}.get(d.y_path), "variants": d.variants,
           "kernels": kernel_table(dls, prof, i8["int8_tops"], peaks)[0]["kernels"],
           "roofline": roofline_of(dls, prof, peaks, i8["int8_tops"]),
           "cudnn_bf16_tflops": round(cd["value"], 1), "cudnn_bf16_us": round(cd["ms_per_step"] * 1e3, 1)}
    from group_wise_int8_b200 import wino
    # the Y path that AUTO did not choose, timed the same way on the same inputs
    out["other_y_path"] = other_y_path_time(d, layer, args, dev, flush, stream, steps)
    # the one-kernel path where it applies, timed the same way on the same inputs (opt-in: slower here)
    fp = make_plan(layer, args, fused=wino.FUSED_ON)
    if fp.resolved_variants(*d.shape) & wino.VARIANT_FUSED:
        d.plan = fp
        # (same points, scales and G: the transformed weights are the same bytes)
        fws = torch.empty(fp.workspace_bytes(*d.shape), dtype=torch.uint8, device=dev)
        fms = time_steps(dls, fws, flush, stream, steps, 3)
        favg = sum(fms) / len(fms)
        out["fused_us"] = round(favg * 1e3, 1)
        out["fused_value"] = round(layer.direct_flops / (favg * 1e-3) / 1e12, 1)
        del fws
    del dls, ws
    torch.cuda.empty_cache()
    return out


def other_y_path_time(d, layer, args, dev, flush, stream, steps):
    """Time of one call on the Y path that AUTO did not choose (the swapped GEMM
    only exists on the fp32-Y path, so recompute there runs unswapped)."""
    import torch
    from group_wise_int8_b200 import wino
    names = {wino.YPATH_RECOMPUTE: "recompute", wino.YPATH_Y32: "y32"}
    other = wino.YPATH_Y32 if d.y_path == wino.YPATH_RECOMPUTE else wino.YPATH_RECOMPUTE
    try:
        op = make_plan(layer, args, y_path=other)
    except wino.WinoError:   # e.g. per-tap Y groups exist only on the fp32-Y path
        return None
    if op.resolved_config(*d.shape)[0] != other:
        return None
    saved = d.plan
    d.plan = op   # same points, scales and G: the transformed weights are the same bytes
    ows = torch.empty(op.workspace_bytes(*d.shape), dtype=torch.uint8, device=dev)
    oms = time_steps([d], ows, flush, stream, steps, 3)
    d.plan = saved
    del ows
    return {"y_path": names[other], "us": round(sum(oms) / len(oms) * 1e3, 1)}


def y_path_check(layers, args, dev, flush, stream, steps):
    """Per distinct shape of the workload: one call on the chosen Y path and one on the other, each
    with the L2 flushed before it, so the AUTO choice can be checked against measurement."""
    import torch
    rows, seen = [], set()
    for layer in layers:
        key = shape_key(layer)
        if key in seen:
            continue
        seen.add(key)
        d = prepare([layer], args, dev)[0]
        ws = torch.empty(d.plan.workspace_bytes(*d.shape), dtype=torch.uint8, device=dev)
        ms = time_steps([d], ws, flush, stream, steps, 3)
        chosen = {1: "recompute", 2: "y32"}.get(d.y_path)
        row = {"layer": key, "chosen": chosen, "chosen_us": round(sum(ms) / len(ms) * 1e3, 1),
               "other": other_y_path_time(d, layer, args, dev, flush, stream, steps)}
        if row["other"] is not None:
            row["chosen_is_faster"] = row["chosen_us"] <= row["other"]["us"]
        rows.append(row)
        del d, ws
        torch.cuda.empty_cache()
    return rows


# ------------------------------------------------------------- CPU oracle timing
_SAMPLE_CACHE = {}


def oracle_samples(layers, rows: int, images: int, int8_transforms: bool = False, max_cout: int = 256):
    """Per distinct layer shape: the first `images` images cropped to `rows` tile rows, and the
    first min(Cout, max_cout) output channels, with the number of convs of that shape in the
    workload.  The seeded streams give the first images and the first output channels of a
    layer as a prefix, so these are exactly the workload's own values."""
    import dataclasses
    import oracle
    groups = collections.OrderedDict()
    for l in layers:
        groups.setdefault((l.m, l.Cin, l.Cout, l.H, l.W, l.N, l.group), []).append(l)
    out = []
    for ls in groups.values():
        layer = ls[0]
        cs = min(layer.Cout, max_cout)
        ni = min(images, layer.N)
        key = (layer, ni, cs, int8_transforms)
        if key not in _SAMPLE_CACHE:
            x_f32, _ = synth.make_input(dataclasses.replace(layer, N=ni))
            w = synth.make_weights(dataclasses.replace(layer, Cout=cs))
            sb, sg = synth.make_scales(layer)
            plan = oracle.Plan(layer.m, layer.points, sb, sg, int8_transforms=int8_transforms)
            Uq, sU, _ = oracle.weight_transform(plan, w, layer.group)
            _SAMPLE_CACHE[key] = (plan, x_f32, Uq, sU)
        plan, x_f32, Uq, sU = _SAMPLE_CACHE[key]
        H = min(layer.H, rows * layer.m)
        xs = np.ascontiguousarray(x_f32[:, :H])
        flops = 2.0 * ni * H * layer.W * layer.Cin * cs * 9
        out.append((len(ls), layer, plan, xs, Uq, sU, flops))
    return out


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


def time_samples(samples, reps, per_tap, x_int8):
    """Workload-weighted CPU throughput: each distinct shape's sample counts as often as the
    shape occurs in the workload."""
    t_tot = f_tot = 0.0
    for count, layer, plan, xs, Uq, sU, flops in samples:
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_step(plan, xs, Uq, sU, layer.group, per_tap, x_int8)
        t_tot += count * (time.perf_counter() - t0) / reps
        f_tot += count * flops
    return f_tot / t_tot, t_tot


def cpu_baseline(label, layers, budget_s: float = 12.0, threads: int = 0, per_tap: bool = False,
                 x_int8: bool = False, int8_transforms: bool = False):
    import oracle
    used = oracle.set_threads(threads)
    rows, images = 1, 1
    samples = oracle_samples(layers, rows, images, int8_transforms)
    _, dt = time_samples(samples, 1, per_tap, x_int8)
    TH = max(-(-l.H // l.m) for l in layers)
    Nmax = max(l.N for l in layers)
    while dt * 2 < budget_s / 2 and (rows < TH or images < Nmax):
        if rows < TH:
            rows = min(TH, rows * 2)
        else:
            images = min(Nmax, images * 2)
        samples = oracle_samples(layers, rows, images, int8_transforms)
        _, dt = time_samples(samples, 1, per_tap, x_int8)
    reps = max(1, int(budget_s / 2 / max(dt, 1e-3)))
    rate, _ = time_samples(samples, reps, per_tap, x_int8)
    oracle.set_threads(0)
    return {"value": rate / 1e12, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": "per distinct conv shape of %s: %d image(s) x %d tile row(s) x the first min(Cout, 256) "
                      "output channels, weighted by the shape's count; input transform, Hadamard, Y requant, "
                      "output transform (weights pre-transformed); %d rep(s)" % (label, images, rows, reps)}


def run_reference(args, label, layers):
    per_tap = args.y_groups == "tap"
    x_int8 = args.x_int8
    import oracle
    threads = oracle.set_threads(0)
    TH = max(-(-l.H // l.m) for l in layers)
    budget = 150.0 / max(1, args.steps + args.warmup)   # seconds per step: whole run within a few minutes
    rows = 1
    samples = oracle_samples(layers, rows, 1, args.int8_transforms)
    _, dt = time_samples(samples, 1, per_tap, x_int8)
    while dt * 2 <= budget and rows < TH:
        rows = min(TH, rows * 2)
        samples = oracle_samples(layers, rows, 1, args.int8_transforms)
        _, dt = time_samples(samples, 1, per_tap, x_int8)
    for _ in range(args.warmup):
        time_samples(samples, 1, per_tap, x_int8)
    ms = []
    for _ in range(args.steps):
        rate, dt = time_samples(samples, 1, per_tap, x_int8)
        ms.append(dt * 1e3)
    flops = sum(c * f for c, _, _, _, _, _, f in samples)
    value = args.steps * flops / (sum(ms) * 1e-3) / 1e12
    sample = ("per distinct conv shape of %s: 1 image x %d tile row(s) x the first min(Cout, 256) output "
              "channels, weighted by the shape's count, per step" % (label, rows))
    return {"value": value, "ms_per_step": sum(ms) / len(ms),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample}}


def main():
    args = parse()
    label, layers = pick_layers(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    l0 = layers[0]
    config = {"workload": label, "model": l0.workload, "convs_per_step": len(layers),
              "global_batch": l0.N * world, "seq_len": None, "m": l0.m, "group": l0.group,
              "parallelism": "dp%d" % world,
              "l2": ("flushed once before every step (256 MiB write), convs back to back" if len(layers) > 1
                     else "flushed before every timed step (256 MiB write)"),
              "output": "bf16 NHWC", "y_groups": args.y_groups, "x_int8": args.x_int8,
              "int8_transforms": args.int8_transforms}
    if len(layers) == 1:
        config.update(H=l0.H, W=l0.W, Cin=l0.Cin, Cout=l0.Cout, N=l0.N)
    line = {"metric": METRIC, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8 (fp32 transforms)",
            "data": "synthetic (seeded)", "config": config}

    if args.impl == "reference":
        if rank != 0:
            return
        r = run_reference(args, label, layers)
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
        r = run_ours(args, label, layers, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        kw = dict(per_tap=args.y_groups == "tap", x_int8=args.x_int8, int8_transforms=args.int8_transforms)
        cpu = cpu_baseline(label, layers, 12.0, 0, **kw)
        cpu["single_thread"] = cpu_baseline(label, layers, 6.0, 1, **kw)
    line.update(value=r["value"], ms_per_step=r["ms_per_step"], e2e=r["e2e"], roofline=r["roofline"],
                cpu_baseline=cpu, clocks=r["clocks"], gpu_launches=r["gpu_launches"], impl="ours",
                kernels=r["kernels"], int8_peak=r["int8_peak"])
    for k in ("cudnn_bf16", "y_path_check", "beside", "layers"):
        if k in r:
            line[k] = r[k]
    print(json.dumps(line))


if __name__ == "__main__":
    main()
