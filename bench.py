#!/usr/bin/env python
"""Throughput benchmark of the DCNv4 forward spatial aggregation on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
    torchrun --nproc-per-node N bench.py --gpus N ...     (one rank per GPU)

(--gpus N > 1 outside torchrun relaunches the same command under torch.distributed.run
as N ranks of one node.)

A step is one dcnv4_forward call over one batch of a named workload (seeded
synthetic inputs in the workload's shape and value distributions). Without
--workload the run prints one JSON line per named workload, in the order
stage1_f32, stage1_f16, stage3_f16, sd_latent_f16, highres_bf16: the last
line, the high-resolution bf16 batch (the largest workload by sampling points,
9.29 M per step), is the headline. tiny_f32 is a parity case, not a line.
With N GPUs every rank processes its own batch of the workload (weak
scaling, no collective on the data path).

Timing: W untimed warm-up steps, a ~1 s untimed soak (clocks settle and are
sampled), then exactly K steps between CUDA events on the launching stream,
bracketed by a barrier and a device synchronise; the time is the max over
ranks. The steps rotate over several resident copies of the inputs whose total
exceeds the L2 cache, so no step starts with its inputs in L2.

End to end (`e2e`): the same metric through dcnv4_forward_host, from pinned
host buffers to a host result, the host-to-device and device-to-host copies
inside the timed region (the library overlaps them with the kernels over
chunks of images, or bands of output rows for a batch of a few images);
the line states the bytes copied each way per step.

--impl reference times the fp64 CPU oracle (the reference arm of this
repository: there is no other implementation to install) on the host cores,
for the same workloads, metric and unit.

Secondary lines (not the headline): --pass backward times dcnv4_backward on
the stage-1 fp16 batch (or --workload); --pass predictor times
dcnv4_predictor (the tcgen05 projection that produces the workload's
offset_mask records); --variant softmax|remove_center|center_scale|all times
dcnv4_forward_ex with those variant flags.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DCNv4 fwd sampling points/s (G/s); achieved HBM GB/s as % of B200 peak"
METRIC_BWD = "DCNv4 bwd sampling points/s (G/s); achieved HBM GB/s as % of B200 peak"
METRIC_PRED = "DCNv4 offset/mask predictor records/s (G pixel-group records/s); achieved HBM GB/s as % of B200 peak"
UNIT = "Gpoints/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="one named workload (default: every forward line; the "
                                                     "stage-1 fp16 batch for the other passes)")
    ap.add_argument("--soak-s", type=float, default=1.0)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward", "predictor"], default="forward",
                    help="forward (the headline), the backward of the same workload, or the offset/mask "
                         "predictor's projection that produces its records")
    ap.add_argument("--variant", choices=["none", "softmax", "remove_center", "center_scale", "all"],
                    default="none", help="forward variant flags (DCNv3 softmax, centre point removed, "
                                         "centre feature scaling, or all three)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the source files that define each profiled kernel and its launch configuration
KERNEL_SOURCES = {
    "forward": ("dcnv4_kernels.cuh", "dcnv4_async.cuh", "dcnv4_window.cuh", "dcnv4_host_common.inl",
                "dcnv4_launch_forward.inl"),
    "backward": ("dcnv4_kernels.cuh", "dcnv4_backward.cuh", "dcnv4_host_common.inl", "dcnv4_launch_backward.inl"),
    "predictor": ("dcnv4_kernels.cuh", "dcnv4_async.cuh", "dcnv4_predictor.cuh", "dcnv4_host_common.inl",
                  "dcnv4_launch_predictor.inl"),
}


SHAPE_ORIGIN = {
    "tiny": "tiny case",
    "stage1": "FlashInternImage-T stage-1 shaped",
    "stage3": "FlashInternImage-T stage-3 shaped",
    "sd_latent": "SD-1.5 latent U-Net block shaped",
    "highres": "high-resolution, dilated",
}


def shape_origin(w) -> str:
    for key, text in SHAPE_ORIGIN.items():
        if w.name.startswith(key):
            return text
    return "synthetic"


def _dist(d) -> str:
    kind, a, b = d
    return f"N({a:g},{b:g}^2)" if kind == "normal" else f"U[{a:g},{b:g}]"


def input_recipe(w) -> str:
    return f"seeded synthetic (seed {w.seed}): x~N(0,1), offsets~{_dist(w.offsets)}, masks~{_dist(w.masks)}"


def workload_text(w, which: str = "forward", variant: str = "none") -> str:
    """config.workload of a line: the same text on both arms for the same pass and variant."""
    P = w.K * w.K - (1 if VARIANT_FLAGS.get(variant, 0) & 2 else 0)
    if which == "predictor":
        M, NO = w.N * w.Hout * w.Wout, 3 * w.G * w.K * w.K
        return (f"{w.name} predictor: y [{M}, {w.C}] x W [{NO}, {w.C}] + bias -> offset_mask "
                f"[{M}, {w.G}, {3 * w.K * w.K}] (the records of the {w.name} aggregation)")
    if which == "backward":
        return (f"{w.name} backward, variant {variant}: N={w.N} per GPU, H=W={w.H}, C={w.C}, "
                f"G={w.G} (C/G={w.Cg}), K={w.K}, {P} points per unit, stride={w.stride}, pad={w.pad}, "
                f"dilation={w.dilation}; fp32 gradients")
    if variant != "none":
        return (f"{w.name} forward, variant {variant}: N={w.N} per GPU, H=W={w.H}, C={w.C}, "
                f"G={w.G}, K={w.K}, {P} points per unit")
    return (f"{w.name}: {shape_origin(w)} DCNv4 forward, N={w.N} per GPU, H=W={w.H}, C={w.C}, G={w.G} "
            f"(C/G={w.Cg}), K={w.K}, stride={w.stride}, pad={w.pad}, dilation={w.dilation}, "
            f"offset_scale={w.offset_scale}")


def kernel_sources_sha(kind: str = "forward") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "deformable_convolution_sparse_b200", "csrc")
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()


def profiled_traffic(workload: str, kind: str = "forward"):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel sources."""
    sha = kernel_sources_sha(kind)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("workload") == workload and fields.get("pass", "forward") == kind \
                and fields.get("kernel_sources_sha256") == sha and "dram_bytes_per_launch" in fields:
            return int(float(fields["dram_bytes_per_launch"])), os.path.relpath(path, ROOT)
    return None, None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is under load."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str):
        self.uuid = gpu_uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def host_cpu(used: int = 1) -> str:
    """Model name of the host CPU (from /proc/cpuinfo) and the cores this process may run on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{model}; {host_cores()} cores available, {used} used"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def cpu_baseline(w, x, om):
    """The fp64 oracle, as it stands, on the whole batch: on every host core this process may use
    (OpenMP over output rows; the same per-element code, so the same bits) and on one thread."""
    import oracle
    xd, omd = x.double().numpy(), om.double().numpy()
    cores = host_cores()
    oracle.dcnv4_forward(xd, omd, **w.kwargs(), n_begin=0, n_end=1, threads=cores)  # load + warm
    t0 = time.perf_counter()
    oracle.dcnv4_forward(xd, omd, **w.kwargs(), threads=cores)
    dt = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.dcnv4_forward(xd, omd, **w.kwargs())
    dt1 = time.perf_counter() - t0
    return {"value": w.points / dt / 1e9, "unit": UNIT, "cores": cores, "cpu": host_cpu(cores), "kind": "oracle",
            "seconds": dt, "sample": f"the whole {w.name} batch ({w.N} images, {w.points} points), fp64 C oracle, "
                                    f"output rows shared out among {cores} OpenMP threads",
            "single_thread": {"value": w.points / dt1 / 1e9, "unit": UNIT, "cores": 1, "seconds": dt1}}


def cpu_baseline_backward(w, x, om, go):
    """The fp64 oracle's backward, as it stands, on the whole batch (single thread)."""
    import oracle
    xd, omd, god = x.double().numpy(), om.double().numpy(), go.double().numpy()
    oracle.dcnv4_backward(xd[:1], omd[:1], god[:1], **w.kwargs())  # load + warm
    t0 = time.perf_counter()
    oracle.dcnv4_backward(xd, omd, god, **w.kwargs())
    dt = time.perf_counter() - t0
    return {"value": w.points / dt / 1e9, "unit": UNIT, "cores": 1, "cpu": host_cpu(), "kind": "oracle",
            "seconds": dt, "sample": f"the whole {w.name} batch ({w.N} images, {w.points} points), "
                                    "fp64 C oracle backward, one thread"}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores, for the same pass, variant,
    workload, metric and unit as this implementation's line; each step is a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from deformable_convolution_sparse_b200.workloads import WORKLOADS
    for name in workloads_to_run(args):
        reference_line(args, WORKLOADS[name])


def reference_line(args, w):
    import torch
    from deformable_convolution_sparse_b200.workloads import make_center_logit, make_inputs, workload_grad_out
    import oracle
    flags = VARIANT_FLAGS.get(args.variant, 0)
    P = w.K * w.K - (1 if flags & 2 else 0)
    kw = w.kwargs()
    # the plain forward runs on every host core (OpenMP over output rows, the same bits as one thread);
    # the other passes time the oracle's single-thread code
    cores = host_cores() if (args.which == "forward" and not flags) else 1
    vkw = dict(softmax=bool(flags & 1), remove_center=bool(flags & 2))
    n_s = max(1, min(w.N, 8))  # images per step: a bounded sample (~0.1 s of CPU work each)
    if args.which == "predictor":
        M, NO = w.N * w.Hout * w.Wout, 3 * w.G * w.K * w.K
        rows = n_s * w.Hout * w.Wout
        # the same draws as this implementation's predictor line (rank 0)
        td = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
        gen = torch.Generator().manual_seed(w.seed)
        y = torch.randn(M, w.C, generator=gen).to(td).double().numpy()
        wt = (torch.randn(NO, w.C, generator=gen) * w.C ** -0.5).to(td).double().numpy()
        b = torch.randn(NO, generator=gen).double().numpy()
        metric, unit, per_step = METRIC_PRED, "Grecords/s", rows * w.G

        def one(i):
            r0 = (i * rows) % (M - rows + 1)
            oracle.dcnv4_predictor(y[r0:r0 + rows], wt, b, G=w.G, P=w.K * w.K)
    else:
        x, om = make_inputs(w.N, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, w.dtype, w.offsets, w.masks,
                            seed=w.seed, points=P)
        xd, omd = x.double().numpy(), om.double().numpy()
        zd = make_center_logit(w.N, w.Hout, w.Wout, w.G, w.dtype, seed=w.seed).double().numpy()
        per_step = w.N * w.Hout * w.Wout * w.G * P // w.N * n_s
        unit = UNIT
        if args.which == "backward":
            metric = METRIC_BWD
            god = workload_grad_out(w).double().numpy()

            def one(i):
                b0 = (i * n_s) % (w.N - n_s + 1)
                sl = slice(b0, b0 + n_s)
                if flags:
                    oracle.dcnv4_backward_variants(xd[sl], omd[sl], god[sl], **kw, **vkw,
                                                   center_logit=zd[sl] if flags & 4 else None)
                else:
                    oracle.dcnv4_backward(xd[sl], omd[sl], god[sl], **kw)
        else:
            metric = METRIC

            def one(i):
                b0 = (i * n_s) % (w.N - n_s + 1)
                sl = slice(b0, b0 + n_s)
                if flags:
                    oracle.dcnv4_forward_variants(xd[sl], omd[sl], **kw, **vkw,
                                                  center_logit=zd[sl] if flags & 4 else None)
                else:
                    oracle.dcnv4_forward(xd, omd, **kw, n_begin=b0, n_end=b0 + n_s, threads=cores)
    for _ in range(args.warmup):
        one(0)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt / 1e9
    what = f"{args.which}" + (f", variant {args.variant}" if args.variant != "none" else "")
    sample = (f"{n_s * w.Hout * w.Wout} of {w.N * w.Hout * w.Wout} pixels ({n_s} images) per step"
              if args.which == "predictor" else f"{n_s} of {w.N} images per step")
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_text(w, args.which, args.variant), "storage_dtype": w.dtype,
                   "accumulate": "f64 (oracle)", "sample_per_step": sample},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "cpu": host_cpu(cores), "kind": "oracle",
                         "sample": f"{sample}, fp64 C oracle {what}, "
                                   + (f"{cores} OpenMP threads" if cores > 1 else "one thread")},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    # the same pass/variant keys as this implementation's line for that row
    if args.which != "forward":
        line["pass"] = args.which
    if args.which == "backward" or (args.which == "forward" and args.variant != "none"):
        line["variant"] = args.variant
    print(json.dumps(line), flush=True)


# the forward lines of the default run, in print order: the last one (the largest
# workload by sampling points) is the headline
FORWARD_LINES = ("stage1_f32", "stage1_f16", "stage3_f16", "sd_latent_f16", "highres_bf16")

# the arithmetic each storage type's forward computes in (the line's "dtype")
ARITH = {"f32": "f32", "bf16": "f32",
         "f16": "f32 accumulate, fp16-rounded corner weights (fp16 x fp16 products exact in f32)"}


def workloads_to_run(args):
    """--workload names one line; without it the forward prints every named workload's line (the
    tiny parity case excepted), the largest last, and the other passes use the stage-1 fp16 batch."""
    if args.workload:
        return [args.workload]
    if args.which == "forward" and args.variant == "none":
        return list(FORWARD_LINES)
    return [BENCH_WORKLOAD]


def time_steps(step, launches, args, dev, stream, barrier, max_over_ranks):
    """W warm-up steps, a soak of --soak-s seconds with the clock sampler running, then exactly
    K steps between CUDA events on `stream`, bracketed by barrier + synchronise. Returns
    (max over ranks of the timed milliseconds, the stopped sampler, launches in the timed region)."""
    import torch
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    t_end = time.perf_counter() + args.soak_s
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches[0] = 0
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    # a kernel that gave up on a bounded wait sets a bit of the device status word and returns
    # early: such a run measured unfinished work and is not reported
    # (every rank reads its own word; all of them stop if any rank's is set)
    import deformable_convolution_sparse_b200 as dcn
    status = dcn.device_status(clear=False)
    barrier()
    sampler.stop()
    if max_over_ranks(float(status)) != 0.0:
        raise SystemExit(f"device status word 0x{status:x} after the timed steps (max over ranks non-zero): "
                         "a kernel gave up a bounded wait")
    return max_over_ranks(ev0.elapsed_time(ev1)), sampler, launches[0]


def run_backward(args, w, dev, world, rank, barrier, max_over_ranks):
    """The backward of the same workload: one dcnv4_backward call (a clear of grad_x plus one
    kernel) per step, fp32 gradients, inputs rotating over resident sets larger than L2."""
    import torch
    import deformable_convolution_sparse_b200 as dcn
    from deformable_convolution_sparse_b200.workloads import workload_grad_out, workload_inputs

    from deformable_convolution_sparse_b200.workloads import make_center_logit, make_inputs

    flags = VARIANT_FLAGS.get(args.variant, 0)
    P = w.K * w.K - (1 if flags & 2 else 0)
    wr = w.with_(seed=w.seed + 1000 * rank)
    x, om = make_inputs(w.N, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, w.dtype, w.offsets, w.masks, seed=wr.seed,
                        points=P)
    go = workload_grad_out(wr)
    z = make_center_logit(w.N, w.Hout, w.Wout, w.G, w.dtype, seed=wr.seed)
    lib = dcn.load_library()
    dtype_code = dcn.binding.TORCH_DTYPE[x.dtype]
    e = x.element_size()
    nx, nom, nout, nz = x.numel(), om.numel(), go.numel(), (z.numel() if flags & 4 else 0)
    # algorithmic bytes: x, offset_mask, grad_out (and the gate logits) read once; grad_x, grad_offset_mask
    # (and the gate gradient) written once in fp32
    foot = (nx + nom + nout + nz) * e + (nx + nom + nz) * 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(3, math.ceil(3 * l2 / foot))
    sets = [(x.to(dev), om.to(dev), go.to(dev), torch.empty(x.shape, dtype=torch.float32, device=dev),
             torch.empty(om.shape, dtype=torch.float32, device=dev)) for _ in range(copies)]
    zd = z.to(dev)
    gzd = torch.empty(z.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    launches = [0]

    def call(xd, omd, god, gxd, gomd):
        if flags:
            rc = lib.dcnv4_backward_ex(xd.data_ptr(), omd.data_ptr(), zd.data_ptr(), god.data_ptr(), gxd.data_ptr(),
                                       gomd.data_ptr(), gzd.data_ptr(), w.N, w.H, w.W, w.C, w.G, w.K, w.stride,
                                       w.pad, w.dilation, w.offset_scale, dtype_code, flags, sh)
        else:
            rc = lib.dcnv4_backward(xd.data_ptr(), omd.data_ptr(), god.data_ptr(), gxd.data_ptr(), gomd.data_ptr(),
                                    w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation, w.offset_scale,
                                    dtype_code, sh)
        if rc != 0:
            raise dcn.DCNv4Error(rc, "dcnv4_backward_ex" if flags else "dcnv4_backward")

    def step(i):
        call(*sets[i % copies])
        launches[0] += 1  # one kernel (the clear of grad_x is a cudaMemsetAsync)

    ms, sampler, timed_launches = time_steps(step, launches, args, dev, stream, barrier, max_over_ranks)
    ms_step = ms / args.steps
    points = w.N * w.Hout * w.Wout * w.G * P
    value = points * world * args.steps / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = foot / (ms_step / 1e3) / 1e9
    traffic, traffic_src = profiled_traffic(w.name, "backward")

    # end to end: pinned host inputs copied in, backward, both gradients copied back, one stream
    xh, omh, goh = x.pin_memory(), om.pin_memory(), go.pin_memory()
    gxh = torch.empty(x.shape, dtype=torch.float32).pin_memory()
    gomh = torch.empty(om.shape, dtype=torch.float32).pin_memory()
    xd, omd, god, gxd, gomd = sets[0]

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        omd.copy_(omh, non_blocking=True)
        god.copy_(goh, non_blocking=True)
        call(xd, omd, god, gxd, gomd)
        gxh.copy_(gxd, non_blocking=True)
        gomh.copy_(gomd, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = points * world * args.e2e_steps / (e2e_ms / 1e3) / 1e9
    if not torch.equal(gomh, gomd.cpu()):
        raise SystemExit("end-to-end gradient record differs from the device-resident one")

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not flags:
        base = cpu_baseline_backward(w, x, om, go)
    if rank == 0:
        line = {
            "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "pass": "backward", "variant": args.variant,
            "config": {
                "workload": workload_text(w, "backward", args.variant),
                "storage_dtype": w.dtype, "accumulate": "f32", "global_batch": w.N * world,
                "points_per_step_per_gpu": points, "parallelism": f"dp{world} (independent batches)",
                "l2": f"steps rotate over {copies} resident sets, {copies * foot / 1e6:.0f} MB in total vs "
                      f"{l2 / 1e6:.0f} MB L2",
                "inputs": input_recipe(w) + f", grad_out~N(0,1) (seed {1000 + w.seed})",
            },
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel": "dcnv4 backward (clear of grad_x + one kernel per step)",
                         "algorithmic_bytes_per_launch": foot, "traffic": traffic, "traffic_source": traffic_src},
            "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms / args.e2e_steps,
                    "steps": args.e2e_steps, "h2d_bytes_per_step": (nx + nom + nout) * e,
                    "d2h_bytes_per_step": (nx + nom) * 4,
                    "path": "pinned host tensors copied in, dcnv4_backward, gradients copied out, one stream"},
            "gpu_launches": timed_launches,
            "clocks": sampler.summary(),
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)


VARIANT_FLAGS = {"softmax": 1, "remove_center": 2, "center_scale": 4, "all": 7}


def run_variant(args, w, dev, world, rank, barrier, max_over_ranks):
    """The forward with variant flags (dcnv4_forward_ex), inputs rotating over resident sets larger than L2."""
    import torch
    import deformable_convolution_sparse_b200 as dcn
    from deformable_convolution_sparse_b200.workloads import make_center_logit, make_inputs

    flags = VARIANT_FLAGS[args.variant]
    P = w.K * w.K - (1 if flags & 2 else 0)
    wr = w.with_(seed=w.seed + 1000 * rank)
    x, om = make_inputs(w.N, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, w.dtype, w.offsets, w.masks, seed=wr.seed,
                        points=P)
    z = make_center_logit(w.N, w.Hout, w.Wout, w.G, w.dtype, seed=wr.seed)
    lib = dcn.load_library()
    dtype_code = dcn.binding.TORCH_DTYPE[x.dtype]
    e = x.element_size()
    nout = w.N * w.Hout * w.Wout * w.C
    # algorithmic bytes: x, offset_mask (and the gate logits) read once, out written once
    foot = (x.numel() + om.numel() + nout + (z.numel() if flags & 4 else 0)) * e
    points = w.N * w.Hout * w.Wout * w.G * P
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(3, math.ceil(3 * l2 / foot))
    sets = [(x.to(dev), om.to(dev), z.to(dev), torch.empty((w.N, w.Hout, w.Wout, w.C), dtype=x.dtype, device=dev))
            for _ in range(copies)]
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    launches = [0]

    def call(xd, omd, zd, od):
        rc = lib.dcnv4_forward_ex(xd.data_ptr(), omd.data_ptr(), zd.data_ptr(), od.data_ptr(), w.N, w.H, w.W, w.C,
                                  w.G, w.K, w.stride, w.pad, w.dilation, w.offset_scale, dtype_code, flags, sh)
        if rc != 0:
            raise dcn.DCNv4Error(rc, "dcnv4_forward_ex")

    def step(i):
        call(*sets[i % copies])
        launches[0] += 1

    ms, sampler, timed_launches = time_steps(step, launches, args, dev, stream, barrier, max_over_ranks)
    ms_step = ms / args.steps
    value = points * world * args.steps / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = foot / (ms_step / 1e3) / 1e9

    xh, omh, zh = x.pin_memory(), om.pin_memory(), z.pin_memory()
    oh = torch.empty((w.N, w.Hout, w.Wout, w.C), dtype=x.dtype).pin_memory()
    xd, omd, zd, od = sets[0]

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        omd.copy_(omh, non_blocking=True)
        if flags & 4:
            zd.copy_(zh, non_blocking=True)
        call(xd, omd, zd, od)
        oh.copy_(od, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = points * world * args.e2e_steps / (e2e_ms / 1e3) / 1e9
    if not torch.equal(oh, od.cpu()):
        raise SystemExit("end-to-end result differs from the device-resident result")

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        xd64, omd64, z64 = x[:1].double().numpy(), om[:1].double().numpy(), z[:1].double().numpy()
        kw = dict(G=w.G, K=w.K, stride=w.stride, pad=w.pad, dilation=w.dilation, offset_scale=w.offset_scale,
                  softmax=bool(flags & 1), remove_center=bool(flags & 2), center_logit=z64 if flags & 4 else None)
        oracle.dcnv4_forward_variants(xd64, omd64, **kw)
        n_s = min(w.N, 8)
        kw["center_logit"] = z[:n_s].double().numpy() if flags & 4 else None
        xs64, oms64 = x[:n_s].double().numpy(), om[:n_s].double().numpy()
        t0 = time.perf_counter()
        oracle.dcnv4_forward_variants(xs64, oms64, **kw)
        dt = time.perf_counter() - t0
        base = {"value": points // w.N * n_s / dt / 1e9, "unit": UNIT, "cores": 1, "cpu": host_cpu(), "kind": "oracle",
                "seconds": dt, "sample": f"{n_s} of {w.N} images, fp64 C oracle ({args.variant}), one thread"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": ARITH[w.dtype], "data": "synthetic", "variant": args.variant,
            "config": {
                "workload": workload_text(w, "forward", args.variant),
                "storage_dtype": w.dtype, "accumulate": "f32", "global_batch": w.N * world,
                "points_per_step_per_gpu": points, "parallelism": f"dp{world} (independent batches)",
                "l2": f"steps rotate over {copies} resident sets, {copies * foot / 1e6:.0f} MB in total vs "
                      f"{l2 / 1e6:.0f} MB L2",
                "inputs": input_recipe(w) + "; gate logits ~N(0,1.5^2)",
            },
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel": "dcnv4 forward with variant flags (one launch per step)",
                         "algorithmic_bytes_per_launch": foot, "traffic": None},
            "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms / args.e2e_steps,
                    "steps": args.e2e_steps,
                    "h2d_bytes_per_step": (x.numel() + om.numel() + (z.numel() if flags & 4 else 0)) * e,
                    "d2h_bytes_per_step": nout * e,
                    "path": "pinned host tensors copied in, dcnv4_forward_ex, result copied out, one stream"},
            "gpu_launches": timed_launches,
            "clocks": sampler.summary(),
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)


def run_predictor(args, w, dev, world, rank, barrier, max_over_ranks):
    """The offset/mask predictor's 1x1 projection + packing (dcnv4_predictor) for the workload's records:
    y [N*Hout*Wout, C] -> offset_mask [N*Hout*Wout, G, 3*K*K], fp16/bf16 on the tensor cores."""
    import torch
    import deformable_convolution_sparse_b200 as dcn

    M, P = w.N * w.Hout * w.Wout, w.K * w.K
    NO = 3 * w.G * P
    gen = torch.Generator().manual_seed(w.seed + 1000 * rank)
    td = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
    y = torch.randn(M, w.C, generator=gen).to(td)
    wt = (torch.randn(NO, w.C, generator=gen) * w.C ** -0.5).to(td)
    b = torch.randn(NO, generator=gen)
    lib = dcn.load_library()
    dtype_code = dcn.binding.TORCH_DTYPE[td]
    e = y.element_size()
    foot = (y.numel() + wt.numel() + M * NO) * e + b.numel() * 4
    flops = 2.0 * M * NO * w.C
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(3, math.ceil(3 * l2 / foot))
    sets = [(y.to(dev), torch.empty(M, w.G, 3 * P, dtype=td, device=dev)) for _ in range(copies)]
    wd, bd = wt.to(dev), b.to(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    launches = [0]

    def call(yd, od):
        rc = lib.dcnv4_predictor(yd.data_ptr(), wd.data_ptr(), bd.data_ptr(), od.data_ptr(), M, w.C, w.G, w.K, 0,
                                 dtype_code, sh)
        if rc != 0:
            raise dcn.DCNv4Error(rc, "dcnv4_predictor")

    def step(i):
        call(*sets[i % copies])
        launches[0] += 1

    ms, sampler, timed_launches = time_steps(step, launches, args, dev, stream, barrier, max_over_ranks)
    ms_step = ms / args.steps
    units = M * w.G
    value = units * world * args.steps / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = foot / (ms_step / 1e3) / 1e9
    traffic, traffic_src = profiled_traffic(w.name, "predictor")

    yh = y.pin_memory()
    oh = torch.empty(M, w.G, 3 * P, dtype=td).pin_memory()
    yd0, od0 = sets[0]

    def e2e_step():
        yd0.copy_(yh, non_blocking=True)
        call(yd0, od0)
        oh.copy_(od0, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    if not torch.equal(oh, od0.cpu()):
        raise SystemExit("end-to-end records differ from the device-resident ones")

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        n_s = min(M, 8 * w.Hout * w.Wout)
        ys, ws, bs = y[:n_s].double().numpy(), wt.double().numpy(), b.double().numpy()
        oracle.dcnv4_predictor(ys[:16], ws, bs, G=w.G, P=P)
        t0 = time.perf_counter()
        oracle.dcnv4_predictor(ys, ws, bs, G=w.G, P=P)
        dt = time.perf_counter() - t0
        base = {"value": n_s * w.G / dt / 1e9, "unit": "Grecords/s", "cores": 1, "cpu": host_cpu(), "kind": "oracle", "seconds": dt,
                "sample": f"{n_s} of {M} pixels (8 images), fp64 C oracle predictor, one thread"}
    if rank == 0:
        line = {
            "metric": METRIC_PRED, "value": value, "unit": "Grecords/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "pass": "predictor",
            "config": {
                "workload": workload_text(w, "predictor"),
                "storage_dtype": w.dtype, "accumulate": "f32 (tensor memory)", "global_batch": w.N * world,
                "parallelism": f"dp{world} (independent batches)",
                "l2": f"steps rotate over {copies} resident sets, {copies * foot / 1e6:.0f} MB in total vs "
                      f"{l2 / 1e6:.0f} MB L2",
                "inputs": "seeded synthetic: y~N(0,1), W~N(0,1/C), bias~N(0,1)",
                "tensor_tflops": flops / (ms_step / 1e3) / 1e12,
            },
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel": "dcnv4 predictor (tcgen05 GEMM + packing epilogue, one launch per step)",
                         "algorithmic_bytes_per_launch": foot, "flops_per_launch": flops,
                         "traffic": traffic, "traffic_source": traffic_src},
            "e2e": {"value": units * world * args.e2e_steps / (e2e_ms / 1e3) / 1e9, "unit": "Grecords/s",
                    "ms_per_step": e2e_ms / args.e2e_steps, "steps": args.e2e_steps,
                    "h2d_bytes_per_step": y.numel() * e, "d2h_bytes_per_step": M * NO * e,
                    "path": "pinned y copied in, dcnv4_predictor, records copied out, one stream"},
            "gpu_launches": timed_launches,
            "clocks": sampler.summary(),
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)


def relaunch_under_torchrun(n: int) -> int:
    """`python bench.py --gpus N` (N > 1) outside torchrun: run this same command line as N ranks of
    one node (rendezvous on 127.0.0.1, a free port) and return their exit status."""
    import socket
    import subprocess
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args.gpus))

    import torch
    import torch.distributed as dist

    import deformable_convolution_sparse_b200 as dcn
    from deformable_convolution_sparse_b200.workloads import BENCH_WORKLOAD, WORKLOADS, workload_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    if args.which != "forward" or args.variant != "none":
        w = WORKLOADS[args.workload or BENCH_WORKLOAD]
        if args.which == "backward":
            run_backward(args, w, dev, world, rank, barrier, max_over_ranks)
        elif args.which == "predictor":
            run_predictor(args, w, dev, world, rank, barrier, max_over_ranks)
        else:
            run_variant(args, w, dev, world, rank, barrier, max_over_ranks)
        if world > 1:
            dist.destroy_process_group()
        return
    for name in workloads_to_run(args):
        run_forward(args, WORKLOADS[name], dev, world, rank, barrier, max_over_ranks)
    if world > 1:
        dist.destroy_process_group()


def run_forward(args, w, dev, world, rank, barrier, max_over_ranks):
    """One forward line: dcnv4_forward over the workload's batch per step (per GPU), inputs rotating over
    resident sets larger than L2; the end-to-end path through dcnv4_forward_host; the CPU oracle."""
    import torch
    import deformable_convolution_sparse_b200 as dcn
    from deformable_convolution_sparse_b200.workloads import workload_inputs

    # weak scaling: rank r owns images [64 r, 64 (r+1)) of the global batch, drawn from seed + r
    wr = w.with_(seed=w.seed + 1000 * rank)
    x, om = workload_inputs(wr)
    lib = dcn.load_library()
    dtype_code = dcn.binding.TORCH_DTYPE[x.dtype]

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    foot = w.algorithmic_bytes()
    copies = max(3, math.ceil(3 * l2 / foot))
    xs = [x.to(dev) for _ in range(copies)]
    oms = [om.to(dev) for _ in range(copies)]
    outs = [torch.empty((w.N, w.Hout, w.Wout, w.C), dtype=x.dtype, device=dev) for _ in range(copies)]
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    launches = [0]

    def step(i):
        j = i % copies
        rc = lib.dcnv4_forward(xs[j].data_ptr(), oms[j].data_ptr(), outs[j].data_ptr(), w.N, w.H, w.W, w.C, w.G,
                               w.K, w.stride, w.pad, w.dilation, w.offset_scale, dtype_code, sh)
        if rc != 0:
            raise dcn.DCNv4Error(rc, "dcnv4_forward")
        launches[0] += 1

    ms, sampler, timed_launches = time_steps(step, launches, args, dev, stream, barrier, max_over_ranks)
    ms_step = ms / args.steps
    total_points = w.points * world * args.steps
    value = total_points / (ms / 1e3) / 1e9

    # roofline of the (only) kernel: algorithmic bytes per launch / average launch duration
    peak, peak_kind = measured_peaks()
    achieved = foot / (ms_step / 1e3) / 1e9
    traffic, traffic_src = profiled_traffic(w.name)

    # end to end: host buffers in, result back to the host, through dcnv4_forward_host
    xh, omh = x.pin_memory(), om.pin_memory()
    oh = torch.empty((w.N, w.Hout, w.Wout, w.C), dtype=x.dtype).pin_memory()
    xd, omd, od = xs[0], oms[0], outs[0]

    def e2e_step():
        rc = lib.dcnv4_forward_host(xh.data_ptr(), omh.data_ptr(), oh.data_ptr(), xd.data_ptr(), omd.data_ptr(),
                                    od.data_ptr(), w.N, w.H, w.W, w.C, w.G, w.K, w.stride, w.pad, w.dilation,
                                    w.offset_scale, dtype_code, sh)
        if rc != 0:
            raise dcn.DCNv4Error(rc, "dcnv4_forward_host")

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = w.points * world * args.e2e_steps / (e2e_ms / 1e3) / 1e9
    # the result came back through the host path: it must equal the device path bit for bit
    if not torch.equal(oh, outs[0].cpu()):
        raise SystemExit("end-to-end result differs from the device-resident result")

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(w, x, om)

    clocks = sampler.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": ARITH[w.dtype], "data": "synthetic",
            "config": {
                "workload": workload_text(w),
                "storage_dtype": w.dtype, "accumulate": "f32", "global_batch": w.N * world,
                "points_per_step_per_gpu": w.points, "parallelism": f"dp{world} (independent batches)",
                "l2": f"steps rotate over {copies} resident input/output sets, {copies * foot / 1e6:.0f} MB "
                      f"in total vs {l2 / 1e6:.0f} MB L2",
                "inputs": input_recipe(w),
            },
            "hbm_gbs": achieved,
            "hbm_pct_of_peak": 100.0 * achieved / peak,
            "hbm_pct_of_8tbs_nominal": 100.0 * achieved / 8000.0,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel": "dcnv4 forward (one launch per step)",
                         "algorithmic_bytes_per_launch": foot,
                         "traffic": traffic, "traffic_source": traffic_src},
            "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms / args.e2e_steps,
                    "steps": args.e2e_steps,
                    "h2d_bytes_per_step": (x.numel() + om.numel()) * x.element_size(),
                    "d2h_bytes_per_step": oh.numel() * oh.element_size(),
                    "path": "dcnv4_forward_host: pinned host buffers; copies in, kernels and copies out on "
                            "one stream each, over chunks of images (bands of output rows when the batch "
                            "has fewer images than chunks)"},
            "gpu_launches": timed_launches,
            "clocks": clocks,
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
