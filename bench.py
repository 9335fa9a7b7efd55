#!/usr/bin/env python
"""AQLM matmul throughput on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the AQLM linear layers of a workload over one batch of
synthetic activations.  The default workload (the headline) is the largest of the
published configurations: the Mixtral-8x7B expert FFNs of one layer, 8 experts x
(w1, w3 14336x4096; w2 4096x14336), 2x8 g8 codebooks (2 bits per weight), batch 1
per expert, 354 MB of codes per step.  By default (--launch group) a step is one
aqlm_matmul_group call over the set (the grouped lookup-table kernel and its
reduction); --launch per-layer makes it one aqlm_matmul call per layer.  The group
run also times the per-layer launches and reports them beside the headline.

After the headline (N = 1, default workload) the other published configurations
are measured the same way, one record each under "per_config": the 4096x4096 1x16
g8 layer, the Llama-2-7B 2x8 g8 set, the Llama-2-70B 1x16 g8 shapes at batch 1 and
4, the batch sweep 1..256 on 11008x4096 and 4096x11008 per scheme, and the
Mixtral-8x7B experts in 1x16 g16.  Every record carries its roofline against the
binding roof, the one with the longest ideal time for the step: HBM (algorithmic
bytes / measured copy bandwidth), tensor (2 batch N K flops / measured bf16 rate)
or, for the 65536-entry codebooks, the L1TEX gather rate (one random codeword
request per SM and clock); every roof's fraction is listed beside it.

Metric: effective HBM GB/s = algorithmic bytes (codes + codebooks + scales + x +
y, each once) / device time, summed over ranks; microseconds per layer are
reported beside it.  Inputs are resident in HBM; every step reads a different
copy of the layer set from a rotating pool larger than 3x the L2 cache, so no
step finds its weights in L2.  The steps run as replays of CUDA graphs that
each hold one pass over the pool (launches inside a graph overlap through
programmatic dependent launch); every graph the timed region uses is replayed
once before it.  The timed region is bracketed by a barrier and a device
synchronise and measured with CUDA events on the launching stream; the max over
ranks is taken.  With N > 1 GPUs each rank runs its own replica (weak scaling,
no data-path collective).

--impl reference times the CPU oracle (decode to fp16, fp64 matmul) on the
host cores on a bounded sample of rows of every layer per step and reports the
same metric.

--op input-grad times the layer's input gradient instead (dx = dy . diag(s) . W,
one aqlm_input_grad call per layer, default batch 1024 rows of dy, a fine-tuning
micro-batch): metric TFLOP/s (2 . batch . N . K per layer), roofline against
the tensor-core peak when the flops bound it.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from weight_only_additive_b200 import synth, workloads  # noqa: E402

METRIC = "AQLM matmul µs/layer & achieved HBM GB/s (frac. of ~8 TB/s), batch 1–256"
DEFAULT_WORKLOAD = "mixtral_8x7b_experts_2x8g8"
L2_FALLBACK = 126 * 1024 * 1024


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default 20000; 1000 with --op input-grad)")
    p.add_argument("--warmup", type=int, default=1000)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.BY_NAME))
    p.add_argument("--batch", type=int, default=None, help="override the workload's batch size")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="skip the records of the other published configurations after the headline")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    p.add_argument("--layer", default=None, help="time only this layer of the workload (e.g. q_proj)")
    p.add_argument("--no-other-launch", action="store_true",
                   help="skip the comparison timings beside the headline: per-layer launches (group mode), "
                        "launches without CUDA graphs, and aqlm_dequantize + cuBLAS (the context line)")
    p.add_argument("--launch", choices=("group", "per-layer"), default="group",
                   help="one aqlm_matmul_group call per step (default) or one aqlm_matmul call per layer")
    p.add_argument("--scheme", default=None,
                   help="replace every layer's codebook scheme (MxBgG, e.g. 4x8g8): the generic shapes")
    p.add_argument("--op", choices=("matmul", "input-grad"), default="matmul",
                   help="the layer (default) or its input gradient dx = dy . diag(s) . W")
    p.add_argument("--schedule", choices=("auto", "tiles", "streamk"), default="auto",
                   help="work schedule of the tensor-core kernel for --launch per-layer and --op input-grad "
                        "(aqlm_schedule; the group call always uses auto)")
    p.add_argument("--pool", type=int, default=None,
                   help="rotating-pool copies (default: enough to exceed 3x L2); smaller for profiler captures")
    a = p.parse_args(argv)
    if a.steps is None:
        a.steps = 1000 if a.op == "input-grad" else 20000
    if a.warmup < 3:
        p.error("--warmup must be at least 3")
    return a


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    """Roofline denominators: MEASURED_PEAKS.json (the machine's measured copy bandwidth and
    cuBLAS bf16 rates; fp16 has the same nominal tensor rate), else the fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured",
                "tc_tflops": float(d.get("bf16_tflops", 1590.0)),
                "tc_tflops_sustained": float(d.get("bf16_tflops_sustained", 1400.0)),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0))}
    return {"hbm_gbs": 6650.0, "source": "fallback", "tc_tflops": 1590.0, "tc_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}


# the files under csrc/ each kernel is compiled from (its .cu first, then the headers
# that hold its device code): a traffic record is valid only while they are unchanged
KERNEL_SOURCES = {"gemv_gather_kernel": ("gemv.cu", "aqlm_device.cuh"),
                  "gemv_lut_kernel": ("gemv_lut.cu", "lut_table.cuh", "aqlm_device.cuh"),
                  "tc_decode_mma_kernel": ("tc_gemm.cu", "aqlm_device.cuh"),
                  "tc_pipe_kernel": ("tc_pipe.cu", "aqlm_device.cuh"),
                  "lut_group_kernel": ("lut_group.cu", "lut_table.cuh", "aqlm_device.cuh")}


def schedule_of(a, native):
    """The aqlm_schedule value of --schedule."""
    return {"auto": native.Schedule.AUTO, "tiles": native.Schedule.TILES,
            "streamk": native.Schedule.STREAMK}[getattr(a, "schedule", "auto")]


def kernel_source_sha256(kernel):
    """sha256 over the kernel's source files, concatenated in KERNEL_SOURCES order."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "weight_only_additive_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload_name, kernel):
    """DRAM bytes per launch (read + write) of `kernel` on this workload, from the ncu
    capture recorded in profiles/roofline_traffic.json -- or None when there is none or
    the kernel's source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    with open(path) as fh:
        rec = json.load(fh).get(f"{workload_name}/{kernel}")
    if not rec or rec.get("kernel") != kernel:
        return None
    if kernel_source_sha256(kernel) != rec.get("source_sha256"):
        return None
    return rec.get("dram_bytes_per_launch")


def workload_batch(w, override):
    return override if override is not None else w.batches[0]


def parse_scheme(text):
    """'MxBgG' (e.g. 4x8g8, 2x16g16) -> workloads.Scheme."""
    import re
    m = re.fullmatch(r"(\d+)x(\d+)g(\d+)", text or "")
    if not m:
        raise SystemExit(f"--scheme {text!r}: expected MxBgG, e.g. 4x8g8")
    return workloads.Scheme(int(m.group(1)), int(m.group(2)), int(m.group(3)))


def select_workload(a):
    """The named workload, restricted to one layer when --layer is given, with every
    layer's codebook scheme replaced when --scheme is given."""
    w = workloads.get(a.workload)
    if getattr(a, "scheme", None):
        sch = parse_scheme(a.scheme)
        layers = tuple(workloads.Layer(l.name, l.N, l.K, sch) for l in w.layers)
        w = workloads.Workload(w.index, f"{w.name}@{sch.name}", layers, w.batches, w.description)
    if a.layer is None:
        return w
    layers = tuple(l for l in w.layers if l.name == a.layer)
    if not layers:
        raise SystemExit(f"--layer {a.layer!r} is not a layer of {w.name}: {[l.name for l in w.layers]}")
    idx = [i for i, l in enumerate(w.layers) if l.name == a.layer][0]
    return workloads.Workload(w.index, f"{w.name}/{a.layer}", layers, w.batches, w.description,
                              extra={"layer_offset": idx})


def max_over_ranks(ms, dist, device):
    """The slowest rank's time: every rank takes part, every rank gets the max."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(bytes_per_step, steps, world, ms):
    """Whole-job GB/s: the algorithmic bytes all ranks processed / the slowest rank's time."""
    return bytes_per_step * steps * world / (ms / 1e3) / 1e9


def step_bytes(w, batch):
    return sum(l.algorithmic_bytes(batch) for l in w.layers)


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.gpu = gpu_index
        self.proc = None
        self.enabled = enabled

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                time.sleep(0.3)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7], sw_power=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": rows[0]["max"],
                "power_w_max": max(r["power"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on the host cores, bounded row samples
# ---------------------------------------------------------------------------
_HOST_LAYERS = {}


def host_layers(w, batch):
    """The workload's layers as host arrays (generated once per process)."""
    key = (w.name, batch)
    if key not in _HOST_LAYERS:
        layers = []
        for li, lay in enumerate(w.layers):
            s = lay.scheme
            ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index, layer=li)
            x = synth.make_x(batch, lay.K, seed=0, workload=w.index, layer=li)
            layers.append((lay, ld, x))
        _HOST_LAYERS[key] = layers
    return _HOST_LAYERS[key]


def oracle_sample_run(w, batch, seconds, copy=0, nthreads=0):
    """Times oracle.linear (decode + fp64 matmul) on row samples of every layer, repeating
    the sample until about `seconds` of CPU time have been spent; nthreads = 0 uses every
    host core (OpenMP), else that many threads.
    Returns (algorithmic bytes of the sampled fraction, seconds, rows per layer, threads)."""
    import oracle

    layers = host_layers(w, batch)
    # probe the per-row cost on a few rows of each layer
    t0 = time.perf_counter()
    for lay, ld, x in layers:
        oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, ld.M, ld.B, ld.g, rows=np.arange(8),
                      nthreads=nthreads)
    probe = (time.perf_counter() - t0) / 8.0  # seconds per "one row of every layer"
    rows = max(1, int(seconds / max(probe, 1e-9)))
    total_bytes, elapsed, sampled = 0.0, 0.0, 0
    rng = np.random.Generator(np.random.PCG64(copy))
    while True:
        for lay, ld, x in layers:
            r = min(rows, lay.N)
            sel = np.sort(rng.choice(lay.N, size=r, replace=False))
            t0 = time.perf_counter()
            oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, ld.M, ld.B, ld.g, rows=sel,
                          nthreads=nthreads)
            elapsed += time.perf_counter() - t0
            total_bytes += lay.algorithmic_bytes(batch) * (r / lay.N)
        sampled += rows
        if elapsed >= 0.9 * seconds:
            break
    return total_bytes, elapsed, sampled, nthreads if nthreads > 0 else oracle.max_threads()


def host_cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_kernel_run(w, batch, seconds):
    """Times libaqlm_cpu.so (the multithreaded lookup-table / decode+dot CPU kernel)
    on whole layers of the workload, repeating the set for about `seconds`.  Not the
    oracle: reported beside cpu_baseline as the fast CPU implementation."""
    from weight_only_additive_b200 import cpu as cpu_lib

    layers = host_layers(w, batch)
    cpu_lib.matmul(layers[0][2], layers[0][1].codes, layers[0][1].codebooks, layers[0][1].scales, None,
                   layers[0][1].M, layers[0][1].B, layers[0][1].g)  # warm-up (thread pool, pages)
    passes, elapsed = 0, 0.0
    while elapsed < seconds or passes < 2:
        t0 = time.perf_counter()
        for lay, ld, x in layers:
            cpu_lib.matmul(x, ld.codes, ld.codebooks, ld.scales, None, ld.M, ld.B, ld.g)
        elapsed += time.perf_counter() - t0
        passes += 1
    sbytes = step_bytes(w, batch)
    level, B = cpu_lib.simd_level(), w.layers[0].scheme.B
    lut = B == 8 and (batch == 1 if level == 2 else batch <= 8)
    method = ("lookup tables per 16-group K slice" if lut
              else "fused decode + dot in registers" if level == 2 else "decode to fp32 + dot products")
    return {"value": sbytes * passes / elapsed / 1e9, "unit": "GB/s",
            "ms_per_step": elapsed * 1e3 / passes, "cores": os.cpu_count(),
            "simd": cpu_lib.SIMD_NAMES.get(cpu_lib.simd_level(), "?"),
            "kind": "libaqlm_cpu.so (aqlm_cpu_matmul)",
            "sample": f"{passes} passes over all {len(w.layers)} whole layers, batch {batch}, {method}, "
                      f"{elapsed:.1f} s"}


def pool_copies(copy_bytes, l2, copies=None):
    """How many seeded copies of a workload's layers the timing pool holds: at least 3x
    L2 so no step finds its weights in L2, and at least 8 copies so a CUDA graph holds
    8 steps (consecutive launches overlap through programmatic dependent launch inside a
    graph, not across graph launches); at most 60 GB.  `copies` overrides the rule."""
    pool = max(8, math.ceil(3 * l2 / copy_bytes)) if copies is None else max(1, copies)
    while pool > 2 and pool * copy_bytes > 60e9:
        pool -= 1
    return pool


def line_config(w, batch, world, launch, schedule, pool, l2):
    """The `config` object of a bench line: the workload, batch, bytes per step, the
    pool that keeps inputs out of L2 and the launch form.  Both arms print it, so the
    two lines name one configuration."""
    copy_bytes = step_bytes(w, batch)
    desc = ("one aqlm_matmul_group call per step (grouped lookup-table kernel + reduction)" if launch == "group"
            else f"one aqlm_matmul_ws call per layer, schedule {schedule}")
    return {"workload": w.name, "layers": len(w.layers), "batch": batch, "scheme": w.layers[0].scheme.name,
            "algorithmic_bytes_per_step": copy_bytes,
            "l2": f"inputs larger than L2: rotating pool of {pool} copies ({pool * copy_bytes / 1e6:.0f} MB > "
                  f"{l2 / 1e6:.0f} MB L2)",
            "launch": desc + f"; CUDA graphs of {pool} consecutive steps (one pass over the pool)",
            "parallelism": f"replicas x{world}"}


def device_l2_bytes():
    """L2 size of device 0, or the fallback size without a usable GPU."""
    try:
        import torch
        if torch.cuda.is_available():
            return getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 0) or L2_FALLBACK
    except Exception:  # no usable device: the fallback size
        pass
    return L2_FALLBACK


def reference_config(a, w, batch, world):
    """The `config` of the matching line of this library's arm (run_ours or
    run_input_grad), with the pool sized by the same rule from the device's L2 size."""
    l2 = device_l2_bytes()
    if a.op == "input-grad":
        return grad_line_config(w, batch, world, a.schedule, grad_pool_copies(grad_step_bytes(w, batch), l2, a.pool),
                                l2)
    return line_config(w, batch, world, a.launch, a.schedule, pool_copies(step_bytes(w, batch), l2, a.pool), l2)


def run_reference(a):
    rank, world, _ = env_rank()
    w = select_workload(a)
    if a.op == "input-grad":
        batch = a.batch if a.batch is not None else GRAD_DEFAULT_BATCH
    else:
        batch = workload_batch(w, a.batch)
    if rank != 0:
        return 0
    # each step is a bounded sample sized so that warmup + steps fit ~2 minutes
    per_step = max(0.002, min(5.0, 120.0 / (a.steps + a.warmup)))
    if a.op == "input-grad":
        return run_reference_grad(a, w, batch, world, per_step)
    for i in range(a.warmup):
        oracle_sample_run(w, batch, per_step, copy=i)
    tot_b, tot_s = 0.0, 0.0
    rows = 0
    for i in range(a.steps):
        b, s, rows, threads = oracle_sample_run(w, batch, per_step, copy=i)
        tot_b += b
        tot_s += s
    value = tot_b / tot_s / 1e9
    sample = (f"{rows} sampled rows of each of the {len(w.layers)} layers per step "
              f"(decode to fp16 + fp64 matmul), batch {batch}")
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": tot_s * 1e3 / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": reference_config(a, w, batch, world),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_grad(a, w, batch, world, per_step):
    """The reference arm of `--op input-grad`: the oracle's input gradient on column
    samples of every layer, per_step seconds of it per step (at least one layer)."""
    for i in range(a.warmup):
        oracle_grad_sample_run(w, batch, per_step, seed=100 + i)
    tot_f, tot_s, cols, threads = 0.0, 0.0, 0, 1
    for i in range(a.steps):
        f, s, cols, threads = oracle_grad_sample_run(w, batch, per_step, seed=1000 + i)
        tot_f += f
        tot_s += s
    value = tot_f / tot_s / 1e12
    sample = (f"{cols} sampled columns of dx per layer and step (the oracle decodes the whole W16 each call, "
              f"then fp64 dy . W16 for those columns), batch {batch}")
    line = {"metric": GRAD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": tot_s * 1e3 / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": reference_config(a, w, batch, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
# One L1TEX request per SM and clock: the rate at which an SM serves gathers of
# random 16-byte (or, with a 256-bit load, 32-byte) codewords from the L2-resident
# 65536-entry codebooks.  Derived from the unit count (one L1TEX unit per SM) and
# the SM clock; probes of random 16-byte gathers on this GPU measured 0.73-1.0.
GATHERS_PER_SM_CLOCK = 1.0

# The published configurations measured after the headline at N = 1, each as
# (workload, scheme filter or None, batch).  The batch sweep holds two schemes and is
# measured per scheme, so every record has one binding roof.
PER_CONFIG = (("single_4096x4096_1x16g8", None, 1),
              ("llama2_7b_layer_set_2x8g8", None, 1),
              ("llama2_70b_layers_1x16g8", None, 1),
              ("llama2_70b_layers_1x16g8", None, 4),
              *(("batch_sweep_11008x4096", "1x16g8", b) for b in (1, 4, 16, 64, 256)),
              *(("batch_sweep_11008x4096", "2x8g8", b) for b in (1, 4, 16, 64, 256)),
              ("mixtral_8x7b_experts_1x16g16", None, 1),
              ("mixtral_8x7b_experts_2x8g8", None, 1))


def scheme_subset(w, scheme_name):
    """The workload restricted to the layers of one codebook scheme."""
    layers = tuple(l for l in w.layers if l.scheme.name == scheme_name)
    if not layers:
        raise SystemExit(f"{w.name} has no {scheme_name} layer")
    return workloads.Workload(w.index, f"{w.name}[{scheme_name}]", layers, w.batches, w.description)


def step_roofs(w, batch, peaks, sms, sm_mhz):
    """The three roofs of one step, each as (time in s, quantity, peak rate, unit):
    HBM (algorithmic bytes), tensor (2 batch N K flops at the measured burst bf16 rate;
    fp16 has the same nominal rate) and the codeword gathers of the B = 16 schemes (one
    request per codeword per code, GATHERS_PER_SM_CLOCK per SM and clock)."""
    nbytes = step_bytes(w, batch)
    flops = sum(l.flops(batch) for l in w.layers)
    gathers = sum(l.N * l.G * l.scheme.M for l in w.layers if l.scheme.B == 16)
    gather_rate = GATHERS_PER_SM_CLOCK * sms * sm_mhz * 1e6
    return {"hbm": (nbytes / (peaks["hbm_gbs"] * 1e9), nbytes / 1e9, peaks["hbm_gbs"], "GB/s"),
            "tensor": (flops / (peaks["tc_tflops"] * 1e12), flops / 1e12, peaks["tc_tflops"], "TFLOP/s"),
            "l1tex_gather": (gathers / gather_rate, gathers / 1e9, gather_rate / 1e9, "Greq/s")}


def roofline_record(w, batch, step_s, peaks, sms, sm_mhz):
    """`roofline` of a step: the binding roof (the one with the longest ideal time),
    achieved = its quantity per step / the measured step time, against its peak; and
    every roof's fraction beside it."""
    roofs = step_roofs(w, batch, peaks, sms, sm_mhz)
    bound = max(roofs, key=lambda k: roofs[k][0])
    out = {}
    for name, (t, qty, peak, unit) in roofs.items():
        if qty == 0:
            continue
        achieved = qty / step_s
        out[name] = {"achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                     "ideal_us": t * 1e6}
    rec = {"bound": bound, **{k: out[bound][k] for k in ("achieved", "peak", "unit", "frac")},
           "roofs": out}
    src = "measured (MEASURED_PEAKS.json)" if peaks["source"] == "measured" else "fallback"
    rec["peak_source"] = {"hbm": f"{src} hbm_gbs", "tensor": f"{src} bf16_tflops (burst)",
                          "l1tex_gather": f"{GATHERS_PER_SM_CLOCK:g} request per SM per clock x {sms} SMs x "
                                          f"{sm_mhz:.0f} MHz"}[bound]
    l2 = l2_gather_traffic(w, batch)
    if l2 is not None:
        rec["l2_gather_sectors"] = l2
    return rec


def l2_gather_traffic(w, batch):
    """The L2 sector traffic of the B = 16 schemes' codeword gathers, next to the HBM
    bytes: one 32-byte L2 sector per codeword piece, once per decode of a weight tile
    (one decode per 256-wide batch tile).  None for a workload without B = 16 layers."""
    sectors = sum(l.N * l.G * l.scheme.M * -(-batch // 256) for l in w.layers if l.scheme.B == 16)
    if not sectors:
        return None
    return {"sectors": sectors, "bytes": 32 * sectors, "per_hbm_byte": 32 * sectors / step_bytes(w, batch),
            "basis": "one 32-byte sector per codeword gather; ncu counted 2,337,475 L2 sectors read by the SMs "
                     "for the 2,097,152 gathers plus 5.3 MB of codes of 4096x4096 1x16 g8 at batch 1 "
                     "(profiles/tc_pipe_1x16g8_4096x4096_b1.md)"}


class Bench:
    """The device, stream and library shared by every measurement of one run."""

    def __init__(self, a):
        import torch

        from weight_only_additive_b200 import layer as L
        from weight_only_additive_b200 import native

        self.torch, self.L, self.native = torch, L, native
        self.a = a
        self.rank, self.world, self.local = env_rank()
        if self.world > 1:
            import torch.distributed as dist
            torch.cuda.set_device(self.local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local))
            self.dist = dist
        else:
            self.dist = None
            torch.cuda.set_device(self.local)
        self.dev = torch.device("cuda", self.local)
        self.lib = native.lib()
        self.props = torch.cuda.get_device_properties(self.dev)
        self.l2 = getattr(self.props, "L2_cache_size", 0) or L2_FALLBACK
        self.sms = self.props.multi_processor_count
        self.stream = torch.cuda.Stream(self.dev)
        self.peaks = measured_peaks()

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()


class Pool:
    """A rotating pool of seeded copies of a workload's layers, resident in HBM and
    larger than 3x L2, with one aqlm_matmul_group problem table (and workspace) per copy."""

    def __init__(self, b, w, batch, copies=None):
        torch, L = b.torch, b.L
        self.w, self.batch = w, batch
        copy_bytes = step_bytes(w, batch)
        pool = pool_copies(copy_bytes, b.l2, copies)
        self.size, self.copy_bytes = pool, copy_bytes
        self.weights, self.xs = [], []
        off = w.extra.get("layer_offset", 0)
        for c in range(pool):
            wc, xc = [], []
            for li, lay in enumerate(w.layers):
                s = lay.scheme
                ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index,
                                      layer=li + off, copy=c + 1000 * b.rank)
                wc.append(L.AqlmWeights.from_numpy(ld, b.dev))
                xc.append(torch.from_numpy(synth.make_x(batch, lay.K, seed=0, workload=w.index, layer=li,
                                                        copy=c + 1000 * b.rank)).to(b.dev))
            self.weights.append(wc)
            self.xs.append(xc)
        self.ys = [torch.empty((batch, lay.N), dtype=torch.float16, device=b.dev) for lay in w.layers]
        self.groups = [L.LayerGroup([(self.weights[c][li], self.xs[c][li], self.ys[li])
                                     for li in range(len(w.layers))]) for c in range(pool)]
        h = b.stream.cuda_stream
        # one zero-filled workspace for the per-layer calls (they run in turn on one stream)
        ws_bytes = max(b.native.aqlm_matmul_workspace_size(l.scheme.M, l.scheme.B, l.scheme.g, l.K, l.N, batch)
                       for l in w.layers)
        self.ws = torch.zeros((max(ws_bytes, 1),), dtype=torch.uint8, device=b.dev)
        ws = (self.ws.data_ptr(), ws_bytes) if ws_bytes else (None, 0)
        self.calls = [[(self.xs[c][li].data_ptr(), wt.codes.data_ptr(), wt.codebooks.data_ptr(), wt.scales.data_ptr(),
                        None, self.ys[li].data_ptr(), wt.M, wt.B, wt.g, lay.K, lay.N, batch, int(b.native.Path.AUTO),
                        int(schedule_of(b.a, b.native)), ws[0] if b.native.aqlm_matmul_workspace_size(wt.M, wt.B, wt.g, lay.K, lay.N, batch) else None,
                        ws[1] if b.native.aqlm_matmul_workspace_size(wt.M, wt.B, wt.g, lay.K, lay.N, batch) else 0, h)
                       for li, (lay, wt) in enumerate(zip(w.layers, self.weights[c]))] for c in range(pool)]
        self.b = b

    def step_group(self, c):
        self.groups[c].run(stream=self.b.stream)

    def step_per_layer(self, c):
        for args in self.calls[c]:
            st = self.b.lib.aqlm_matmul_ws(*args)
            if st != 0:
                raise self.b.native.AqlmError(st, "aqlm_matmul_ws")

    def grouped_layers(self):
        return sum(1 for l in self.w.layers if l.scheme.B == 8 and self.batch == 1 and l.K % l.scheme.g == 0
                   and (l.K // l.scheme.g * l.scheme.M) % 16 == 0)

    def launches(self, mode):
        """Kernel launches of one step: the grouped layers take two (partial sums and
        reduction) per run of up to MAX_GROUP_LAYERS; every other layer one."""
        n = len(self.w.layers)
        if mode == "per-layer":
            return n
        grouped = self.grouped_layers()
        runs = (grouped + self.b.native.MAX_GROUP_LAYERS - 1) // self.b.native.MAX_GROUP_LAYERS
        return 2 * runs + (n - grouped)

    def kernel(self, mode):
        if mode == "group" and self.grouped_layers() == len(self.w.layers):
            return "lut_group_kernel"
        lay = self.w.layers[0]
        path = self.b.native.aqlm_select_path(lay.scheme.M, lay.scheme.B, lay.scheme.g, lay.K, lay.N, self.batch)
        P = self.b.native.Path
        return {int(P.GEMV): "gemv_gather_kernel", int(P.GEMV_LUT): "gemv_lut_kernel",
                int(P.TENSOR_CORE): "tc_pipe_kernel"}.get(int(path), "?")

    def timed(self, step, steps, warmup, sample_clocks=False):
        """`steps` steps as replays of CUDA graphs that each hold one pass over the pool
        (copy c at step c), plus one graph for the remainder; launches inside a graph
        overlap through programmatic dependent launch.  Every graph the timed region
        replays is captured and replayed at least once before it, whatever `warmup` is,
        so no first-replay cost lands in the timed region."""
        b, torch, pool = self.b, self.b.torch, self.size
        with torch.cuda.stream(b.stream):
            for c in range(pool):
                step(c)
        torch.cuda.synchronize(b.dev)

        def capture(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=b.stream):
                for c in range(n):
                    step(c)
            return g

        full = capture(pool)
        rest = {}
        for n in (steps % pool, warmup % pool):
            if n and n not in rest:
                rest[n] = capture(n)

        def run(n):
            for _ in range(n // pool):
                full.replay()
            if n % pool:
                rest[n % pool].replay()

        with torch.cuda.stream(b.stream):
            full.replay()
            for g in rest.values():
                g.replay()
            run(warmup)
        torch.cuda.synchronize(b.dev)
        b.barrier()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        with ClockSampler(b.local, enabled=sample_clocks) as clocks:
            torch.cuda.synchronize(b.dev)
            b.barrier()
            with torch.cuda.stream(b.stream):
                start.record(b.stream)
                run(steps)
                end.record(b.stream)
            torch.cuda.synchronize(b.dev)
            b.barrier()
        ms = max_over_ranks(start.elapsed_time(end), b.dist, b.dev)
        st, detail = b.L.check_device_status(stream=b.stream)
        if st != b.native.Status.OK:
            raise RuntimeError(f"device status {st.name} {detail:#x}")
        del full, rest
        return ms, clocks.summary()

    def e2e(self, mode, steps):
        """The same metric through the public API with host buffers: per step one pinned
        H2D copy of every layer's x (packed), the group call (aqlm_matmul_group_host, the
        copies inside the call) or one aqlm_matmul per layer, one D2H copy of every y.
        Steps alternate between two streams, each with its own host and device buffers
        (double buffering, as a serving loop would), so one step's copies overlap the
        other stream's kernels; every step still moves its own inputs and result."""
        b, torch, w, batch = self.b, self.b.torch, self.w, self.batch
        L = b.L
        koff = np.cumsum([0] + [batch * lay.K for lay in w.layers])
        noff = np.cumsum([0] + [batch * lay.N for lay in w.layers])
        streams = [b.stream, torch.cuda.Stream(b.dev)]
        sets = []
        for si in range(2):
            hx_flat = torch.empty((int(koff[-1]),), dtype=torch.float16).pin_memory()
            for li, lay in enumerate(w.layers):
                hx_flat[koff[li]:koff[li + 1]] = torch.from_numpy(
                    synth.make_x(batch, lay.K, seed=7 + si, layer=li)).reshape(-1)
            hy_flat = torch.empty((int(noff[-1]),), dtype=torch.float16).pin_memory()
            dx_flat = torch.empty_like(hx_flat, device=b.dev)
            dy_flat = torch.empty_like(hy_flat, device=b.dev)
            dx = [dx_flat[koff[li]:koff[li + 1]].view(batch, lay.K) for li, lay in enumerate(w.layers)]
            dy = [dy_flat[noff[li]:noff[li + 1]].view(batch, lay.N) for li, lay in enumerate(w.layers)]
            groups = ([L.LayerGroup([(self.weights[c][li], dx[li], dy[li]) for li in range(len(w.layers))])
                       for c in range(self.size)] if mode == "group" else None)
            sets.append((hx_flat, hy_flat, dx_flat, dy_flat, dx, dy, groups))

        def e2e_step(i):
            si, c = i % 2, i % self.size
            hx_flat, hy_flat, dx_flat, dy_flat, dx, dy, groups = sets[si]
            st = streams[si]
            if mode == "group":
                groups[c].run_host(hx_flat, hy_flat, stream=st)
            else:
                with torch.cuda.stream(st):
                    dx_flat.copy_(hx_flat, non_blocking=True)
                    for li in range(len(w.layers)):
                        L.matmul(dx[li], self.weights[c][li], out=dy[li], stream=st)
                    hy_flat.copy_(dy_flat, non_blocking=True)

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize(b.dev)
        b.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(steps):
            e2e_step(i)
        done1 = torch.cuda.Event()
        done1.record(streams[1])
        streams[0].wait_event(done1)
        e1.record(streams[0])
        torch.cuda.synchronize(b.dev)
        ems = max_over_ranks(e0.elapsed_time(e1), b.dist, b.dev)
        api = ("weight_only_additive_b200.layer.LayerGroup.run_host -> aqlm_matmul_group_host (the copies "
               "inside the call)" if mode == "group"
               else "weight_only_additive_b200.layer.matmul -> aqlm_matmul_ws, per layer")
        return {"value": job_throughput_gbs(self.copy_bytes, steps, b.world, ems), "unit": "GB/s",
                "h2d_bytes_per_step": sets[0][0].numel() * 2, "d2h_bytes_per_step": sets[0][1].numel() * 2,
                "steps": steps, "us_per_layer": ems * 1e3 / (steps * len(w.layers)),
                "how": f"per step: one pinned H2D copy of every layer's x (packed), {api}, one D2H copy "
                       f"of every y (packed); no CUDA graph; steps alternate between two streams with their "
                       f"own host and device buffers, so one step's copies overlap the other's kernels"}


def measure_config(b, w, batch, steps, warmup, with_e2e=True):
    """One per-config record: the group call of every layer per step (graphs over the
    pool), its binding roofline, and the end-to-end number through host buffers."""
    pool = Pool(b, w, batch)
    ms, _ = pool.timed(pool.step_group, steps, warmup)
    step_s = ms / 1e3 / steps
    sm_mhz = b.peaks["sm_max_mhz"]
    rec = {"workload": w.name, "batch": batch, "scheme": w.layers[0].scheme.name, "layers": len(w.layers),
           "value": job_throughput_gbs(pool.copy_bytes, steps, b.world, ms), "unit": "GB/s",
           "us_per_layer": step_s * 1e6 / len(w.layers), "us_per_step": step_s * 1e6, "steps": steps,
           "kernel": pool.kernel("group"), "gpu_launches_per_step": pool.launches("group"),
           "roofline": roofline_record(w, batch, step_s, b.peaks, b.sms, sm_mhz),
           "pool": f"{pool.size} copies ({pool.size * pool.copy_bytes / 1e6:.0f} MB)"}
    if with_e2e:
        rec["e2e"] = pool.e2e("group", steps)
    del pool
    b.torch.cuda.empty_cache()
    return rec


def run_ours(a):
    b = Bench(a)
    torch, L, native = b.torch, b.L, b.native
    rank, world, dev = b.rank, b.world, b.dev
    w = select_workload(a)
    batch = workload_batch(w, a.batch)
    sbytes = step_bytes(w, batch)
    pool = Pool(b, w, batch, a.pool)
    mode = a.launch
    ms, clock_summary = pool.timed(pool.step_group if mode == "group" else pool.step_per_layer, a.steps, a.warmup,
                                   not a.no_clocks)
    launches_per_step = pool.launches(mode)
    value = job_throughput_gbs(sbytes, a.steps, world, ms)
    ms_step = ms / a.steps
    other = None
    if mode == "group" and not a.no_other_launch:
        # the same workload with one aqlm_matmul launch per layer, for comparison
        o_steps = min(a.steps, 20000)
        o_ms, _ = pool.timed(pool.step_per_layer, o_steps, max(3, min(a.warmup, 200)))
        other = {"launch": "per-layer", "value": job_throughput_gbs(sbytes, o_steps, world, o_ms),
                 "unit": "GB/s", "us_per_layer": o_ms * 1e3 / (o_steps * len(w.layers)), "steps": o_steps}

    direct = context = None
    if not a.no_other_launch:
        # launch overhead included: the same steps issued one by one from the host, no graph
        d_steps = min(a.steps, 2000)
        step = pool.step_group if mode == "group" else pool.step_per_layer
        with torch.cuda.stream(b.stream):
            for i in range(3):
                step(i % pool.size)
        torch.cuda.synchronize(dev)
        b.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(b.stream):
            e0.record(b.stream)
            for i in range(d_steps):
                step(i % pool.size)
            e1.record(b.stream)
        torch.cuda.synchronize(dev)
        d_ms = max_over_ranks(e0.elapsed_time(e1), b.dist, dev)
        direct = {"launch": mode, "value": job_throughput_gbs(sbytes, d_steps, world, d_ms), "unit": "GB/s",
                  "us_per_layer": d_ms * 1e3 / (d_steps * len(w.layers)), "steps": d_steps,
                  "how": "the timed step launched from Python once per step, no CUDA graph"}
        # context: the dequantise-then-GEMM route on the same layers (W written to HBM by
        # aqlm_dequantize, then cuBLAS through torch.matmul); not this library's path
        wbuf = [torch.empty((lay.N, lay.K), dtype=torch.float16, device=dev) for lay in w.layers]

        def step_context(c):
            for li in range(len(w.layers)):
                L.dequantize(pool.weights[c][li], out=wbuf[li], stream=b.stream)
                torch.matmul(pool.xs[c][li], wbuf[li].t(), out=pool.ys[li])

        c_steps = min(a.steps, 2000)
        c_ms, _ = pool.timed(step_context, c_steps, 3)
        context = {"what": "aqlm_dequantize + torch.matmul (cuBLAS fp16) per layer", "unit": "GB/s",
                   "value": job_throughput_gbs(sbytes, c_steps, world, c_ms),
                   "us_per_layer": c_ms * 1e3 / (c_steps * len(w.layers)), "steps": c_steps,
                   "how": "algorithmic bytes of the step / time; W itself crosses HBM twice more"}
        del wbuf

    peaks = b.peaks
    kernel = pool.kernel(mode)
    sm_mhz = clock_summary.get("sm_mhz") or peaks["sm_max_mhz"]
    if kernel == "lut_group_kernel":
        # every layer grouped: the timed launches are the partial-sum kernel and its
        # reduction, measured together (one step = one group call); the rate below is
        # therefore a lower bound on the partial-sum kernel's own
        timed_as = "step: lut_group_kernel + lut_group_reduce_kernel"
    else:
        timed_as = "step: every launch of the step (one family of kernels)"
    roofline = roofline_record(w, batch, ms_step / 1e3, peaks, b.sms, sm_mhz)
    roofline.update({"traffic": measured_traffic(w.name, kernel) if roofline["bound"] == "hbm" else None,
                     "kernel": kernel, "timed": timed_as, "algorithmic_bytes": sbytes})

    e2e = pool.e2e(mode, min(a.steps, 2000)) if not a.no_e2e else None

    cpu = None
    cpu_kernel = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        bb, s, rows, threads = oracle_sample_run(w, batch, a.cpu_seconds)
        cpu = {"value": bb / s / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} rows of each of the {len(w.layers)} layers (whole layers repeated "
                         f"when the budget exceeds them; decode to fp16 + fp64 matmul), batch {batch}, "
                         f"{s:.1f} s on the host cores"}
        cpu["cpu_model"] = host_cpu_model()
        # the same oracle on one thread, a shorter sample
        b1, s1, rows1, _ = oracle_sample_run(w, batch, min(3.0, a.cpu_seconds / 4), copy=1, nthreads=1)
        cpu["single_thread"] = {"value": b1 / s1 / 1e9, "unit": "GB/s", "cores": 1,
                                "sample": f"{rows1} rows of each layer, {s1:.1f} s on one thread"}
        cpu_kernel = cpu_kernel_run(w, batch, min(a.cpu_seconds, 5.0))
    config = line_config(w, batch, world, mode, a.schedule, pool.size, b.l2)
    del pool
    torch.cuda.empty_cache()

    per_config = None
    if world == 1 and not a.no_per_config and a.workload == DEFAULT_WORKLOAD and a.scheme is None \
            and a.layer is None and a.batch is None:
        per_config = []
        sub_steps = min(max(a.steps, 20), 2000)
        for name, scheme, bt in PER_CONFIG:
            sw = workloads.get(name)
            if scheme is not None:
                sw = scheme_subset(sw, scheme)
            if sw.name == w.name and bt == batch:
                continue  # the headline itself
            per_config.append(measure_config(b, sw, bt, sub_steps, max(3, min(a.warmup, 50)),
                                             with_e2e=not a.no_e2e))

    b.close()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms_step,
                "us_per_layer": ms_step * 1e3 / len(w.layers),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
                "data": "synthetic",
                "config": config,
                "roofline": roofline, "cpu_baseline": cpu, "cpu_kernel": cpu_kernel, "e2e": e2e,
                "other_launch": other, "no_graph": direct, "context": context,
                "per_config": per_config,
                "gpu_launches": launches_per_step * a.steps,
                "clocks": clock_summary, "gpu": b.props.name}
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# input gradient dx = dy . diag(s) . W
# ---------------------------------------------------------------------------
GRAD_METRIC = "AQLM input gradient dx = dy·diag(s)·W: TFLOP/s (2·batch·N·K per layer) & µs/layer"
GRAD_DEFAULT_BATCH = 1024


def grad_step_bytes(w, batch):
    """Algorithmic bytes of one pass: codes + codebooks + scales + dy + dx per layer."""
    out = 0
    for l in w.layers:
        s = l.scheme
        out += (l.N * l.G * s.M * s.code_bytes + s.M * (1 << s.B) * s.g * 2 + 2 * l.N
                + 2 * batch * l.N + 2 * batch * l.K)
    return out


_GRAD_HOST = {}


def grad_host_layers(w, batch):
    """The workload's layers and dy [batch, N] as host arrays (generated once per process)."""
    key = (w.name, batch)
    if key not in _GRAD_HOST:
        host = []
        for li, lay in enumerate(w.layers):
            s = lay.scheme
            host.append((synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index, layer=li),
                         synth.make_x(batch, lay.N, seed=1, workload=w.index, layer=li)))
        _GRAD_HOST[key] = host
    return _GRAD_HOST[key]


def oracle_grad_sample_run(w, batch, seconds, seed=5):
    """Times oracle.input_grad (decode to fp16 + fp64 dy . W16) on column samples of
    every layer until about `seconds` have been spent (at least one layer).  Returns
    (flops credited, seconds, columns per layer, threads)."""
    import oracle

    rng = np.random.Generator(np.random.PCG64(seed))
    flops, elapsed, cols = 0.0, 0.0, 16
    host = grad_host_layers(w, batch)
    while elapsed < 0.9 * seconds:
        for lay, (ld, dy) in zip(w.layers, host):
            s = lay.scheme
            sel = np.sort(rng.choice(lay.K, size=cols, replace=False))
            t0 = time.perf_counter()
            oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, s.M, s.B, s.g, cols=sel)
            elapsed += time.perf_counter() - t0
            flops += 2.0 * batch * lay.N * cols
            if elapsed >= 0.9 * seconds:
                break
    return flops, elapsed, cols, oracle.max_threads()


def grad_pool_copies(step_bytes_, l2, copies=None):
    """Copies of the workload in the input-gradient timing pool: at least 3x L2 and at
    least 2 (`copies` overrides)."""
    return max(2, math.ceil(3 * l2 / step_bytes_)) if copies is None else max(1, copies)


def grad_line_config(w, batch, world, schedule, pool, l2):
    """The `config` object of an input-gradient line; both arms print it."""
    sbytes = grad_step_bytes(w, batch)
    return {"workload": w.name, "op": "input-grad", "layers": len(w.layers), "batch": batch,
            "scheme": w.layers[0].scheme.name, "algorithmic_bytes_per_step": sbytes,
            "flops_per_step": sum(2.0 * batch * l.N * l.K for l in w.layers),
            "l2": f"inputs larger than L2: rotating pool of {pool} copies "
                  f"({pool * sbytes / 1e6:.0f} MB > {l2 / 1e6:.0f} MB L2)",
            "launch": f"one aqlm_input_grad_ws call per layer, schedule {schedule}; CUDA graphs of {pool} steps",
            "parallelism": f"replicas x{world}"}


def run_input_grad(a):
    import torch

    from weight_only_additive_b200 import layer as L
    from weight_only_additive_b200 import native

    rank, world, local = env_rank()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        dist = None
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = native.lib()
    w = select_workload(a)
    batch = a.batch if a.batch is not None else GRAD_DEFAULT_BATCH
    sbytes = grad_step_bytes(w, batch)
    sflops = sum(2.0 * batch * l.N * l.K for l in w.layers)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 0) or L2_FALLBACK
    pool = grad_pool_copies(sbytes, l2, a.pool)

    weights, dys = [], []
    for c in range(pool):
        wc, dc = [], []
        for li, lay in enumerate(w.layers):
            s = lay.scheme
            ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index,
                                  layer=li + w.extra.get("layer_offset", 0), copy=c + 1000 * rank)
            wc.append(L.AqlmWeights.from_numpy(ld, dev))
            dc.append(torch.from_numpy(synth.make_x(batch, lay.N, seed=1, workload=w.index, layer=li,
                                                    copy=c + 1000 * rank)).to(dev))
        weights.append(wc)
        dys.append(dc)
    dxs = [torch.empty((batch, lay.K), dtype=torch.float16, device=dev) for lay in w.layers]
    stream = torch.cuda.Stream(dev)
    h = stream.cuda_stream
    # one zero-filled workspace for the stream-K schedule, shared by the calls in turn
    ws_need = [native.aqlm_input_grad_workspace_size(l.scheme.M, l.scheme.B, l.scheme.g, l.K, l.N, batch)
               for l in w.layers]
    ws = torch.zeros((max(max(ws_need), 1),), dtype=torch.uint8, device=dev)
    calls = [[(dys[c][li].data_ptr(), weights[c][li].codes.data_ptr(), weights[c][li].codebooks.data_ptr(),
               weights[c][li].scales.data_ptr(), dxs[li].data_ptr(), lay.scheme.M, lay.scheme.B, lay.scheme.g,
               lay.K, lay.N, batch, int(schedule_of(a, native)), ws.data_ptr() if ws_need[li] else None,
               ws.numel() if ws_need[li] else 0, h)
              for li, lay in enumerate(w.layers)] for c in range(pool)]

    def step(c):
        for args in calls[c]:
            st = lib.aqlm_input_grad_ws(*args)
            if st != 0:
                raise native.AqlmError(st, "aqlm_input_grad_ws")

    def barrier():
        if dist is not None:
            dist.barrier()

    with torch.cuda.stream(stream):
        for c in range(pool):
            step(c)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for c in range(pool):
            step(c)
    passes = max(1, a.steps // pool)
    steps = passes * pool
    with torch.cuda.stream(stream):
        for _ in range(-(-a.warmup // pool)):  # at least `warmup` steps
            graph.replay()
    torch.cuda.synchronize(dev)
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, enabled=not a.no_clocks) as clocks:
        torch.cuda.synchronize(dev)
        barrier()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(passes):
                graph.replay()
            end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    st, detail = L.check_device_status(stream=stream)
    if st != native.Status.OK:
        raise RuntimeError(f"device status {st.name} {detail:#x}")
    del graph
    ms_step = ms / steps
    value = sflops * steps * world / (ms / 1e3) / 1e12
    peaks = measured_peaks()
    launch_s = (ms / 1e3) / (steps * len(w.layers))
    t_tc = sflops / len(w.layers) / (peaks["tc_tflops_sustained"] * 1e12)
    t_hbm = sbytes / len(w.layers) / (peaks["hbm_gbs"] * 1e9)
    if t_tc >= t_hbm:
        roofline = {"bound": "tensor", "achieved": sflops / len(w.layers) / launch_s / 1e12,
                    "peak": peaks["tc_tflops_sustained"], "unit": "TFLOP/s"}
    else:
        roofline = {"bound": "hbm", "achieved": sbytes / len(w.layers) / launch_s / 1e9,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roofline.update({"frac": roofline["achieved"] / roofline["peak"], "traffic": None,
                     "kernel": "tc_pipe_kernel (input gradient)", "timed": "average launch of the step",
                     "peak_source": ("measured (MEASURED_PEAKS.json bf16_tflops_sustained; fp16 has the same "
                                     "nominal tensor rate)" if roofline["bound"] == "tensor"
                                     else "measured (MEASURED_PEAKS.json hbm_gbs)")
                     if peaks["source"] == "measured" else "fallback"})

    e2e = None
    if not a.no_e2e:
        e2e_steps = max(3, min(steps, 200))
        noff = np.cumsum([0] + [batch * lay.N for lay in w.layers])
        koff = np.cumsum([0] + [batch * lay.K for lay in w.layers])
        # two streams, each with its own host and device buffers (double buffering):
        # one step's copies overlap the other stream's kernels
        streams = [stream, torch.cuda.Stream(dev)]
        sets = []
        for si in range(2):
            hdy = torch.empty((int(noff[-1]),), dtype=torch.float16).pin_memory()
            for li, lay in enumerate(w.layers):
                hdy[noff[li]:noff[li + 1]] = torch.from_numpy(
                    synth.make_x(batch, lay.N, seed=7 + si, layer=li)).reshape(-1)
            hdx = torch.empty((int(koff[-1]),), dtype=torch.float16).pin_memory()
            ddy, ddx = torch.empty_like(hdy, device=dev), torch.empty_like(hdx, device=dev)
            vdy = [ddy[noff[li]:noff[li + 1]].view(batch, lay.N) for li, lay in enumerate(w.layers)]
            vdx = [ddx[koff[li]:koff[li + 1]].view(batch, lay.K) for li, lay in enumerate(w.layers)]
            sets.append((hdy, hdx, ddy, ddx, vdy, vdx))

        def e2e_step(i):
            hdy, hdx, ddy, ddx, vdy, vdx = sets[i % 2]
            st = streams[i % 2]
            with torch.cuda.stream(st):
                ddy.copy_(hdy, non_blocking=True)
                for li in range(len(w.layers)):
                    L.input_grad(vdy[li], weights[i % pool][li], out=vdx[li], stream=st,
                                 schedule=schedule_of(a, native))
                hdx.copy_(ddx, non_blocking=True)

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        done1 = torch.cuda.Event()
        done1.record(streams[1])
        streams[0].wait_event(done1)
        e1.record(streams[0])
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": sflops * e2e_steps * world / (ems / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sets[0][0].numel() * 2, "d2h_bytes_per_step": sets[0][1].numel() * 2,
               "steps": e2e_steps, "us_per_layer": ems * 1e3 / (e2e_steps * len(w.layers)),
               "how": "per step: one pinned H2D copy of every layer's dy (packed), "
                      "weight_only_additive_b200.layer.input_grad -> aqlm_input_grad_ws per layer, one D2H "
                      "copy of every dx (packed); no CUDA graph; steps alternate between two streams with "
                      "their own host and device buffers, so one step's copies overlap the other's kernels"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        f, s, cols, threads = oracle_grad_sample_run(w, batch, a.cpu_seconds)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{cols} sampled columns of dx per layer (the oracle decodes the whole W16 each call, "
                         f"then fp64 dy . W16 for those columns), batch {batch}, {s:.1f} s on the host cores"}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        line = {"metric": GRAD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
                "warmup": a.warmup, "ms_per_step": ms_step, "us_per_layer": ms_step * 1e3 / len(w.layers),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
                "data": "synthetic",
                "config": grad_line_config(w, batch, world, a.schedule, pool, l2),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": len(w.layers) * steps, "clocks": clocks.summary(), "gpu": props.name}
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    a = parse_args(argv)
    if a.impl == "reference":
        return run_reference(a)
    if a.op == "input-grad":
        return run_input_grad(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
