#!/usr/bin/env python
"""Benchmark: NVFP4 4/6 quantize GB/s and fraction of B200 HBM bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fos|reference]

One step = one pass of the quantizer over the MoE expert workload
(128 x 2880 x 2880 bf16, per-expert N(0, 0.02^2) times U(0.5, 2)): the
per-expert amax and the 4/6 quantize to packed E2M1 codes + E4M3 scales +
FP32 per-expert scales, which the library runs as one fused kernel launch.  value = bytes / time with bytes = 2 (bf16 in) + 0.5
(codes) + 1/16 (scales) per element, summed over ranks (weak scaling: every
rank quantizes its own 128 experts).  Under torchrun one process per GPU;
rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

BYTES_PER_ELEM = 2 + 0.5 + 1 / 16           # one orientation, NVFP4
BYTES_PER_ELEM_DUAL = 2 + 2 * (0.5 + 1 / 16)  # two orientations from one read
BYTES_PER_ELEM_MX = 2 + 0.5 + 1 / 32
BYTES_PER_ELEM_DEQ = 0.5 + 1 / 16 + 2
WORKLOAD = "moe_experts_128x2880x2880_nvfp4_46_1x16_rne"
L2_BYTES = 126 * 1024 * 1024


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


def fp4_peak_tflops():
    """Dense FP4 tensor peak: the measured bf16 GEMM peak (burst) times the
    nominal FP4 : bf16 ratio of 4 (9 : 2.25 PFLOP/s dense); fallback 1590 TF/s
    bf16 when no measurement is present."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return 4.0 * float(d["bf16_tflops"]), "measured bf16_tflops x 4"
    return 4.0 * 1590.0, "fallback 1590 TF/s bf16 x 4"


# ------------------------------------------------------------------ dist
def relaunch_as_ranks(n: int) -> int:
    """Run this same command as n ranks, one process per GPU, under
    torch.distributed.run on this node (127.0.0.1); returns its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def dist_setup(n_gpus, dry_run=False):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%d" % (n_gpus, world))
    if world > 1:
        import datetime
        if dry_run:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        else:
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local))
    elif not dry_run:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.cmd = ["nvidia-smi", "-i", ident, "--query-gpu=timestamp," + self.FIELDS,
                        "--format=csv,noheader,nounits", "-lms", "50"]
        except Exception:
            self.cmd = None

    def start(self):
        if self.cmd is None:
            return
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self, busy_from=0):
        rows = []
        for l in self.lines[busy_from:]:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for r in rows:
            for name, v in zip(names[1:], r[3][1:]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ------------------------------------------------------------------ timing
def time_loop(fn, steps, warmup, world, stream):
    """Device time of `steps` calls of fn (CUDA events on `stream`), ms total."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world)


# ------------------------------------------------------------------ ncu traffic
# DRAM bytes per element of each kernel's committed ncu capture, with the
# source hash it was taken at (written beside the summaries in profiles/)
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


# The sources each profiled kernel is built from: a profile stays current
# while these files are unchanged.
KERNEL_SOURCES = {
    "k_q1x16_fused_moe_experts": ["csrc/fos_rowwise.cu", "csrc/fos_core.cuh", "csrc/fos_device.cuh",
                                  "csrc/fos_internal.h"],
}


def source_hash(kernel: str = "k_q1x16_fused_moe_experts") -> str:
    """SHA-256 over the sources `kernel` is built from (and the public header),
    to tell whether its profile is current."""
    import hashlib
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "mxfp4_block_scaled_fos_b200")
    files = [os.path.join(pkg, f) for f in KERNEL_SOURCES[kernel]] + [os.path.join(ROOT, "include", "fos.h")]
    for fn in files:
        with open(fn, "rb") as f:
            h.update(os.path.basename(fn).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def issue_bound(kernel, elems, ms, sm_mhz, sms=148):
    """The issue-slot roofline of `kernel` for a launch over `elems` elements
    taking `ms`: warp instructions per element from its ncu capture
    (profiles/traffic.json, smsp__inst_executed.sum over the captured
    elements), against 4 warp schedulers per SM each issuing one warp
    instruction per cycle at the sampled SM clock.  None if the sources
    changed since the capture."""
    try:
        with open(TRAFFIC_JSON) as f:
            d = json.load(f)[kernel]
        if d.get("source_sha256") != source_hash(kernel):
            return None
        wi = float(d["warp_instructions_per_element"]) * elems
    except (OSError, KeyError, ValueError, TypeError):
        return None
    slots_per_s = sms * 4 * sm_mhz * 1e6
    min_ms = wi / slots_per_s * 1e3
    return {"warp_instructions_per_launch": int(wi), "issue_slots_per_s": slots_per_s,
            "min_ms": round(min_ms, 4), "frac": round(min_ms / ms, 4)}


def profiled_traffic(kernel, elems):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json (its ncu
    capture's dram__bytes_read.sum + dram__bytes_write.sum per element,
    scaled to `elems`), or None if the sources changed since the capture."""
    try:
        with open(TRAFFIC_JSON) as f:
            d = json.load(f)[kernel]
        if d.get("source_sha256") != source_hash(kernel):
            return None
        return int(float(d["dram_bytes_per_element"]) * elems)
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ------------------------------------------------------------------ CPU baseline
def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_all_cores(entries, threads):
    """Wall time (s) of the oracle quantizing `entries` (per-entry amax +
    4/6 quantize) on `threads` host threads."""
    import oracle
    t0 = time.perf_counter()
    oracle.quantize_parallel(entries, threads)
    return time.perf_counter() - t0


def cpu_baseline(x_cpu_bits, budget_s=12.0):
    """The oracle as it stands on the host cores: all cores (threads over
    row chunks of whole experts) and, beside it, one thread."""
    import numpy as np
    import oracle
    oracle.lib()
    per = x_cpu_bits.shape[1] * x_cpu_bits.shape[2]
    cores = host_cores()
    entries = [np.ascontiguousarray(x_cpu_bits[e]) for e in range(x_cpu_bits.shape[0])]
    dt = oracle_all_cores(entries, cores)
    elems = len(entries) * per
    # single thread: whole experts until ~budget_s / 2
    done = 0
    t0 = time.perf_counter()
    while True:
        oracle.quantize(entries[done % len(entries)][None])
        done += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    dt1 = time.perf_counter() - t0
    return {"value": round(elems * BYTES_PER_ELEM / dt / 1e9, 6), "unit": "GB/s",
            "elems_per_s": round(elems / dt, 1), "cores": cores, "threads": cores, "kind": "oracle",
            "sample": "%d experts of 2880x2880 (%d elements), per-expert amax + 4/6 quantize, C oracle on "
                      "%d host threads (row chunks, GIL released)" % (len(entries), elems, cores),
            "single_thread": {"value": round(done * per * BYTES_PER_ELEM / dt1 / 1e9, 6), "unit": "GB/s",
                              "sample": "%d expert(s), one thread" % done}}


# ------------------------------------------------------------------ main arms
def run_fos(args, world, rank):
    import mxfp4_block_scaled_fos_b200 as F
    from mxfp4_block_scaled_fos_b200 import workloads

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    E, R, C = 128, 2880, 2880
    x = workloads.moe_experts(E, R, C, device=dev, seed=rank)
    elems = x.numel()
    row = F.quantize(x)[0]  # allocate outputs once
    ws = torch.empty(F.workspace_size(E, R, C), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    launches_per_step = 1  # the fused amax + quantize kernel (plus a 1.5 KB memset)

    def step():
        F.quantize(x, out_row=row, workspace=ws, status=status)

    clk = ClockSampler(torch.cuda.current_device())
    clk.start()
    time.sleep(0.15)
    t_ms = time_loop(step, args.steps, args.warmup, world, stream)
    clk.stop()

    # the step's only kernel is the fused one: its duration is the step time
    ms_per_step = t_ms / args.steps
    peak, peak_kind = measured_peaks()
    achieved = elems * BYTES_PER_ELEM / (ms_per_step * 1e-3) / 1e9
    # context: the quantize kernel alone with the amaxes supplied, and the amax pass
    amax = F.amax(x)
    k_steps = max(args.steps, 20)
    tq_ms = time_loop(lambda: F.quantize(x, out_row=row, amax=amax, status=status), k_steps, 3,
                      world, stream) / k_steps
    ta_ms = time_loop(lambda: F.amax(x, out=amax), k_steps, 3, world, stream) / k_steps

    extra = {}
    if not args.no_modes:
        extra = measure_modes(args, world, x, dev, stream, peak)

    # end to end through the public API with host buffers
    e2e = measure_e2e(args, world, x, row, ws, status, stream)
    assert int(status.item()) == 0, "non-finite input reported"

    value = world * elems * BYTES_PER_ELEM / (ms_per_step * 1e-3) / 1e9
    clocks = clk.summary()
    out = {
        "metric": "NVFP4 4/6 quantize GB/s and % of B200 HBM peak (bf16 in, FP4+E4M3 out)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "frac_of_hbm": round(value / world / peak, 4),
        "config": {"workload": WORKLOAD, "batch": E, "rows": R, "cols": C,
                   "formats": "bf16 in; E2M1 codes, E4M3 block scales, f32 tensor scales out",
                   "elements_per_gpu": elems, "bytes_per_elem": BYTES_PER_ELEM,
                   "amax": "computed in-step (per expert)", "parallelism": "dp%d" % world,
                   "l2": "input %.2f GB > 126 MB L2; no flush needed" % (2 * elems / 1e9)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic("k_q1x16_fused_moe_experts", elems),
                     "kernel": "k_q1x16_fused<4/6, RNE> (per-expert amax + quantize, one persistent launch)",
                     "kernel_ms": round(ms_per_step, 4),
                     "bytes_per_launch": int(elems * BYTES_PER_ELEM),
                     "quantize_only_ms": round(tq_ms, 4),
                     "quantize_only_GB_s": round(elems * BYTES_PER_ELEM / (tq_ms * 1e-3) / 1e9, 1),
                     "amax_pass_ms": round(ta_ms, 4),
                     "peak_source": "%s hbm_gbs (copy, read+write)" % peak_kind,
                     # the two ways of counting the step's bytes: (i) amax
                     # supplied, 2.5625 B/element; (ii) amax in the step,
                     # whose algorithm reads the input twice, 4.5625 B/element
                     # (this launch reads it about once from DRAM: traffic)
                     "mode_i_amax_supplied": {
                         "ms": round(tq_ms, 4),
                         "GB_s": round(elems * BYTES_PER_ELEM / (tq_ms * 1e-3) / 1e9, 1),
                         "frac": round(elems * BYTES_PER_ELEM / (tq_ms * 1e-3) / 1e9 / peak, 4),
                         "frac_of_8tbs_spec": round(elems * BYTES_PER_ELEM / (tq_ms * 1e-3) / 8e12, 4)},
                     "mode_ii_amax_in_step": {
                         "ms": round(ms_per_step, 4),
                         "bytes_per_elem": BYTES_PER_ELEM + 2.0,
                         "GB_s": round(elems * (BYTES_PER_ELEM + 2.0) / (ms_per_step * 1e-3) / 1e9, 1),
                         "frac": round(elems * (BYTES_PER_ELEM + 2.0) / (ms_per_step * 1e-3) / 1e9 / peak, 4)},
                     "frac_of_8tbs_spec": round(achieved / 8000.0, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clocks,
        "modes": extra,
    }
    issue = issue_bound("k_q1x16_fused_moe_experts", elems, ms_per_step,
                        clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0)
    if issue is not None:
        out["roofline"]["issue"] = issue
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_cpu = max(4, min(E, host_cores()))
        xs = workloads.bits(x[:n_cpu])
        out["cpu_baseline"] = cpu_baseline(xs, budget_s=args.cpu_seconds)
    return out


def measure_modes(args, world, x, dev, stream, peak):
    """Every other mode of the hot path at its workload (context, not the
    headline).  Full steps include the amax pass; "kernel" lines give the
    quantize kernel alone with the amax supplied.  Inputs that fit in L2 are
    rotated over copies whose total exceeds L2."""
    import mxfp4_block_scaled_fos_b200 as F
    from mxfp4_block_scaled_fos_b200 import workloads
    res = {}
    n = max(5, min(args.steps, 20))
    elems = x.numel()

    def rec(name, ms, bpe, n_elems, note=""):
        gbs = n_elems * bpe / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "GB_s": round(gbs, 1), "frac": round(gbs / peak, 4),
                     "bytes_per_elem": bpe, "elements": n_elems}
        if note:
            res[name]["note"] = note

    def rotating(xs, fn, reps):
        it = [0]

        def f():
            i = it[0] % len(xs)
            it[0] += 1
            fn(i)
        return time_loop(f, reps * len(xs), len(xs), world, stream) / (reps * len(xs))

    # MoE experts: 6-only, MXFP4 and the dequantizers
    try:
        ws = torch.empty(F.workspace_size(x.shape[0], x.shape[1], x.shape[2]), dtype=torch.uint8, device=dev)
        r6 = F.quantize(x, fmt="nvfp4_6")[0]
        ms = time_loop(lambda: F.quantize(x, fmt="nvfp4_6", out_row=r6, workspace=ws), n, 3, world, stream) / n
        rec("moe_nvfp4_6only_step", ms, BYTES_PER_ELEM, elems, "per-expert amax in the step (fused)")
        a6 = F.amax(x)
        ms = time_loop(lambda: F.quantize(x, fmt="nvfp4_6", out_row=r6, amax=a6), n, 3, world, stream) / n
        rec("moe_nvfp4_6only_kernel", ms, BYTES_PER_ELEM, elems, "amax supplied")
        rm = F.quantize(x, fmt="mxfp4")[0]
        ms = time_loop(lambda: F.quantize(x, fmt="mxfp4", out_row=rm), n, 3, world, stream) / n
        rec("moe_mxfp4_step", ms, BYTES_PER_ELEM_MX, elems)
        r46 = F.quantize(x)[0]
        y = torch.empty_like(x)
        ms = time_loop(lambda: F.dequantize(r46, out=y), n, 3, world, stream) / n
        rec("moe_nvfp4_dequant", ms, BYTES_PER_ELEM_DEQ, elems)
        ms = time_loop(lambda: F.dequantize(rm, out=y), n, 3, world, stream) / n
        rec("moe_mxfp4_dequant", ms, 0.5 + 1 / 32 + 2, elems)
        ms = time_loop(lambda: F.fake_quantize(x, out=y, workspace=ws), n, 3, world, stream) / n
        rec("moe_nvfp4_46_fake_quant_step", ms, 4.0, elems,
            "quantize + dequantize in one launch, bf16 in and out, per-expert amax in the step")
        del y, r6, rm, r46
    except Exception as e:  # report, do not hide
        res["moe_error"] = repr(e)
    torch.cuda.empty_cache()
    # activations 8192x4096, 1% outlier channels, RHT16, 4/6: 4 rotating copies (256 MiB)
    try:
        xs = [workloads.activation_outliers(8192, 4096, device=dev, seed=s) for s in range(4)]
        outs = [F.quantize(t, rht=True)[0] for t in xs]
        wss = [torch.empty(F.workspace_size(1, 8192, 4096), dtype=torch.uint8, device=dev) for _ in xs]
        ms = rotating(xs, lambda i: F.quantize(xs[i], rht=True, out_row=outs[i], workspace=wss[i]), n)
        rec("activation_rht16_step", ms, BYTES_PER_ELEM, xs[0].numel(), "amax in the step; 4 rotating copies")
        am = [F.amax(t, rht=True) for t in xs]
        ms = rotating(xs, lambda i: F.quantize(xs[i], rht=True, out_row=outs[i], amax=am[i]), n)
        rec("activation_rht16_kernel", ms, BYTES_PER_ELEM, xs[0].numel(), "amax supplied; 4 rotating copies")
        del xs, outs, am
    except Exception as e:
        res["activation_error"] = repr(e)
    torch.cuda.empty_cache()
    # weights 14336x4096 N(0, 0.02^2), 16x16 2D 4/6 with the transposed copy: 2 rotating copies
    try:
        xs = [workloads.weight_normal(14336, 4096, device=dev, seed=s) for s in range(2)]
        outs = [F.quantize(t, block="16x16", colwise=True) for t in xs]
        ms = rotating(xs, lambda i: F.quantize(xs[i], block="16x16", colwise=True, out_row=outs[i][0],
                                               out_col=outs[i][1]), n)
        rec("weight_2d_both_step", ms, BYTES_PER_ELEM_DUAL, xs[0].numel(), "amax in the step; 2 rotating copies")
        am = [F.amax(t) for t in xs]
        ms = rotating(xs, lambda i: F.quantize(xs[i], block="16x16", colwise=True, amax=am[i],
                                               out_row=outs[i][0], out_col=outs[i][1]), n)
        rec("weight_2d_both_kernel", ms, BYTES_PER_ELEM_DUAL, xs[0].numel(), "amax supplied")
        del xs, outs, am
    except Exception as e:
        res["weight_error"] = repr(e)
    torch.cuda.empty_cache()
    # gradients 16384x8192 Student-t(3)*1e-3, SR, rowwise + colwise (256 MiB > L2)
    try:
        g = workloads.gradient_student_t(16384, 8192, device=dev)
        r, c = F.quantize(g, rounding="sr", colwise=True)
        ms = time_loop(lambda: F.quantize(g, rounding="sr", colwise=True, out_row=r, out_col=c), n, 3,
                       world, stream) / n
        rec("gradient_sr_dual_step", ms, BYTES_PER_ELEM_DUAL, g.numel(), "amax in the step")
        am = F.amax(g)
        ms = time_loop(lambda: F.quantize(g, rounding="sr", colwise=True, amax=am, out_row=r, out_col=c),
                       n, 3, world, stream) / n
        rec("gradient_sr_dual_kernel", ms, BYTES_PER_ELEM_DUAL, g.numel(), "amax supplied")
        r1 = F.quantize(g, rounding="sr")[0]
        ms = time_loop(lambda: F.quantize(g, rounding="sr", amax=am, out_row=r1), n, 3, world, stream) / n
        rec("gradient_sr_rowwise_kernel", ms, BYTES_PER_ELEM, g.numel(), "amax supplied")
        rt, ct = F.quantize(g, rounding="sr", colwise=True, rht_col=True)
        wst = torch.empty(F.workspace_size(1, g.shape[-2], g.shape[-1]), dtype=torch.uint8, device=dev)
        ms = time_loop(lambda: F.quantize(g, rounding="sr", colwise=True, rht_col=True, amax=am, out_row=rt,
                                          out_col=ct, workspace=wst), n, 3, world, stream) / n
        rec("gradient_sr_dual_colwise_rht_step", ms, BYTES_PER_ELEM_DUAL, g.numel(),
            "rowwise amax supplied; the colwise copy transformed along M with its own amax in the step")
        del rt, ct, wst
        del g, r, c, r1
    except Exception as e:
        res["gradient_error"] = repr(e)
    torch.cuda.empty_cache()
    # NVFP4 block-scaled GEMM on the tensor cores, fed by the quantizer
    try:
        peak_tf, peak_src = fp4_peak_tflops()
        for n_ in (4096, 8192):
            g_ = torch.Generator(device=dev).manual_seed(0)
            xa = torch.randn(n_, n_, generator=g_, device=dev).to(torch.bfloat16)
            xb = torch.randn(n_, n_, generator=g_, device=dev).to(torch.bfloat16)
            qa = F.quantize(xa, swizzle=True, choice=False)[0]
            qb = F.quantize(xb, swizzle=True, choice=False)[0]
            d_ = torch.empty(n_, n_, dtype=torch.bfloat16, device=dev)
            ws_ = torch.empty(F.gemm_workspace_size(n_, n_, n_), dtype=torch.uint8, device=dev)
            ms = time_loop(lambda: F.gemm_nvfp4(qa, qb, out=d_, workspace=ws_), n, 3, world, stream) / n
            tf = 2.0 * n_ ** 3 / (ms * 1e-3) / 1e12
            res["gemm_nvfp4_%d" % n_] = {"ms": round(ms, 4), "TFLOP_s": round(tf, 1),
                                         "frac": round(tf / peak_tf, 4), "peak_TFLOP_s": peak_tf,
                                         "peak_source": peak_src, "shape": [n_, n_, n_],
                                         "note": "bf16 out, 128x256 tiles, kind::mxf4nvf4; both operands' "
                                                 "scales rewritten into the wide copy layout inside the timed call"}
            del xa, xb, qa, qb, d_, ws_
    except Exception as e:
        res["gemm_error"] = repr(e)
    torch.cuda.empty_cache()
    # a quantized Linear layer, 8192 tokens x 4096 -> 4096: the forward GEMM,
    # then dgrad and wgrad, with every operand quantized inside the step
    # (x 1x16 rowwise and along M, dy with SR in both orientations); the 2D
    # weight quantization is done once, outside the step
    try:
        peak_tf, peak_src = fp4_peak_tflops()
        M_, N_, K_ = 8192, 4096, 4096
        xl = workloads.activation_outliers(M_, K_, device=dev)[0]
        wl = workloads.weight_normal(N_, K_, device=dev)[0]
        dyl = workloads.gradient_student_t(M_, N_, device=dev)[0]
        qw = F.quantize_weight(wl)

        def layer_step():
            _, qx_t = F.linear_forward(xl, qw, save_colwise=True, seed=7)
            F.linear_backward(dyl, None, qw, seed=7, qx_t=qx_t)

        ms = time_loop(layer_step, n, 3, world, stream) / n
        tf = 3 * 2.0 * M_ * N_ * K_ / (ms * 1e-3) / 1e12
        res["linear_layer_fwd_bwd"] = {"ms": round(ms, 4), "TFLOP_s": round(tf, 1),
                                       "frac": round(tf / peak_tf, 4), "peak_TFLOP_s": peak_tf,
                                       "peak_source": peak_src, "shape": [M_, N_, K_],
                                       "note": "3 GEMMs (forward, dgrad, wgrad) + the quantization of "
                                               "x (both orientations, from one read in the forward) and dy "
                                               "(SR, both orientations) per step; f32 gradients, bf16 y"}
        del xl, wl, dyl, qw
    except Exception as e:
        res["linear_error"] = repr(e)
    torch.cuda.empty_cache()
    return res


def run_rows(args, world, rank):
    """--split rows: one tensor of world x 16384 rows x 8192 cols (Student-t
    gradients), each rank holding its 16384 rows.  One step = the local
    per-tensor amax, an all-reduce(MAX) of it over the ranks (NCCL), and the
    4/6 1x16 rowwise quantize of the local rows with the global amax."""
    import mxfp4_block_scaled_fos_b200 as F
    from mxfp4_block_scaled_fos_b200 import shard, workloads
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    R, C = 16384, 8192
    x = workloads.gradient_student_t(R, C, device=dev, seed=rank)
    row0 = rank * R
    out = F.quantize(x, amax=F.amax(x))[0]
    amax = torch.empty(1, dtype=torch.float32, device=dev)

    def step():
        F.amax(x, out=amax)
        shard.global_amax(amax)
        F.quantize(x, amax=amax, elem_offset=row0 * C, out_row=out)

    clk = ClockSampler(torch.cuda.current_device())
    clk.start()
    t_ms = time_loop(step, args.steps, args.warmup, world, stream)
    clk.stop()
    ms = t_ms / args.steps
    peak, peak_kind = measured_peaks()
    elems = x.numel()
    value = world * elems * BYTES_PER_ELEM / (ms * 1e-3) / 1e9
    return {"metric": "NVFP4 4/6 quantize GB/s and % of B200 HBM peak (bf16 in, FP4+E4M3 out)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "gradient_student_t_rows_split_%dx16384x8192_nvfp4_46_1x16_rne" % world,
                       "rows_per_gpu": R, "cols": C, "collective": "all_reduce(MAX) of 1 float per step",
                       "parallelism": "rows%d" % world},
            "frac_of_hbm": round(value / world / peak, 4),
            "gpu_launches": 2 * args.steps, "clocks": clk.summary(),
            "peak_source": "%s hbm_gbs" % peak_kind}


def measure_e2e(args, world, x, row, ws, status, stream):
    """Same metric through the C-ABI call with pinned host buffers
    (fos_quantize_host, bound as host.HostQuantizer): every step copies the
    input in, quantizes it (per-expert amax + 4/6) and copies codes, scales
    and S_t back, in chunks of 4 experts pipelined over three streams, so
    that the copies in both directions and the kernels overlap."""
    from mxfp4_block_scaled_fos_b200.host import HostQuantizer
    batch, rows, cols = x.shape
    hq = HostQuantizer(batch, rows, cols, chunk=4, device=x.device)
    h_in = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h_in.copy_(x)
    h_codes, h_scales, h_ts = hq.host_outputs()

    def step():
        hq(h_in, h_codes, h_scales, h_ts)

    n = max(3, min(args.steps, 5))
    ms = time_loop(step, n, 1, world, stream) / n
    elems = x.numel()
    h2d = x.numel() * 2
    d2h = h_codes.numel() + h_scales.numel() + 4 * h_ts.numel()
    return {"value": round(world * elems * BYTES_PER_ELEM / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": "chunks of 4 experts: host-to-device copy, quantize and device-to-host copy "
                        "of successive chunks overlap on three streams"}


def run_reference(args, world, rank):
    """The oracle on the host cores, one expert of the workload per step
    (its rows split over all host threads)."""
    import oracle
    from mxfp4_block_scaled_fos_b200 import workloads
    if rank != 0:
        return None
    x = workloads.moe_experts(1, 2880, 2880, device="cpu", seed=0)
    xb = workloads.bits(x)[0]
    oracle.lib()
    cores = host_cores()
    for _ in range(args.warmup):
        oracle_all_cores([xb], cores)
    dt = 0.0
    for _ in range(args.steps):
        dt += oracle_all_cores([xb], cores)
    elems = xb.size * args.steps
    v = elems * BYTES_PER_ELEM / dt / 1e9
    sample = ("one 2880x2880 expert per step (per-expert amax + 4/6 quantize), C oracle on %d host "
              "threads over row chunks" % cores)
    return {"impl": "reference", "metric": "NVFP4 4/6 quantize GB/s and % of B200 HBM peak "
            "(bf16 in, FP4+E4M3 out)", "value": round(v, 6), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": "1 of 128 experts per step"},
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "kind": "oracle", "cores": cores,
                             "threads": cores, "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_dry(args, world, rank):
    """--dry-run: the launch and rank plumbing only, no GPU work."""
    sys.stderr.write("bench dry run: rank %d of %d\n" % (rank, world))
    if world > 1:
        t = torch.tensor([1.0])
        torch.distributed.all_reduce(t)
        assert int(t.item()) == world
    return {"metric": "dry run", "value": 0.0, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "dry_run": True, "world_size_env": int(os.environ.get("WORLD_SIZE", "1"))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fos", "reference"], default="fos")
    ap.add_argument("--no-modes", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--split", choices=["entries", "rows"], default="entries",
                    help="entries: each rank quantizes its own 128 experts (no collective); rows: each "
                         "rank quantizes its rows of one tensor after an amax all-reduce")
    ap.add_argument("--dry-run", action="store_true", help="launch the ranks and exit (no GPU work)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch_as_ranks(args.gpus))
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, _ = dist_setup(args.gpus, args.dry_run)
    if args.dry_run:
        out = run_dry(args, world, rank)
    else:
        from mxfp4_block_scaled_fos_b200 import build as fbuild
        if rank == 0:
            fbuild.build()
        barrier(world)
        out = run_rows(args, world, rank) if args.split == "rows" else run_fos(args, world, rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
