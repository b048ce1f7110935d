#!/usr/bin/env python
"""Benchmark of the fused norm + activation-quantization hot path on B200.

Metric: achieved HBM bandwidth of the fused norm + quantization calls (GB/s,
and as a fraction of the measured device copy bandwidth), with µs per call and
tokens/s, for M = 1 ... 65536 tokens.  Bytes are algorithmic: every input read
once, every output written once, gamma / beta / scales once per call.

Headline workload (one "step" = one call over one batch): fused residual-add +
RMSNorm + dynamic per-token e4m3 (division quantization, eps 1e-6) at
M = 65536 tokens x d = 8192, the largest cell of the sweep configuration: bf16
x ~ N(0, 1) with four channels scaled x100 (activation outliers), residual
~ N(0, 1), gamma = 1 + 0.1 N(0, 1); residual_out is written to its own buffer so
the inputs stay the same from step to step.  One call moves 3.76 GB, far more
than the 126 MB L2, so no step finds its inputs in L2.  W untimed warm-up
calls, then exactly K timed calls bracketed by CUDA events on the launching
stream (with a barrier and a device synchronize on both sides); each call's
own duration comes from events between calls, for the roofline.  Multi-GPU
runs (torchrun, one process per GPU) give every rank the same per-GPU workload
(weak scaling, no data-path collective); the time is the max over ranks.

Every default run also times each configuration's cells ("configs" in the
JSON line): the sweep (d in {2816, 4096, 7168, 8192} x M in {1, 16, 256, 4096,
65536}), the small dynamic case (64 x 2816), the static RMSNorm and LayerNorm
calls (4096 x 4096), per-token-group FP8 (32768 x 4096 and M = 1, fp32 and
UE8M0 scales) and NVFP4 (d in {7168, 1536 of a [M, 2112] tensor, 512} x M in
{1, 64, 8192}, with and without residual), plus the fused RMSNorm + group FP8
and MoE-dispatch calls.  A cell is timed as CUDA graphs of S launches over S
rotating input / output sets (S x bytes >= 3 x L2 where that fits), launched
with programmatic dependent launch; each graph is replayed once before its
timed replays.  Cells of M <= 64 also give the median host-to-completion
latency of one call through the Python API (``host_latency_us``).

``e2e`` is the headline measured through the Python API with the inputs in
pinned host memory: per step the host -> device copy of x and residual, the
call, and the device -> host copy of q, the scales and residual_out, pipelined
over two buffer sets on three streams.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead, on a bounded sample of the headline workload per step.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused norm+quant HBM GB/s (% of B200 peak) and µs/call, M=1..65536"
HEAD_M, HEAD_D, HEAD_EPS = 65536, 8192, 1e-6
HEAD_WORKLOAD = ("fused residual-add + RMSNorm + dynamic per-token e4m3 (division), "
                 "M=65536 tokens x d=8192, x with 4 channels x100")
HEAD_KERNEL = "nq_fused_add_rmsnorm_quant_fp8"
STATIC_SCALE, STATIC_EPS = 0.05, 1e-5
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


# ------------------------------------------------- algorithmic bytes ----
def fused_dyn_bytes(M, d):
    return M * (7 * d + 4) + 2 * d         # x, residual read; residual, e4m3, scale write; gamma


def rms_static_bytes(M, d):
    return M * 3 * d + 2 * d + 4           # x read, e4m3 write; bf16 gamma; scale


def ln_static_bytes(M, d):
    return M * 3 * d + 8 * d + 4           # x read, e4m3 write; fp32 gamma + beta; scale


def group_bytes(M, K, g=128):
    return M * (3 * K + 4 * (K // g))      # x read, e4m3 + fp32 scales write


def rms_group_bytes(M, d, residual, g=128):
    # x (+ residual read and write) bf16, e4m3 write, fp32 group scales; bf16 gamma
    return M * ((6 * d if residual else 2 * d) + d + 4 * (d // g)) + 2 * d


def moe_bytes(M, d, topk, group, residual=True):
    # x (+ residual read and write) bf16, topk copies of the e4m3 row and its scales, dest; bf16 gamma
    per_scale = 4 if group == 0 else 4 * (d // group)
    return M * ((6 * d if residual else 2 * d) + topk * (d + per_scale + 4)) + 2 * d


def nvfp4_bytes(M, d, residual):
    per = (6 * d if residual else 2 * d) + d // 2 + d // 16
    return M * per + 2 * d + 4


def _strip_comments(src: str) -> str:
    """C/C++ source without // and /* */ comments (string literals left alone)."""
    return re.sub(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"',
                  lambda m: m.group(0) if m.group(0).startswith('"') else "", src, flags=re.S)


HEAD_KERNEL_SOURCES = ("nq_row_rms_dyn.cu", "nq_row_kernel.cuh", "nq_device.cuh", "nq_internal.h")


def kernel_source_hash() -> str:
    """Hash of the headline kernel's device code (its translation unit and the
    headers it includes, comments stripped and whitespace collapsed): the
    headline profile's counters stay valid while it matches."""
    h = hashlib.sha256()
    for name in HEAD_KERNEL_SOURCES:
        p = os.path.join(ROOT, "fp4_activation_quantization_b200", "csrc", name)
        with open(p, encoding="utf-8") as f:
            h.update(os.path.basename(p).encode())
            h.update(" ".join(_strip_comments(f.read()).split()).encode())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(kernel_tag: str):
    """DRAM bytes read and written per launch of the headline kernel, from a
    committed ncu summary of the same workload, if that summary was taken on the
    current kernel sources (else None)."""
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(p).read()
        tag = re.search(r"^bench_kernel:\s*(\S+)", text, re.M)
        rd = re.search(r"^dram_read_bytes_per_launch:\s*(\d+)", text, re.M)
        wr = re.search(r"^dram_write_bytes_per_launch:\s*(\d+)", text, re.M)
        hs = re.search(r"^kernel_source_hash:\s*(\S+)", text, re.M)
        if tag and rd and wr and hs and tag.group(1) == kernel_tag:
            if hs.group(1) != kernel_source_hash():
                return None
            return {"read": int(rd.group(1)), "write": int(wr.group(1)), "source": os.path.relpath(p, ROOT)}
    return None


# ----------------------------------------------------------- clocks ----
class ClockSampler:
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str, interval_ms: int = 50):
        self.gpu_id, self.interval_ms = gpu_id, interval_ms
        self.lines, self.proc, self.err = [], None, None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-i", self.gpu_id, "-lms", str(self.interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception as e:  # no nvidia-smi: report it
            self.err = str(e)

    def _read(self):
        for line in self.proc.stdout:
            line = line.strip()
            ts = time.time()
            try:  # the sample's own timestamp (the pipe may deliver lines late)
                ts = datetime.datetime.strptime(line.split(",")[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                pass
            self.lines.append((ts, line))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self, t0: float, t1: float):
        if self.err or not self.lines:
            return {"error": self.err or "no samples"}
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed_region"
        if len(inside) < 3:
            inside = [r for r in rows if t0 - 0.5 <= r[0] <= t1 + 0.5]
            window = "timed_region_pm_0.5s"
        if not inside:
            return {"error": "no samples in window", "samples": len(rows)}
        sm = sorted(r[1] for r in inside)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for name, val in zip(names, r[3][1:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


def gpu_id_for(dev_index: int) -> str:
    import torch
    props = torch.cuda.get_device_properties(dev_index)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        s = str(uuid)
        return s if s.startswith("GPU-") else f"GPU-{s}"
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[dev_index]
    return str(dev_index)


# ------------------------------------------------------- distributed ----
def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    """Largest value over the ranks (host plumbing: one float, on the process group's device)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, step_bytes: int, elapsed_ms: float) -> float:
    """Whole-job GB/s: every rank processed `steps` steps of `step_bytes` (weak scaling)
    in at most `elapsed_ms` (the max over ranks)."""
    return world * steps * step_bytes / (elapsed_ms * 1e-3) / 1e9


# ------------------------------------------------------- GPU inputs ----
def outlier_x(M, d, gen, scale=100.0):
    """bf16 x ~ N(0, 1) with the sweep's four outlier channels scaled (device-seeded)."""
    import torch
    import synthetic as S
    x = torch.randn(M, d, device="cuda", generator=gen)
    for c in S.outlier_channels(d):
        x[:, c] *= scale
    return x.to(torch.bfloat16)


class Headline:
    """The headline call's device buffers (one set: every call moves more than L2)."""

    def __init__(self, nq, M, d, seed):
        import torch
        gen = torch.Generator(device="cuda").manual_seed(seed)
        self.nq, self.M, self.d = nq, M, d
        self.x = outlier_x(M, d, gen)
        self.res = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
        self.gamma = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(torch.bfloat16)
        self.res_out = torch.empty_like(self.res)
        self.q = torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda")
        self.s = torch.empty(M, dtype=torch.float32, device="cuda")

    def call(self, flags=0, stream=None):
        self.nq.nq_fused_add_rmsnorm_quant_fp8(self.x, self.res, self.gamma, HEAD_EPS, residual_out=self.res_out,
                                               q_out=self.q, scale_out=self.s, flags=flags, stream=stream)


def run_gpu_arm(args):
    import torch
    import fp4_activation_quantization_b200 as nq

    world, rank, local = dist_setup(args.gpus)
    M, d = HEAD_M, HEAD_D
    flags = 0 if args.no_pdl else nq.FLAG_PDL
    hl = Headline(nq, M, d, seed=1234 + rank)
    K, W = args.steps, max(3, args.warmup)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()

    # warm-up: exactly W calls, the same launches as the timed region
    with torch.cuda.stream(stream):
        for _ in range(W):
            hl.call(flags)
    torch.cuda.synchronize()

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    sampler = ClockSampler(gpu_id_for(torch.cuda.current_device()))
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        ev[0].record()
        for i in range(K):
            hl.call(flags)
            ev[i + 1].record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    time.sleep(0.15)
    sampler.stop()

    per_call_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    elapsed_ms = max_over_ranks(world, ev[0].elapsed_time(ev[K]))
    step_bytes = fused_dyn_bytes(M, d)
    value = job_throughput(world, K, step_bytes, elapsed_ms)
    peak, peak_src = measured_peak()
    call_us = sum(per_call_ms) * 1e3 / K
    achieved = step_bytes / (call_us * 1e-6) / 1e9
    clocks = sampler.summary(t0, t1)

    e2e = None if args.no_e2e else run_e2e(nq, hl, world, min(K, args.e2e_steps), flags)

    configs = run_configs(nq, flags) if rank == 0 and not args.no_configs else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    if world > 1:
        import torch.distributed as dist
        barrier(world)  # every rank waits for rank 0's configuration cells before leaving the group
        dist.destroy_process_group()

    if rank != 0:
        return
    traffic = profiled_traffic(HEAD_KERNEL)
    out = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(elapsed_ms / K, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (device-seeded: x bf16 N(0,1) with 4 channels x100; residual bf16 N(0,1); "
                "gamma bf16 1+0.1N)",
        "config": {"workload": HEAD_WORKLOAD, "M": M, "d": d, "eps": HEAD_EPS,
                   "io": "bf16 x, residual, gamma in; bf16 residual_out, e4m3 codes, fp32 scales out; fp32 math",
                   "l2": f"inputs larger than L2 ({2 * M * d * 2 / 2**30:.1f} GiB read per call, L2 126 MB)",
                   "launch": "one launch per step, CUDA events between launches",
                   "pdl": not args.no_pdl,
                   "parallelism": f"replicas x{world} (rows shard, no collective)"},
        "per_call": {HEAD_KERNEL: {"us": round(call_us, 3), "GBps": round(achieved, 1),
                                   "tokens_per_s": round(M / (call_us * 1e-6), 1)}},
        "roofline": {"bound": "hbm", "kernel": HEAD_KERNEL, "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": peak_src, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_nominal_8000": round(achieved / NOMINAL_HBM_GBS, 4),
                     "algorithmic_bytes_per_launch": step_bytes,
                     "traffic": None if traffic is None else traffic["read"] + traffic["write"],
                     "traffic_read": None if traffic is None else traffic["read"],
                     "traffic_write": None if traffic is None else traffic["write"],
                     "traffic_source": None if traffic is None else traffic["source"]},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": K,
        "clocks": clocks,
        "kernel_source_hash": kernel_source_hash(),
    }
    if configs is not None:
        out["configs"] = configs
    print(json.dumps(out), flush=True)


def run_e2e(nq, hl, world, steps, flags):
    """The headline through the public API with host buffers: H2D of x and the
    residual, the call, D2H of q, the scales and residual_out, pipelined over two
    device buffer sets (copy-in, compute and copy-out streams)."""
    import torch
    M, d = hl.M, hl.d
    xh = hl.x.cpu().pin_memory()
    rh = hl.res.cpu().pin_memory()
    qh = torch.empty(M, d, dtype=torch.float8_e4m3fn).pin_memory()
    sh = torch.empty(M, dtype=torch.float32).pin_memory()
    roh = torch.empty(M, d, dtype=torch.bfloat16).pin_memory()
    sets = [dict(x=torch.empty_like(hl.x), r=torch.empty_like(hl.res), q=torch.empty_like(hl.q),
                 s=torch.empty_like(hl.s), ro=torch.empty_like(hl.res_out)) for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i & 1
        B = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])      # the call of step i - 2 has read this set's inputs
            B["x"].copy_(xh, non_blocking=True)
            B["r"].copy_(rh, non_blocking=True)
            ev_in[b].record()
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])     # step i - 2's outputs have left this set
            nq.nq_fused_add_rmsnorm_quant_fp8(B["x"], B["r"], hl.gamma, HEAD_EPS, residual_out=B["ro"],
                                              q_out=B["q"], scale_out=B["s"], flags=flags)
            ev_comp[b].record()
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            qh.copy_(B["q"], non_blocking=True)
            sh.copy_(B["s"], non_blocking=True)
            roh.copy_(B["ro"], non_blocking=True)
            ev_out[b].record()

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s_in):
        a.record()
    for i in range(steps):
        step(i)
    with torch.cuda.stream(s_out):
        b_.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, a.elapsed_time(b_))
    barrier(world)
    return {"value": round(job_throughput(world, steps, fused_dyn_bytes(M, d), e2e_ms), 3), "unit": "GB/s",
            "h2d_bytes_per_step": 2 * M * d * 2, "d2h_bytes_per_step": M * d + 4 * M + 2 * M * d,
            "steps": steps, "ms_per_step": round(e2e_ms / steps, 4),
            "how": "pinned host buffers; H2D of x and residual, the call, D2H of codes, scales and residual_out "
                   "each step, pipelined over two device buffer sets on three streams"}


# ------------------------------------------------------ config cells ----
def time_calls(fn, n_sets, reps):
    """µs per call of fn(i) (i = set index), captured as one CUDA graph of n_sets
    launches; the graph is replayed once untimed, then reps times under events."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n_sets):
            fn(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n_sets):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * n_sets)
    del g
    return us


def sets_for(nbytes):
    """Rotating sets so that a set is reused only after >= 3 x L2 of other traffic (2 .. 16)."""
    return int(max(2, min(16, -(-3 * L2_BYTES // max(1, nbytes)))))


def reps_for(nbytes, n_sets):
    return max(3, min(200, int(4e8 // max(nbytes * n_sets, 1))))


def host_latency_us(fn, reps=50):
    """Median wall time of one call from the host to its completion (the Python API's
    call, the launch and a device synchronize): the latency a decode step sees."""
    import torch
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        fn(0)
        torch.cuda.synchronize()
        ts.append(time.perf_counter() - t0)
    ts.sort()
    return round(ts[len(ts) // 2] * 1e6, 2)


def cell(peak, tokens, nbytes, us, **kw):
    gbs = nbytes / us / 1e3
    return dict(kw, us=round(us, 3), GBps=round(gbs, 1), frac=round(gbs / peak, 4),
                tokens_per_s=round(tokens / (us * 1e-6), 1), bytes=nbytes)


def run_configs(nq, flags):
    """µs per call, GB/s, fraction of the measured copy bandwidth and tokens/s of
    every configuration's cells.  Cells of M >= 4096 also carry `copy_frac`: the
    fraction of the measured copy bandwidth that a device copy moving the same
    bytes reaches, timed the same way (the ceiling at that size for a kernel
    that only moves data).  The copy is torch's elementwise kernel dst = src * 1
    on bf16, an SM copy: a captured copy_ becomes a graph memcpy node, which ran
    at 0.42-0.46 of the measured bandwidth for some sizes (80 MB, 205 MB,
    1.3 GB) and 0.86-0.96 for others."""
    import torch
    import synthetic as S
    gen = torch.Generator(device="cuda").manual_seed(7)
    bf = torch.bfloat16
    peak, _ = measured_peak()
    out = {}
    copy_us = {}

    def with_copy(c):
        if c["M"] < 4096:
            return c
        nb = c["bytes"]
        if nb not in copy_us:
            nel = nb // 4  # bf16 elements each way: 2 bytes read and 2 written per element
            n = sets_for(nb)
            src = [torch.empty(nel, dtype=bf, device="cuda") for _ in range(n)]
            dst = [torch.empty(nel, dtype=bf, device="cuda") for _ in range(n)]
            copy_us[nb] = time_calls(lambda i: torch.mul(src[i], 1, out=dst[i]), n, reps_for(nb, n))
            del src, dst
        c["copy_frac"] = round(nb / copy_us[nb] / 1e3 / peak, 4)
        return c

    def dyn_cell(M, d, outliers):
        nb = fused_dyn_bytes(M, d)
        n = sets_for(nb)
        xs = [outlier_x(M, d, gen, 100.0 if outliers else 1.0) for _ in range(n)]
        rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)]
        ro = [torch.empty(M, d, dtype=bf, device="cuda") for _ in range(n)]
        qs = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
        ss = [torch.empty(M, dtype=torch.float32, device="cuda") for _ in range(n)]
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        fn = lambda i: nq.nq_fused_add_rmsnorm_quant_fp8(xs[i], rs[i], g, 1e-6, residual_out=ro[i], q_out=qs[i],
                                                         scale_out=ss[i], flags=flags)
        us = time_calls(fn, n, reps_for(nb, n))
        extra = {"host_latency_us": host_latency_us(fn)} if M <= 64 else {}
        c = cell(peak, M, nb, us, call="nq_fused_add_rmsnorm_quant_fp8", M=M, d=d, sets=n, **extra)
        del xs, rs, ro, qs, ss
        return with_copy(c)

    out["1_fused_dynamic_small"] = [dyn_cell(64, 2816, False)]
    out["5_fused_dynamic_sweep"] = [dyn_cell(M, d, True) for d in (2816, 4096, 7168, 8192)
                                    for M in (1, 16, 256, 4096, 65536)]

    # config 2: static RMSNorm and LayerNorm, 4096 x 4096, scale 0.05 in device memory, eps 1e-5
    M, d = 4096, 4096
    n = 8
    sc = torch.tensor([STATIC_SCALE], dtype=torch.float32, device="cuda")
    xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)]
    qs = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
    g_rms = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
    g_ln = 1 + 0.1 * torch.randn(d, device="cuda", generator=gen)
    b_ln = 0.02 * torch.randn(d, device="cuda", generator=gen)
    reps = 100
    us_rms = time_calls(lambda i: nq.nq_rmsnorm_quant_fp8_static(xs[i], g_rms, sc, STATIC_EPS, q_out=qs[i],
                                                                 flags=flags), n, reps)
    us_ln = time_calls(lambda i: nq.nq_layernorm_quant_fp8(xs[i], g_ln, b_ln, sc, STATIC_EPS, q_out=qs[i],
                                                           flags=flags), n, reps)
    out["2_static"] = [cell(peak, M, rms_static_bytes(M, d), us_rms, call="nq_rmsnorm_quant_fp8_static", M=M, d=d,
                            sets=n),
                       cell(peak, M, ln_static_bytes(M, d), us_ln, call="nq_layernorm_quant_fp8", M=M, d=d, sets=n)]
    # the same bytes moved by a device copy (reads 2 bytes and writes 1 per element, as a copy of
    # 2/3 of the bytes each way): the ceiling at this size for a kernel that only moves data
    nel = M * d * 3 // 4
    src = [torch.empty(nel, dtype=bf, device="cuda") for _ in range(n)]
    dst = [torch.empty(nel, dtype=bf, device="cuda") for _ in range(n)]
    us_cp = time_calls(lambda i: torch.mul(src[i], 1, out=dst[i]), n, reps)  # an SM copy (see with_copy)
    out["2_static"].append(cell(peak, M, 4 * nel, us_cp, call="device copy of the same bytes (context)",
                                elements=nel, sets=n))
    for c in out["2_static"][:2]:
        c["copy_frac"] = out["2_static"][2]["frac"]
    del xs, qs, src, dst

    rows = []
    for M in (32768, 1):
        K = 4096
        for fl, tag in ((0, "fp32"), (nq.FLAG_UE8M0, "ue8m0")):
            nb = group_bytes(M, K)
            n = sets_for(nb)
            xs = [torch.randn(M, K, device="cuda", generator=gen).to(bf) for _ in range(n)]
            for x in xs:  # 0.1 % of elements x50
                x.mul_(torch.where(torch.rand(M, K, device="cuda", generator=gen) < 1e-3, 50.0, 1.0).to(bf))
            qs = [torch.empty(M, K, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
            sc_ = [torch.empty(M, K // 128, dtype=torch.float32, device="cuda") for _ in range(n)]
            fn = lambda i: nq.nq_per_token_group_quant_fp8(xs[i], 128, q_out=qs[i], scales_out=sc_[i],
                                                           flags=fl | flags)
            us = time_calls(fn, n, reps_for(nb, n))
            extra = {"host_latency_us": host_latency_us(fn)} if M <= 64 else {}
            del xs, qs, sc_
            rows.append(with_copy(cell(peak, M, nb, us, call="nq_per_token_group_quant_fp8", scales=tag, M=M, K=K,
                                       sets=n, **extra)))
    out["3_group"] = rows

    rows = []
    gs = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    for d, ld in ((7168, 7168), (1536, 2112), (512, 512)):
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        for M in (1, 64, 8192):
            for residual in (False, True):
                nb = nvfp4_bytes(M, d, residual)
                n = sets_for(nb)
                xs = [torch.randn(M, ld, device="cuda", generator=gen).to(bf)[:, :d] for _ in range(n)]
                rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)] if residual else None
                qs = [torch.empty(M, d // 2, dtype=torch.uint8, device="cuda") for _ in range(n)]
                sf = [torch.empty(M, d // 16, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
                fn = lambda i: nq.nq_rmsnorm_quant_nvfp4(
                    xs[i], g, gs, 1e-6, residual=rs[i] if residual else None,
                    residual_out=rs[i] if residual else None, q_out=qs[i], sf_out=sf[i], flags=flags)
                us = time_calls(fn, n, reps_for(nb, n))
                extra = {"host_latency_us": host_latency_us(fn)} if M <= 64 else {}
                del xs, rs, qs, sf
                rows.append(with_copy(cell(peak, M, nb, us, call="nq_rmsnorm_quant_nvfp4", residual=residual, M=M,
                                           d=d, ld_x=ld, sets=n, **extra)))
    out["4_nvfp4"] = rows

    rows = []
    for d in (4096, 7168):
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        for M in (1, 256, 8192, 32768):
            for residual in (False, True):
                nb = rms_group_bytes(M, d, residual)
                n = sets_for(nb)
                xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)]
                rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)] if residual else None
                qs = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
                sc_ = [torch.empty(M, d // 128, dtype=torch.float32, device="cuda") for _ in range(n)]
                us = time_calls(lambda i: nq.nq_rmsnorm_quant_fp8_group(
                    xs[i], g, 1e-6, residual=rs[i] if residual else None,
                    residual_out=rs[i] if residual else None, q_out=qs[i], scales_out=sc_[i], flags=flags), n,
                    reps_for(nb, n))
                del xs, rs, qs, sc_
                rows.append(with_copy(cell(peak, M, nb, us, call="nq_rmsnorm_quant_fp8_group", residual=residual,
                                           M=M, d=d, sets=n)))
    out["next_fused_group"] = rows

    rows = []
    d, E, topk = 7168, 256, 8
    g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
    for M in (256, 4096, 32768):
        route = S.make_moe_routing(M, E, topk, seed=M)
        dest = torch.from_numpy(route["dest"]).cuda()
        n_rows = route["rows"]
        for group in (0, 128):
            nb = moe_bytes(M, d, topk, group)
            n = sets_for(nb)
            xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)]
            rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(n)]
            qs = [torch.empty(n_rows, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(n)]
            sc_ = [torch.empty((n_rows, d // 128) if group else (n_rows,), dtype=torch.float32, device="cuda")
                   for _ in range(n)]
            us = time_calls(lambda i: nq.nq_fused_add_rmsnorm_quant_fp8_moe(
                xs[i], g, dest, n_rows, 1e-6, group=group, residual=rs[i], residual_out=rs[i], q_out=qs[i],
                scales_out=sc_[i], flags=flags), n, reps_for(nb, n))
            del xs, rs, qs, sc_
            rows.append(with_copy(cell(peak, M, nb, us, call="nq_fused_add_rmsnorm_quant_fp8_moe", group=group, M=M,
                                       d=d, experts=E, topk=topk, sets=n)))
    out["next_moe_dispatch"] = rows
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------- CPU baseline ----
def _oracle_sample(rows: int, seed: int = 0):
    """A bounded sample of the headline workload for the oracle: `rows` tokens of
    the same width and input distribution, from the seeded host generator."""
    import synthetic as S
    return S.make_rms_inputs(rows, HEAD_D, seed=seed, x_outlier_channels=True)


def cpu_baseline(seconds: float = 15.0, rows: int = 256):
    """The oracle as it stands (single-threaded C++) on the host cores, on
    samples of the headline workload, repeated until ~`seconds` have passed."""
    import oracle
    w = _oracle_sample(rows)
    oracle.build()
    calls, t0 = 0, time.perf_counter()
    while True:
        oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], eps=HEAD_EPS)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    nb = fused_dyn_bytes(rows, HEAD_D)
    return {"value": round(calls * nb / el / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{calls} calls of {rows} of the 65536 tokens (d = 8192, same input distribution) "
                      f"in {el:.1f} s",
            "cpu": _cpu_model(), "host_cores": os.cpu_count()}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def run_reference_arm(args):
    """The oracle timed on host cores, each step a bounded sample of the headline
    workload (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    rows = args.ref_rows
    w = _oracle_sample(rows)
    oracle.build()
    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], eps=HEAD_EPS)
    t0 = time.perf_counter()
    for _ in range(K):
        oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], eps=HEAD_EPS)
    el = time.perf_counter() - t0
    nb = fused_dyn_bytes(rows, HEAD_D)
    value = K * nb / el / 1e9
    sample = f"{rows} of the 65536 tokens per step (d = 8192, same input distribution)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC,
        "value": round(value, 4), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": K,
        "warmup": W, "ms_per_step": round(el * 1e3 / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded host generator)",
        "config": {"workload": HEAD_WORKLOAD, "M": HEAD_M, "d": HEAD_D, "eps": HEAD_EPS, "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "cpu": _cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_case(args):
    """Run one call a few times on a device-seeded input (for ncu captures of a
    single kernel); prints nothing but 'ok'."""
    import torch
    import fp4_activation_quantization_b200 as nq
    M, d, op = args.M, args.d, args.case
    bf = torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(0)
    ld = max(args.ld, d)  # > d: x is the first d columns of an [M, ld] tensor
    x = outlier_x(M, d, g) if op == "fused_add_rmsnorm_quant_fp8" else \
        torch.randn(M, ld, device="cuda", generator=g).to(bf)[:, :d]
    res = (torch.randn(M, d, device="cuda", generator=g).to(bf)
           if op in ("fused_add_rmsnorm_quant_fp8", "nvfp4_res", "rmsnorm_quant_fp8_group_res") else None)
    gam = (1 + 0.1 * torch.randn(d, device="cuda", generator=g)).to(bf)
    gl = 1 + 0.1 * torch.randn(d, device="cuda", generator=g)
    bl = 0.02 * torch.randn(d, device="cuda", generator=g)
    sc = torch.tensor([STATIC_SCALE], device="cuda")
    ro = torch.empty_like(res) if res is not None else None
    for _ in range(args.iters):
        if op == "rmsnorm_quant_fp8_static":
            nq.nq_rmsnorm_quant_fp8_static(x, gam, sc, STATIC_EPS)
        elif op == "layernorm_quant_fp8":
            nq.nq_layernorm_quant_fp8(x, gl, bl, sc, STATIC_EPS)
        elif op == "fused_add_rmsnorm_quant_fp8":
            nq.nq_fused_add_rmsnorm_quant_fp8(x, res, gam, HEAD_EPS, residual_out=ro)
        elif op in ("nvfp4", "nvfp4_res"):
            nq.nq_rmsnorm_quant_nvfp4(x, gam, sc, 1e-6, residual=res, residual_out=ro)
        elif op == "per_token_group_quant_fp8":
            nq.nq_per_token_group_quant_fp8(x, 128)
        elif op in ("rmsnorm_quant_fp8_group", "rmsnorm_quant_fp8_group_res"):
            nq.nq_rmsnorm_quant_fp8_group(x, gam, 1e-6, residual=res, residual_out=ro)
    torch.cuda.synchronize()
    print("ok")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["nq", "reference"], default="nq")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch (default: with)")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration cells")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--case", choices=["rmsnorm_quant_fp8_static", "layernorm_quant_fp8",
                                       "fused_add_rmsnorm_quant_fp8", "nvfp4", "nvfp4_res",
                                       "per_token_group_quant_fp8", "rmsnorm_quant_fp8_group",
                                       "rmsnorm_quant_fp8_group_res"],
                    help="run one call --iters times on M x d and exit (for profiler captures)")
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--ld", type=int, default=0, help="--case: row stride of x (a column slice when > d)")
    args = ap.parse_args()
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference_arm(args)
    else:
        run_gpu_arm(args)


if __name__ == "__main__":
    main()
