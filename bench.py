#!/usr/bin/env python
"""Benchmark of the fused norm + FP8 quantization hot path on B200.

Workload (one "step"): RMSNorm -> e4m3 with a static device scale (0.05) and
LayerNorm(gamma, beta) -> e4m3 with the same static scale, each over a batch
of M = 4096 tokens x d = 4096 bf16 activations (eps 1e-5).  The metric is
achieved HBM bandwidth of the whole step: algorithmic bytes (every input read
once, every output written once, gamma/beta/scale once per call) divided by
device time.

Timing: inputs are generated on the device (seeded), and a step uses one of S
rotating input/output sets whose total (S x 96 MiB) is several times the
126 MB L2, so no step finds its inputs in L2.  Calls are captured into CUDA
graphs of S launches (with programmatic dependent launch; ``--no-pdl``
without) and replayed back to back; CUDA events on the launching
stream bracket the whole timed region (exactly K steps) and every graph, which
gives each kernel's mean launch duration for the roofline.  Multi-GPU runs
(torchrun, one process per GPU) give every rank the same per-GPU workload
(weak scaling, no data-path collective); the time is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead, on a bounded sample per step.  ``--sweep`` adds a per-configuration
table (fused add+RMSNorm+dynamic FP8 sweep, group FP8, fused RMSNorm + group
FP8, NVFP4) under "sweep".
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

M_TOK, D_HID, SCALE, EPS = 4096, 4096, 0.05, 1e-5
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def rms_static_bytes(M, d):
    return M * 3 * d + 2 * d + 4           # x read, e4m3 write; bf16 gamma; scale


def ln_static_bytes(M, d):
    return M * 3 * d + 8 * d + 4           # x read, e4m3 write; fp32 gamma + beta; scale


def fused_dyn_bytes(M, d):
    return M * (7 * d + 4) + 2 * d         # x, residual read; residual, e4m3, scale write; gamma


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


def kernel_source_hash() -> str:
    """Hash of the device-code sources (every csrc file except the host-side
    launcher nq_host.cu): a profile's counters stay valid while it matches."""
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "fp4_activation_quantization_b200", "csrc", "*"))):
        if os.path.basename(p) == "nq_host.cu":
            continue
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
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
    """dram read+write bytes per launch from a committed ncu summary, if it is
    for the current kernel sources (else None)."""
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(p).read()
        m_tag = re.search(r"^bench_kernel:\s*(\S+)", text, re.M)
        m_b = re.search(r"^traffic_bytes_per_launch:\s*(\d+)", text, re.M)
        m_h = re.search(r"^kernel_source_hash:\s*(\S+)", text, re.M)
        if m_tag and m_b and m_h and m_tag.group(1) == kernel_tag:
            return int(m_b.group(1)) if m_h.group(1) == kernel_source_hash() else None
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


# ------------------------------------------------------------ GPU arm ----
class Workload:
    """S rotating sets of RMSNorm / LayerNorm inputs and outputs on the device."""

    def __init__(self, nq, M, d, sets, seed=0):
        import torch
        self.nq, self.M, self.d, self.S = nq, M, d, sets
        gen = torch.Generator(device="cuda").manual_seed(seed)
        bf = torch.bfloat16
        self.x_rms = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(sets)]
        self.x_ln = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(sets)]
        self.q_rms = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(sets)]
        self.q_ln = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(sets)]
        self.g_rms = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        self.g_ln = 1 + 0.1 * torch.randn(d, device="cuda", generator=gen)
        self.b_ln = 0.02 * torch.randn(d, device="cuda", generator=gen)
        self.scale = torch.tensor([SCALE], dtype=torch.float32, device="cuda")

    def rms(self, i, flags=0):
        self.nq.nq_rmsnorm_quant_fp8_static(self.x_rms[i], self.g_rms, self.scale, EPS, q_out=self.q_rms[i],
                                            flags=flags)

    def ln(self, i, flags=0):
        self.nq.nq_layernorm_quant_fp8(self.x_ln[i], self.g_ln, self.b_ln, self.scale, EPS, q_out=self.q_ln[i],
                                       flags=flags)

    def capture(self, fn, n, flags=0):
        import torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(n):
                fn(i, flags)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                fn(i, flags)
        return g


def run_gpu_arm(args):
    import torch
    import fp4_activation_quantization_b200 as nq

    world, rank, local = dist_setup(args.gpus)
    M, d = M_TOK, D_HID
    set_bytes = M * d * 2 * 2 + M * d * 2          # two bf16 inputs + two e4m3 outputs
    S = max(8, -(-4 * L2_BYTES // set_bytes))      # > 4x L2 in flight between reuses
    wl = Workload(nq, M, d, S, seed=1234 + rank)
    # Programmatic dependent launch: each kernel waits (griddepcontrol.wait)
    # for the previous one before its first read, so no work is skipped; its
    # CTAs are resident earlier, as when these kernels follow a GEMM.
    flags = 0 if args.no_pdl else nq.FLAG_PDL
    g_rms, g_ln = wl.capture(wl.rms, S, flags), wl.capture(wl.ln, S, flags)
    K, W = args.steps, max(3, args.warmup)
    q_full, r = divmod(K, S)
    g_rms_r = wl.capture(wl.rms, r, flags) if r else None
    g_ln_r = wl.capture(wl.ln, r, flags) if r else None

    def run_steps(n, events=None):
        full, rem = divmod(n, S)
        chunks = [(g_rms, g_ln)] * full
        if rem:
            chunks.append((wl.capture(wl.rms, rem, flags), wl.capture(wl.ln, rem, flags)) if rem != r
                          else (g_rms_r, g_ln_r))
        for ci, (ga, gb) in enumerate(chunks):
            if events is not None:
                events[ci][0].record()
            ga.replay()
            if events is not None:
                events[ci][1].record()
            gb.replay()
            if events is not None:
                events[ci][2].record()

    # warm-up: exactly W steps
    run_steps(W)
    torch.cuda.synchronize()

    n_chunks = q_full + (1 if r else 0)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_chunks)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id_for(torch.cuda.current_device()))
    sampler.start()
    time.sleep(0.3)

    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    e0.record()
    run_steps(K, ev)
    e1.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    time.sleep(0.15)
    sampler.stop()

    elapsed_ms = e0.elapsed_time(e1)
    rms_ms = sum(c[0].elapsed_time(c[1]) for c in ev)
    ln_ms = sum(c[1].elapsed_time(c[2]) for c in ev)
    elapsed_ms = max_over_ranks(world, elapsed_ms)

    step_bytes = rms_static_bytes(M, d) + ln_static_bytes(M, d)
    value = job_throughput(world, K, step_bytes, elapsed_ms)
    peak, peak_src = measured_peak()
    rms_us, ln_us = rms_ms * 1e3 / K, ln_ms * 1e3 / K
    dom = ("nq_rmsnorm_quant_fp8_static", rms_us, rms_static_bytes(M, d)) if rms_us >= ln_us else \
        ("nq_layernorm_quant_fp8", ln_us, ln_static_bytes(M, d))
    achieved = dom[2] / (dom[1] * 1e-6) / 1e9
    clocks = sampler.summary(t0, t1)

    # ---- end to end through the public API: pinned host buffers, copies in the timed region
    e2e = None
    if not args.no_e2e:
        ke = min(K, args.e2e_steps)
        xh_r = [wl.x_rms[i % S].cpu().pin_memory() for i in range(2)]
        xh_l = [wl.x_ln[i % S].cpu().pin_memory() for i in range(2)]
        qh_r = torch.empty(M, d, dtype=torch.float8_e4m3fn).pin_memory()
        qh_l = torch.empty(M, d, dtype=torch.float8_e4m3fn).pin_memory()
        xd_r, xd_l = torch.empty_like(wl.x_rms[0]), torch.empty_like(wl.x_ln[0])
        qd_r, qd_l = wl.q_rms[0], wl.q_ln[0]

        def e2e_step(i):
            xd_r.copy_(xh_r[i % 2], non_blocking=True)
            xd_l.copy_(xh_l[i % 2], non_blocking=True)
            nq.nq_rmsnorm_quant_fp8_static(xd_r, wl.g_rms, wl.scale, EPS, q_out=qd_r)
            nq.nq_layernorm_quant_fp8(xd_l, wl.g_ln, wl.b_ln, wl.scale, EPS, q_out=qd_l)
            qh_r.copy_(qd_r, non_blocking=True)
            qh_l.copy_(qd_l, non_blocking=True)

        for i in range(3):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(ke):
            e2e_step(i)
        b.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(world, a.elapsed_time(b))
        barrier(world)
        e2e = {"value": round(job_throughput(world, ke, step_bytes, e2e_ms), 3), "unit": "GB/s",
               "h2d_bytes_per_step": 2 * M * d * 2, "d2h_bytes_per_step": 2 * M * d, "steps": ke,
               "ms_per_step": round(e2e_ms / ke, 4)}

    sweep = run_sweep(nq) if args.sweep and rank == 0 else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    if world > 1:
        import torch.distributed as dist
        del g_rms, g_ln, g_rms_r, g_ln_r
        dist.destroy_process_group()

    if rank != 0:
        return
    out = {
        "metric": "fused norm+quant HBM GB/s (% of B200 peak) and µs/call, M=1..65536",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(elapsed_ms / K, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (device-seeded: x bf16 N(0,1); RMS gamma bf16 1+0.1N; LN gamma f32 1+0.1N, beta f32 0.02N)",
        "config": {"workload": "RMSNorm->e4m3 static + LayerNorm->e4m3 static, M=4096 tokens, d=4096",
                   "M": M, "d": d, "scale": SCALE, "eps": EPS, "io": "bf16 in, e4m3 out, fp32 math",
                   "l2": f"inputs rotate over {S} sets ({S * set_bytes / 2**20:.0f} MiB, > L2 126 MB)",
                   "graphs": f"CUDA graphs of {S} launches replayed back to back", "pdl": not args.no_pdl,
                   "parallelism": f"replicas x{world} (rows shard, no collective)"},
        "per_call": {"nq_rmsnorm_quant_fp8_static": {"us": round(rms_us, 3),
                                                     "GBps": round(rms_static_bytes(M, d) / rms_us / 1e3, 1)},
                     "nq_layernorm_quant_fp8": {"us": round(ln_us, 3),
                                                "GBps": round(ln_static_bytes(M, d) / ln_us / 1e3, 1)},
                     "tokens_per_s_per_gpu": round(M * 2 / ((rms_us + ln_us) * 1e-6), 1)},
        "roofline": {"bound": "hbm", "kernel": dom[0], "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": peak_src, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_nominal_8000": round(achieved / NOMINAL_HBM_GBS, 4),
                     "algorithmic_bytes_per_launch": dom[2],
                     "traffic": profiled_traffic(dom[0])},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * K,
        "clocks": clocks,
        "kernel_source_hash": kernel_source_hash(),
    }
    if sweep is not None:
        out["sweep"] = sweep
    print(json.dumps(out), flush=True)


# ------------------------------------------------------ sweep table ----
def _time_graph(fn, n_sets, reps=20):
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
    return a.elapsed_time(b) * 1e3 / (reps * n_sets)  # us per call


def run_sweep(nq):
    """Per-configuration µs/call and GB/s (rotating sets > L2 where they fit, graphs)."""
    import torch
    gen = torch.Generator(device="cuda").manual_seed(7)
    bf = torch.bfloat16
    rows = []
    peak, _ = measured_peak()

    def sets_for(nbytes):
        return int(max(2, min(16, -(-3 * L2_BYTES // max(1, nbytes)))))

    for d in (2816, 4096, 7168, 8192):
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        for M in (1, 16, 256, 4096, 65536):
            nb = fused_dyn_bytes(M, d)
            S = sets_for(nb)
            xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S)]
            rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S)]
            qs = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(S)]
            ss = [torch.empty(M, dtype=torch.float32, device="cuda") for _ in range(S)]
            us = _time_graph(lambda i: nq.nq_fused_add_rmsnorm_quant_fp8(
                xs[i], rs[i], g, 1e-6, residual_out=rs[i], q_out=qs[i], scale_out=ss[i]), S,
                reps=max(3, min(200, int(2e8 // max(nb * S, 1)))))
            rows.append({"op": "fused_add_rmsnorm_quant_fp8", "M": M, "d": d, "us": round(us, 3),
                         "GBps": round(nb / us / 1e3, 1), "frac": round(nb / us / 1e3 / peak, 4)})
            del xs, rs, qs, ss
    for M in (1, 32768):
        for flags, tag in ((0, "fp32"), (nq.FLAG_UE8M0, "ue8m0")):
            K = 4096
            nb = group_bytes(M, K)
            S = sets_for(nb)
            xs = [torch.randn(M, K, device="cuda", generator=gen).to(bf) for _ in range(S)]
            qs = [torch.empty(M, K, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(S)]
            sc = [torch.empty(M, K // 128, dtype=torch.float32, device="cuda") for _ in range(S)]
            us = _time_graph(lambda i: nq.nq_per_token_group_quant_fp8(xs[i], 128, q_out=qs[i], scales_out=sc[i],
                                                                       flags=flags), S)
            rows.append({"op": f"per_token_group_quant_fp8[{tag}]", "M": M, "K": K, "us": round(us, 3),
                         "GBps": round(nb / us / 1e3, 1), "frac": round(nb / us / 1e3 / peak, 4)})
            del xs, qs, sc
    for d in (4096, 7168):
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        for M in (1, 256, 8192, 32768):
            for residual in (False, True):
                nb = rms_group_bytes(M, d, residual)
                S = sets_for(nb)
                xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S)]
                rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S)] if residual else None
                qs = [torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(S)]
                sc = [torch.empty(M, d // 128, dtype=torch.float32, device="cuda") for _ in range(S)]
                us = _time_graph(lambda i: nq.nq_rmsnorm_quant_fp8_group(
                    xs[i], g, 1e-6, residual=rs[i] if residual else None,
                    residual_out=rs[i] if residual else None, q_out=qs[i], scales_out=sc[i]), S)
                rows.append({"op": "rmsnorm_quant_fp8_group" + ("+res" if residual else ""), "M": M, "d": d,
                             "us": round(us, 3), "GBps": round(nb / us / 1e3, 1),
                             "frac": round(nb / us / 1e3 / peak, 4)})
                del xs, rs, qs, sc
    import synthetic as S
    d, E, topk = 7168, 256, 8
    g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
    for M in (256, 4096, 32768):
        route = S.make_moe_routing(M, E, topk, seed=M)
        dest = torch.from_numpy(route["dest"]).cuda()
        n_rows = route["rows"]
        for group in (0, 128):
            nb = moe_bytes(M, d, topk, group)
            S_ = sets_for(nb)
            xs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S_)]
            rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S_)]
            qs = [torch.empty(n_rows, d, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(S_)]
            sc = [torch.empty((n_rows, d // 128) if group else (n_rows,), dtype=torch.float32, device="cuda")
                  for _ in range(S_)]
            us = _time_graph(lambda i: nq.nq_fused_add_rmsnorm_quant_fp8_moe(
                xs[i], g, dest, n_rows, 1e-6, group=group, residual=rs[i], residual_out=rs[i], q_out=qs[i],
                scales_out=sc[i]), S_)
            rows.append({"op": "fused_add_rmsnorm_quant_fp8_moe" + ("[group128]" if group else "[per-token]"),
                         "M": M, "d": d, "experts": E, "topk": topk, "us": round(us, 3),
                         "GBps": round(nb / us / 1e3, 1), "frac": round(nb / us / 1e3 / peak, 4)})
            del xs, rs, qs, sc
    gs = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    for d, ld in ((7168, 7168), (1536, 2112), (512, 512)):
        g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(bf)
        for M in (1, 64, 8192):
            for residual in (False, True):
                nb = nvfp4_bytes(M, d, residual)
                S = sets_for(nb)
                xs = [torch.randn(M, ld, device="cuda", generator=gen).to(bf)[:, :d] for _ in range(S)]
                rs = [torch.randn(M, d, device="cuda", generator=gen).to(bf) for _ in range(S)] if residual else None
                qs = [torch.empty(M, d // 2, dtype=torch.uint8, device="cuda") for _ in range(S)]
                sf = [torch.empty(M, d // 16, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(S)]
                us = _time_graph(lambda i: nq.nq_rmsnorm_quant_nvfp4(
                    xs[i], g, gs, 1e-6, residual=rs[i] if residual else None,
                    residual_out=rs[i] if residual else None, q_out=qs[i], sf_out=sf[i]), S)
                rows.append({"op": "rmsnorm_quant_nvfp4" + ("+res" if residual else ""), "M": M, "d": d,
                             "ld_x": ld, "us": round(us, 3), "GBps": round(nb / us / 1e3, 1),
                             "frac": round(nb / us / 1e3 / peak, 4)})
                del xs, rs, qs, sf
    torch.cuda.empty_cache()
    return rows


# ----------------------------------------------------- CPU baseline ----
def cpu_baseline(seconds: float = 15.0):
    """The oracle as it stands (single-threaded C++), on the host cores, on the
    same workload (full M x d calls, repeated until ~`seconds` have passed)."""
    import oracle
    import synthetic as S
    w = S.make_rms_inputs(M_TOK, D_HID, seed=0, residual=False)
    lw = S.make_ln_inputs(M_TOK, D_HID, seed=0)
    oracle.build()
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], SCALE, eps=EPS)
        oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], SCALE, eps=EPS)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    step_bytes = rms_static_bytes(M_TOK, D_HID) + ln_static_bytes(M_TOK, D_HID)
    return {"value": round(steps * step_bytes / el / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps} full steps (RMSNorm + LayerNorm static e4m3, 4096x4096) in {el:.1f} s",
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
    """The oracle timed on host cores on a bounded sample per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synthetic as S
    rows = args.ref_rows
    w = S.make_rms_inputs(rows, D_HID, seed=0, residual=False)
    lw = S.make_ln_inputs(rows, D_HID, seed=0)
    oracle.build()
    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], SCALE, eps=EPS)
        oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], SCALE, eps=EPS)
    t0 = time.perf_counter()
    for _ in range(K):
        oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], SCALE, eps=EPS)
        oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], SCALE, eps=EPS)
    el = time.perf_counter() - t0
    step_bytes = rms_static_bytes(rows, D_HID) + ln_static_bytes(rows, D_HID)
    value = K * step_bytes / el / 1e9
    sample = f"{rows} of 4096 tokens per step (RMSNorm + LayerNorm static e4m3, d=4096)"
    print(json.dumps({
        "impl": "reference", "metric": "fused norm+quant HBM GB/s (% of B200 peak) and µs/call, M=1..65536",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": K,
        "warmup": W, "ms_per_step": round(el * 1e3 / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded host generator)",
        "config": {"workload": "RMSNorm->e4m3 static + LayerNorm->e4m3 static, M=4096 tokens, d=4096",
                   "M": M_TOK, "d": D_HID, "scale": SCALE, "eps": EPS, "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "cpu": _cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_case(args):
    """Run one call a few times on a device-seeded input (for ncu captures of a
    single kernel on a small case); prints nothing but 'ok'."""
    import torch
    import fp4_activation_quantization_b200 as nq
    M, d, op = args.M, args.d, args.case
    bf = torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.randn(M, d, device="cuda", generator=g).to(bf)
    res = (torch.randn(M, d, device="cuda", generator=g).to(bf)
           if op in ("fused_add_rmsnorm_quant_fp8", "nvfp4_res", "rmsnorm_quant_fp8_group_res") else None)
    gam = (1 + 0.1 * torch.randn(d, device="cuda", generator=g)).to(bf)
    gl = 1 + 0.1 * torch.randn(d, device="cuda", generator=g)
    bl = 0.02 * torch.randn(d, device="cuda", generator=g)
    sc = torch.tensor([SCALE], device="cuda")
    for _ in range(args.iters):
        if op == "rmsnorm_quant_fp8_static":
            nq.nq_rmsnorm_quant_fp8_static(x, gam, sc, EPS)
        elif op == "layernorm_quant_fp8":
            nq.nq_layernorm_quant_fp8(x, gl, bl, sc, EPS)
        elif op == "fused_add_rmsnorm_quant_fp8":
            nq.nq_fused_add_rmsnorm_quant_fp8(x, res, gam, 1e-6, residual_out=res)
        elif op in ("nvfp4", "nvfp4_res"):
            nq.nq_rmsnorm_quant_nvfp4(x, gam, sc, 1e-6, residual=res, residual_out=res)
        elif op == "per_token_group_quant_fp8":
            nq.nq_per_token_group_quant_fp8(x, 128)
        elif op in ("rmsnorm_quant_fp8_group", "rmsnorm_quant_fp8_group_res"):
            nq.nq_rmsnorm_quant_fp8_group(x, gam, 1e-6, residual=res, residual_out=res)
    torch.cuda.synchronize()
    print("ok")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=40)
    ap.add_argument("--impl", choices=["nq", "reference"], default="nq")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch (default: with)")
    ap.add_argument("--sweep", action="store_true", help="add the per-configuration table")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
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
    args = ap.parse_args()
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference_arm(args)
    else:
        run_gpu_arm(args)


if __name__ == "__main__":
    main()
