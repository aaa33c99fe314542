"""Benchmark: exact attention forward + backward on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one fa_fwd + one fa_bwd over one batch of the workload (the whole
hot path). The default workload is the 12-layer decoder's attention: B=4,
N=4096, H=8, d=128, bf16, causal. Timing: CUDA events on the launching stream
around each call, and around the backward's dK/dV kernel itself (the
library's profiling hook); L2 flushed (256 MiB write) before every step, the
flush not timed; the K timed steps are bracketed by a barrier and a device
synchronize on both sides and the time is the max over ranks. SM clocks and
throttle reasons are polled through NVML every 2 ms while the timed steps run.
Multi-GPU (torchrun): every rank runs its own independent batch (attention
heads share nothing), no collective on the data path, weak scaling.

Metric: fwd+bwd TFLOPS with counted FLOPs 4*B*H*N^2*d (fwd) + 10*B*H*N^2*d
(bwd), halved when causal; fwd-only TFLOPS is reported beside it.

--impl reference runs the fp64 CPU oracle on a bounded sample of the same
workload (the only reference that exists for this path) and prints the same
JSON line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd and fwd+bwd TFLOPS (bf16/fp16) and % of B200 tensor peak"

# Workloads of the pages' shapes (batch, seqlen, heads, head_dim, dtype, causal).
WORKLOADS = {
    "tiny": (1, 128, 2, 64, "fp16", False),
    "p4_B2_N2048_H12_d64_fp16": (2, 2048, 12, 64, "fp16", False),
    "decoder_B4_N4096_H8_d128_bf16_causal": (4, 4096, 8, 128, "bf16", True),
    "llama7b_B1_N4096_H32_d128_bf16_causal": (1, 4096, 32, 128, "bf16", True),
}
for _n in (512, 1024, 2048, 4096, 8192, 16384, 32768):
    for _c in (False, True):
        WORKLOADS[f"sweep_N{_n}_H16_d128_bf16{'_causal' if _c else ''}"] = (max(1, 16384 // _n), _n, 16, 128, "bf16", _c)
DEFAULT_WORKLOAD = "decoder_B4_N4096_H8_d128_bf16_causal"

# Kernel sources whose hash keys a committed ncu traffic figure: a figure
# taken from an older version of the kernel is not reported.
KERNEL_SOURCES = {
    "fa_bwd_dkdv": ["sm100.cuh", "bwd_kernels.cuh"],
    "fa_fwd_kernel": ["sm100.cuh", "fwd_kernel.cuh"],
}


def sources_sha256(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "exact_attention_119_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from the ncu summaries
    under profiles/ (a line 'bench-key: workload=W kernel=K traffic_bytes=T
    sources_sha256=S'); (bytes, note). Null when no summary matches or the
    kernel source has changed since the capture."""
    import glob
    import re
    want = sources_sha256(kernel)
    stale = None
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as f:
            for line in f:
                m = re.search(r"bench-key: workload=(\S+) kernel=(\S+) traffic_bytes=(\d+) sources_sha256=(\w+)", line)
                if m and m.group(1) == workload and m.group(2) == kernel:
                    if m.group(4) == want:
                        return int(m.group(3)), f"ncu capture in profiles/{os.path.basename(path)}"
                    stale = os.path.basename(path)
    if stale:
        return None, f"profiles/{stale} was captured from an older kernel source (stale)"
    return None, "no ncu capture of this kernel and workload under profiles/"


SPEC_TFLOPS = 2250.0  # nominal dense fp16/bf16 tensor rate of one B200

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def flops(B, N, H, d, causal):
    base = B * H * N * N * d * (0.5 if causal else 1.0)
    return 4 * base, 10 * base


def exp_rate(B, N, H, causal, ms_sum, steps, world, sm_mhz, n_sm):
    """Exponentials per second in one pass (the forward, or the backward's
    recompute of P: one exp per unmasked score, halved when causal), whole job,
    and the exp unit's rate at the sampled SM clock (16 per clock per SM)."""
    count = B * H * N * N * (0.5 if causal else 1.0)
    achieved = world * steps * count / (ms_sum * 1e-3)
    peak = 16.0 * n_sm * sm_mhz * 1e6 * world if sm_mhz else None
    return achieved, peak


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock, power and throttle reasons polled through NVML every 2 ms on
    a host thread while the timed steps run (nvidia-smi -lms 50 is the
    fallback); only samples inside the marked window count."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.window = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self._nvml = pynvml
        except Exception:  # no NVML: no samples, the line says so
            return
        self._stop = threading.Event()

        def poll():
            mx = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    pw = pynvml.nvmlDeviceGetPowerUsage(handle) / 1000.0
                    self.samples.append((time.time(), sm, mx, rs, pw))
                except Exception:
                    pass
                time.sleep(0.002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        time.sleep(0.05)

    def mark(self, t0, t1):
        """Host wall-clock bounds of the timed region."""
        self.window = (t0, t1)

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        self._stop.set()
        self._thread.join(timeout=5)
        inside = [x for x in self.samples if self.window and self.window[0] <= x[0] <= self.window[1]]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": f"no sample inside the timed window ({len(self.samples)} outside)"}
        reasons = sorted({name for x in inside for name, bit in self.REASONS.items() if x[3] & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "sm_min_mhz": min(x[1] for x in inside), "power_w_median": statistics.median(x[4] for x in inside),
                "reasons": reasons, "samples": len(inside), "source": "NVML, 2 ms polling"}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(values, world, device=None):
    """Element-wise max over ranks of a list of floats (identity when world == 1)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(world, steps, flops_per_step, max_ms):
    """Throughput of the whole job: every rank's FLOPs over the slowest rank's time."""
    return world * steps * flops_per_step / (max_ms * 1e-3) / 1e12


def oracle_sample(workload, budget_s=15.0, max_heads=None):
    """Time the fp64 oracle on whole heads of the workload until budget_s."""
    import numpy as np
    from exact_attention_119_b200 import inputs
    from oracle import attention_backward, attention_forward
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count() or 1
    B, N, H, d, dtype, causal = workload
    scale = 1.0 / math.sqrt(d)
    one = (1, N, 1, d)
    t_all, heads = 0.0, 0
    limit = max_heads or B * H
    while heads < limit and (t_all < budget_s or heads == 0):
        seed = 1000 + heads
        q, k, v, do = (inputs.bits_to_f64(inputs.make_tensor_bits(one, dtype, seed, s), dtype) for s in range(4))
        t0 = time.perf_counter()
        attention_forward(q, k, v, scale, causal)
        attention_backward(q, k, v, do, scale, causal)
        t_all += time.perf_counter() - t0
        heads += 1
    f_fwd, f_bwd = flops(1, N, 1, d, causal)
    return {"heads": heads, "seconds": t_all, "flops": heads * (f_fwd + f_bwd), "cores": cores}


def run_reference(args, workload):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    B, N, H, d, dtype, causal = workload
    # Each step: a bounded sample (whole heads) of the workload on the host.
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(workload, budget_s=budget, max_heads=1)
    samples = [oracle_sample(workload, budget_s=budget) for _ in range(args.steps)]
    secs = sum(s["seconds"] for s in samples)
    fl = sum(s["flops"] for s in samples)
    tflops = fl / secs / 1e12
    heads = samples[0]["heads"]
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(args.workload, workload),
        "cpu_baseline": {"value": tflops, "unit": "TFLOPS", "cores": samples[0]["cores"], "kind": "oracle",
                         "sample": f"{heads} whole head(s) of {B * H} per step, fwd+bwd, fp64 numpy oracle"},
        "e2e": {"value": tflops, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# Reported beside the headline, same protocol, fewer steps: the other
# workloads the stated targets are quoted on (N >= 4096, d = 128) and the
# pages' d = 64 comparison shape.
EXTRA_WORKLOADS = ["llama7b_B1_N4096_H32_d128_bf16_causal", "sweep_N4096_H16_d128_bf16",
                   "sweep_N16384_H16_d128_bf16", "sweep_N16384_H16_d128_bf16_causal", "p4_B2_N2048_H12_d64_fp16"]


class Buffers:
    """Device inputs and outputs of one workload (inputs seeded on the host)."""

    def __init__(self, workload, dev, rank, pinned=False):
        import torch
        import exact_attention_119_b200 as fa
        from exact_attention_119_b200 import inputs
        B, N, H, d, dtype, causal = workload
        self.workload = workload
        self.scale = 1.0 / math.sqrt(d)
        bits = inputs.attention_inputs(B, N, H, d, dtype, seed=rank)
        self.host = {k: inputs.bits_to_torch(v, dtype) for k, v in bits.items()}
        if pinned:
            self.host = {k: v.pin_memory() for k, v in self.host.items()}
        self.q, self.k, self.v, self.do = (self.host[n].to(dev) for n in ("q", "k", "v", "do"))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.ws = torch.empty(max(16, fa.bwd_workspace_size(B, N, H, d, causal)), dtype=torch.uint8, device=dev)

    def fwd(self):
        import exact_attention_119_b200 as fa
        fa.forward(self.q, self.k, self.v, self.scale, self.workload[5], out=self.o, lse=self.lse)

    def bwd(self):
        import exact_attention_119_b200 as fa
        fa.backward(self.q, self.k, self.v, self.o, self.do, self.lse, self.scale, self.workload[5],
                    self.dq, self.dk, self.dv, workspace=self.ws)


def timed_steps(buf, steps, stream, flush):
    """Run `steps` steps with events around fa_fwd, fa_bwd and the backward's
    dK/dV kernel; returns per-step (fwd, bwd, dkdv) milliseconds. The L2 is
    flushed before each step unless flush is None."""
    import torch
    import exact_attention_119_b200 as fa
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        fa.profile_bwd_events(ev[i][3], ev[i][4])
        ev[i][0].record(stream)
        buf.fwd()
        ev[i][1].record(stream)
        buf.bwd()
        ev[i][2].record(stream)
    fa.profile_bwd_events(None, None)
    return ev


def elapsed(ev):
    return ([e[0].elapsed_time(e[1]) for e in ev], [e[1].elapsed_time(e[2]) for e in ev],
            [e[3].elapsed_time(e[4]) for e in ev])


def e2e_steps(buf, steps, dev, flush):
    """Device milliseconds of `steps` end-to-end steps: overlapped (two device
    buffer sets, an upload, a compute and a download stream) and, for
    context, serial (one stream, copy in, compute, copy out)."""
    import torch
    import exact_attention_119_b200 as fa
    B, N, H, d, dtype, causal = buf.workload
    host_in = buf.host
    sets = [buf, Buffers(buf.workload, dev, 1)]
    host_out = [{n: torch.empty_like(host_in["q"]).pin_memory() for n in ("o", "dq", "dk", "dv")} for _ in sets]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done = [ev() for _ in sets]
    comp_done = [ev() for _ in sets]
    out_done = [ev() for _ in sets]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    flush.fill_(0)
    torch.cuda.synchronize(dev)
    start.record(s_in)
    for i in range(steps):
        x = i % 2
        bs, ho = sets[x], host_out[x]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[x])      # the inputs of step i-2 are no longer read
            for n, t in (("q", bs.q), ("k", bs.k), ("v", bs.v), ("do", bs.do)):
                t.copy_(host_in[n], non_blocking=True)
            in_done[x].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[x])
            if i >= 2:
                s_comp.wait_event(out_done[x])     # step i-2's results are out
            fa.forward(bs.q, bs.k, bs.v, bs.scale, causal, out=bs.o, lse=bs.lse, stream=s_comp)
            fa.backward(bs.q, bs.k, bs.v, bs.o, bs.do, bs.lse, bs.scale, causal, bs.dq, bs.dk, bs.dv,
                        workspace=bs.ws, stream=s_comp)
            comp_done[x].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[x])
            for n, t in (("o", bs.o), ("dq", bs.dq), ("dk", bs.dk), ("dv", bs.dv)):
                ho[n].copy_(t, non_blocking=True)
            out_done[x].record(s_out)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_comp)
    end.record(s_in)
    torch.cuda.synchronize(dev)
    overlapped = start.elapsed_time(end)
    # serial, one stream, for context
    stream = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for i in range(steps):
        for n, t in (("q", buf.q), ("k", buf.k), ("v", buf.v), ("do", buf.do)):
            t.copy_(host_in[n], non_blocking=True)
        buf.fwd()
        buf.bwd()
        for n, t in (("o", buf.o), ("dq", buf.dq), ("dk", buf.dk), ("dv", buf.dv)):
            host_out[0][n].copy_(t, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(dev)
    if fa.check_device_status() != 0:
        raise RuntimeError("device status not OK after the end-to-end steps")
    del sets[1]
    return overlapped, a.elapsed_time(b)


def time_workload(workload, steps, warmup, dev, stream, flush, world, rank):
    """fwd, bwd, fwd+bwd and dK/dV-kernel TFLOPS of one workload (events per
    call, L2 flushed)."""
    import torch
    import exact_attention_119_b200 as fa
    buf = Buffers(workload, dev, rank)
    for _ in range(warmup):
        buf.fwd()
        buf.bwd()
    torch.cuda.synchronize(dev)
    ev = timed_steps(buf, steps, stream, flush)
    torch.cuda.synchronize(dev)
    if fa.check_device_status() != 0:
        raise RuntimeError("device status not OK")
    f, b, k = (sum(x) for x in elapsed(ev))
    f_ms, b_ms, k_ms = reduce_max([f, b, k], world, dev)
    B, N, H, d, dtype, causal = workload
    f_fwd, f_bwd = flops(B, N, H, d, causal)
    out = {"fwd_tflops": whole_job_tflops(world, steps, f_fwd, f_ms),
           "bwd_tflops": whole_job_tflops(world, steps, f_bwd, b_ms),
           "fwd_bwd_tflops": whole_job_tflops(world, steps, f_fwd + f_bwd, f_ms + b_ms),
           "dkdv_kernel_tflops": whole_job_tflops(world, steps, f_bwd, k_ms),
           "steps": steps}
    del buf
    torch.cuda.empty_cache()
    return out


# KV-cache decode (one new position per sequence against a long cache): an
# HBM-bound workload, reported as GB/s of cache read against the HBM peak.
DECODE_WORKLOADS = {
    "decode_B8_H32_L8192_d128_bf16": (8, 1, 32, 128, 8192, "bf16"),
    "decode_B1_H32_L32768_d128_bf16": (1, 1, 32, 128, 32768, "bf16"),
}


def time_decode(workload, steps, dev, stream, flush, world, rank):
    """fa_decode over a full cache: device time per call (events, L2 flushed
    before each call), and the cache bytes it must read per call."""
    import torch
    import exact_attention_119_b200 as fa
    from exact_attention_119_b200 import inputs
    B, Nq, H, d, L, dtype = workload
    q = inputs.bits_to_torch(inputs.make_tensor_bits((B, Nq, H, d), dtype, rank, 0), dtype).to(dev)
    kc = inputs.bits_to_torch(inputs.make_tensor_bits((B, L, H, d), dtype, rank, 1), dtype).to(dev)
    vc = inputs.bits_to_torch(inputs.make_tensor_bits((B, L, H, d), dtype, rank, 2), dtype).to(dev)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, fa.decode_workspace_size(B, Nq, H, d, L)), dtype=torch.uint8, device=dev)
    for _ in range(3):
        fa.decode(q, kc, vc, lens, None, False, out=o, lse=lse, workspace=ws)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        fa.decode(q, kc, vc, lens, None, False, out=o, lse=lse, workspace=ws)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if fa.check_device_status() != 0:
        raise RuntimeError("device status not OK")
    (ms,) = reduce_max([sum(a.elapsed_time(b) for a, b in ev)], world, dev)
    nbytes = 2 * B * L * H * d * 2 + 2 * B * Nq * H * d * 2 + B * H * Nq * 4
    out = {"us_per_call": 1e3 * ms / steps, "gbs": world * steps * nbytes / (ms * 1e-3) / 1e9,
           "bytes_per_call": nbytes, "steps": steps,
           "note": "K and V cache read once, q read, O and LSE written (the partial states stay in L2)"}
    del q, kc, vc, o, lse, ws
    torch.cuda.empty_cache()
    return out


def run_decode_only(args):
    """--workload decode_*: only the KV-cache decode, as GB/s of cache read
    (a side measurement; the headline is the attention fwd+bwd step)."""
    import torch
    world, rank, local = dist_env()
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if args.impl == "reference":
        print(json.dumps({"impl": "reference", "unavailable": "the decode side measurement has no reference arm"}))
        return 0
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    r = time_decode(DECODE_WORKLOADS[args.workload], args.steps, dev, torch.cuda.current_stream(dev), flush, 1, 0)
    peaks, kind = load_peaks()
    B, Nq, H, d, L, dtype = DECODE_WORKLOADS[args.workload]
    print(json.dumps({"metric": "KV-cache decode GB/s", "value": r["gbs"], "unit": "GB/s", "n_gpus": 1,
                      "steps": args.steps, "higher_is_better": True, "dtype": dtype,
                      "config": {"workload": args.workload, "batch": B, "new_rows": Nq, "heads": H, "head_dim": d,
                                 "cache_len": L},
                      "frac_of_hbm_peak": r["gbs"] / float(peaks["hbm_gbs"]), "peak_kind": kind, **r}))
    return 0


def config_dict(name, workload):
    B, N, H, d, dtype, causal = workload
    return {"workload": name, "batch": B, "seqlen": N, "heads": H, "head_dim": d, "dtype": dtype,
            "causal": causal, "layout": "[B,N,H,d]",
            "l2": "flushed before every step (256 MiB write), flush not timed"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads reported beside the headline")
    ap.add_argument("--extra-steps", type=int, default=30)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in DECODE_WORKLOADS:
        return run_decode_only(args)
    workload = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, workload)

    import torch
    import torch.distributed as dist

    import exact_attention_119_b200 as fa

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    B, N, H, d, dtype, causal = workload
    buf = Buffers(workload, dev, rank, pinned=True)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        flush.fill_(1)
        buf.fwd()
        buf.bwd()
    torch.cuda.synchronize(dev)
    assert fa.check_device_status() == 0

    # ---- the timed steps (device-resident inputs)
    sampler = ClockSampler(dev.index)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev = timed_steps(buf, args.steps, stream, flush)
    torch.cuda.synchronize(dev)
    sampler.mark(t_wall0, time.time())
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    status = fa.check_device_status()
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after the timed steps")
    fwd_ms, bwd_ms, dkdv_ms = elapsed(ev)
    tot_ms, fwd_sum, bwd_sum, dkdv_sum = reduce_max(
        [sum(fwd_ms) + sum(bwd_ms), sum(fwd_ms), sum(bwd_ms), sum(dkdv_ms)], world, dev)

    f_fwd, f_bwd = flops(B, N, H, d, causal)
    value = whole_job_tflops(world, args.steps, f_fwd + f_bwd, tot_ms)
    fwd_tflops = whole_job_tflops(world, args.steps, f_fwd, fwd_sum)
    bwd_tflops = whole_job_tflops(world, args.steps, f_bwd, bwd_sum)
    dkdv_tflops = whole_job_tflops(world, args.steps, f_bwd, dkdv_sum)

    # ---- end to end through the public API: every step copies its inputs in
    # from pinned host memory and its results out to pinned host memory.
    # Double-buffered over three streams, so step i+1's upload and step i-1's
    # download overlap step i's kernels (PCIe is full duplex); the timed
    # region runs from the first upload to the last download.
    e2e_ms, e2e_serial_ms = e2e_steps(buf, args.steps, dev, flush)
    (e2e_ms, e2e_serial_ms) = reduce_max([e2e_ms, e2e_serial_ms], world, dev)
    if world > 1:
        dist.barrier()
    e2e_value = whole_job_tflops(world, args.steps, f_fwd + f_bwd, e2e_ms)
    tensor_bytes = B * N * H * d * 2

    # ---- the same steps back to back without the L2 flush, reported beside the headline
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    nf = timed_steps(buf, args.steps, stream, None)
    torch.cuda.synchronize(dev)
    nf_f, nf_b, _ = (sum(x) for x in elapsed(nf))
    nf_f, nf_b = reduce_max([nf_f, nf_b], world, dev)
    if world > 1:
        dist.barrier()
    no_flush = {"value": whole_job_tflops(world, args.steps, f_fwd + f_bwd, nf_f + nf_b),
                "fwd_tflops": whole_job_tflops(world, args.steps, f_fwd, nf_f),
                "bwd_tflops": whole_job_tflops(world, args.steps, f_bwd, nf_b), "unit": "TFLOPS",
                "note": "the same steps back to back, L2 not flushed between them"}

    peaks, peak_kind = load_peaks()
    # fp16 and bf16 run at the same dense tensor rate. A kernel timed inside a
    # step of a few hundred microseconds is a burst, not a seconds-long loop.
    peak = float(peaks["bf16_tflops"])
    traffic, traffic_note = committed_traffic(args.workload, "fa_bwd_dkdv")

    extra, decode = {}, {}
    if not args.no_extra and args.workload == DEFAULT_WORKLOAD:
        for name in EXTRA_WORKLOADS:
            extra[name] = time_workload(WORKLOADS[name], args.extra_steps, 3, dev, stream, flush, world, rank)
        for name, wl in DECODE_WORKLOADS.items():
            decode[name] = time_decode(wl, 50, dev, stream, flush, world, rank)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16" if dtype == "fp16" else "bf16",
            "data": "synthetic", "config": config_dict(args.workload, workload),
            "fwd_tflops": fwd_tflops, "bwd_tflops": bwd_tflops,
            "fwd_ms": fwd_sum / args.steps, "bwd_ms": bwd_sum / args.steps, "dkdv_kernel_ms": dkdv_sum / args.steps,
            "frac_of_peak": {"fwd": fwd_tflops / world / peak, "fwd_bwd": value / world / peak,
                             "peak_tflops": peak, "peak_kind": peak_kind + " bf16 dense (cuBLAS burst)",
                             "fwd_spec": fwd_tflops / world / SPEC_TFLOPS, "fwd_bwd_spec": value / world / SPEC_TFLOPS,
                             "spec_tflops": SPEC_TFLOPS},
            "no_l2_flush": no_flush,
            "roofline": {"bound": "tensor", "kernel": "fa_bwd_dkdv", "achieved": dkdv_tflops / world, "peak": peak,
                         "unit": "TFLOP/s", "frac": dkdv_tflops / world / peak, "traffic": traffic,
                         "note": ("the backward's dK/dV kernel, which runs all five backward contractions "
                                  "(10*B*H*N^2*d, halved when causal) and then sums and casts dQ, timed by "
                                  "events on its own launch; "
                                  f"peak {peak_kind}; traffic: {traffic_note}")},
            "kernels": {
                "fa_fwd_kernel": {"tflops": fwd_tflops / world, "frac": fwd_tflops / world / peak,
                                  "ms": fwd_sum / args.steps},
                "fa_bwd_dkdv": {"tflops": dkdv_tflops / world, "frac": dkdv_tflops / world / peak,
                                "ms": dkdv_sum / args.steps},
                "fa_bwd_prep": {"ms": (bwd_sum - dkdv_sum) / args.steps}},
            "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": 4 * tensor_bytes,
                    "d2h_bytes_per_step": 4 * tensor_bytes,
                    "note": "q, k, v, dO in and O, dQ, dK, dV out every step; copies of neighbouring steps "
                            "overlap the kernels (two buffer sets, three streams)",
                    "serial_value": whole_job_tflops(world, args.steps, f_fwd + f_bwd, e2e_serial_ms)},
            "gpu_launches": 3 * args.steps,  # fa_fwd_kernel, fa_bwd_prep, fa_bwd_dkdv
            "clocks": clocks,
        }
        try:
            # median sampled SM clock; the maximum clock when no sample fell inside the window
            sm_mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz")
            n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
            ef, peak_e = exp_rate(B, N, H, causal, fwd_sum, args.steps, world, sm_mhz, n_sm)
            eb, _ = exp_rate(B, N, H, causal, bwd_sum, args.steps, world, sm_mhz, n_sm)
            line["exp_throughput"] = {
                "fwd_per_s": ef, "bwd_per_s": eb, "peak_per_s": peak_e,
                "fwd_frac": ef / peak_e if peak_e else None, "bwd_frac": eb / peak_e if peak_e else None,
                "note": "one exp per unmasked score per pass; peak = 16/clk/SM x SMs x median sampled SM clock"}
        except Exception as exc:  # a secondary figure; never lose the bench line over it
            line["exp_throughput"] = {"error": str(exc)[:200]}
        if extra:
            for v in extra.values():
                v["fwd_frac_of_peak"] = v["fwd_tflops"] / peak
                v["fwd_bwd_frac_of_peak"] = v["fwd_bwd_tflops"] / peak
                v["dkdv_frac_of_peak"] = v["dkdv_kernel_tflops"] / peak
            line["other_workloads"] = extra
        if decode:
            hbm = float(peaks["hbm_gbs"])
            for v in decode.values():
                v["frac_of_hbm_peak"] = v["gbs"] / world / hbm
                v["hbm_peak_gbs"] = hbm
            line["decode_workloads"] = decode
        if world == 1 and not args.no_cpu_baseline:
            smp = oracle_sample(workload, budget_s=15.0)
            line["cpu_baseline"] = {
                "value": smp["flops"] / smp["seconds"] / 1e12, "unit": "TFLOPS", "cores": smp["cores"],
                "kind": "oracle",
                "sample": f"{smp['heads']} whole head(s) of {B * H}, fwd+bwd, fp64 numpy oracle, {smp['seconds']:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
