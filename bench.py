"""Benchmark: exact attention forward + backward on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one fa_fwd + one fa_bwd over one batch of the workload (the whole
hot path). Timing: CUDA events on the launching stream around each step, L2
flushed (256 MiB write) before every step and the flush excluded; the K timed
steps are bracketed by a barrier and a device synchronize on both sides and
the time is the max over ranks. Multi-GPU (torchrun): every rank runs its own
independent batch (attention heads share nothing), no collective on the data
path, weak scaling.

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
import subprocess
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
DEFAULT_WORKLOAD = "p4_B2_N2048_H12_d64_fp16"

# ncu DRAM bytes per launch of the dominant kernel, from the capture summarised
# in profiles/ for the default workload; None when the kernel has changed since.
NCU_TRAFFIC_BYTES = {
    # fa_bwd_dkdv<64,0,0>: dram__bytes_read.sum 25,630,976 + dram__bytes_write.sum 304,384
    ("p4_B2_N2048_H12_d64_fp16", "fa_bwd_dkdv"): 25_935_360,
}

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
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.window = None

    def start(self):
        """Start sampling every 50 ms; give nvidia-smi a head start."""
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except OSError:
            self.proc = None

    def mark(self, t0, t1):
        """Host wall-clock bounds of the timed region."""
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        import datetime
        sms, maxes, reasons, total = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                cols = [c.strip() for c in line.split(",")]
                if len(cols) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(cols[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    sm, mx = float(cols[2]), float(cols[3])
                except ValueError:
                    continue
                total += 1
                if self.window and not (self.window[0] <= ts <= self.window[1]):
                    continue
                sms.append(sm)
                maxes.append(mx)
                for name, val in zip(names, cols[6:10]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": f"no sample inside the timed window ({total} outside)"}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


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


EXTRA_WORKLOADS = ["decoder_B4_N4096_H8_d128_bf16_causal", "llama7b_B1_N4096_H32_d128_bf16_causal",
                   "sweep_N4096_H16_d128_bf16", "sweep_N16384_H16_d128_bf16"]


def time_workload(workload, steps, warmup, dev, stream, flush, world, rank):
    """fwd, bwd and fwd+bwd TFLOPS of one workload (events per call, L2 flushed)."""
    import torch
    import exact_attention_119_b200 as fa
    from exact_attention_119_b200 import inputs
    B, N, H, d, dtype, causal = workload
    scale = 1.0 / math.sqrt(d)
    bits = inputs.attention_inputs(B, N, H, d, dtype, seed=rank)
    q, k, v, do = (inputs.bits_to_torch(bits[n], dtype).to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(max(16, fa.bwd_workspace_size(B, N, H, d, causal)), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        fa.forward(q, k, v, scale, causal, out=o, lse=lse)
        fa.backward(q, k, v, o, do, lse, scale, causal, dq, dk, dv, workspace=ws)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        fa.forward(q, k, v, scale, causal, out=o, lse=lse)
        ev[i][1].record(stream)
        fa.backward(q, k, v, o, do, lse, scale, causal, dq, dk, dv, workspace=ws)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    if fa.check_device_status() != 0:
        raise RuntimeError("device status not OK")
    f_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    b_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    f_ms, b_ms = reduce_max([f_ms, b_ms], world, dev)
    f_fwd, f_bwd = flops(B, N, H, d, causal)
    out = {"fwd_tflops": whole_job_tflops(world, steps, f_fwd, f_ms),
           "bwd_tflops": whole_job_tflops(world, steps, f_bwd, b_ms),
           "fwd_bwd_tflops": whole_job_tflops(world, steps, f_fwd + f_bwd, f_ms + b_ms),
           "steps": steps}
    del q, k, v, do, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def config_dict(name, workload):
    B, N, H, d, dtype, causal = workload
    return {"workload": name, "batch": B, "seqlen": N, "heads": H, "head_dim": d, "dtype": dtype,
            "causal": causal, "layout": "[B,N,H,d]",
            "l2": "flushed before every step (256 MiB write), flush not timed"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the N>=4096, d=128 workloads reported beside the default one")
    ap.add_argument("--extra-steps", type=int, default=30)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    workload = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, workload)

    import torch
    import torch.distributed as dist

    import exact_attention_119_b200 as fa
    from exact_attention_119_b200 import inputs

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    B, N, H, d, dtype, causal = workload
    scale = 1.0 / math.sqrt(d)
    bits = inputs.attention_inputs(B, N, H, d, dtype, seed=rank)
    host = {k: inputs.bits_to_torch(v, dtype).pin_memory() for k, v in bits.items()}
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(max(16, fa.bwd_workspace_size(B, N, H, d, causal)), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.forward(q, k, v, scale, causal, out=o, lse=lse)
        fa.backward(q, k, v, o, do, lse, scale, causal, dq, dk, dv, workspace=ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    assert fa.check_device_status() == 0

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        fa.forward(q, k, v, scale, causal, out=o, lse=lse)
        ev[i][1].record(stream)
        fa.backward(q, k, v, o, do, lse, scale, causal, dq, dk, dv, workspace=ws)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark(t_wall0, time.time())
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    status = fa.check_device_status()
    if status != 0:
        raise RuntimeError(f"device status {fa.status_string(status)} after the timed steps")
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
    tot_ms = sum(fwd_ms) + sum(bwd_ms)
    tot_ms, fwd_sum, bwd_sum = reduce_max([tot_ms, sum(fwd_ms), sum(bwd_ms)], world, dev)

    f_fwd, f_bwd = flops(B, N, H, d, causal)
    value = whole_job_tflops(world, args.steps, f_fwd + f_bwd, tot_ms)
    fwd_tflops = whole_job_tflops(world, args.steps, f_fwd, fwd_sum)
    bwd_tflops = whole_job_tflops(world, args.steps, f_bwd, bwd_sum)

    # ---- end to end through the public API: pinned host in, results back out
    out_host = {n: torch.empty_like(host["q"]).pin_memory() for n in ("o", "dq", "dk", "dv")}
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e2e_ev[i][0].record(stream)
        q.copy_(host["q"], non_blocking=True)
        k.copy_(host["k"], non_blocking=True)
        v.copy_(host["v"], non_blocking=True)
        do.copy_(host["do"], non_blocking=True)
        step()
        out_host["o"].copy_(o, non_blocking=True)
        out_host["dq"].copy_(dq, non_blocking=True)
        out_host["dk"].copy_(dk, non_blocking=True)
        out_host["dv"].copy_(dv, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    (e2e_ms,) = reduce_max([sum(a.elapsed_time(b) for a, b in e2e_ev)], world, dev)
    if world > 1:
        dist.barrier()
    e2e_value = whole_job_tflops(world, args.steps, f_fwd + f_bwd, e2e_ms)
    tensor_bytes = B * N * H * d * 2

    # ---- the same steps back to back without the L2 flush, reported beside the headline
    nf_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        nf_ev[i][0].record(stream)
        fa.forward(q, k, v, scale, causal, out=o, lse=lse)
        nf_ev[i][1].record(stream)
        fa.backward(q, k, v, o, do, lse, scale, causal, dq, dk, dv, workspace=ws)
        nf_ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    nf_f, nf_b = reduce_max([sum(e[0].elapsed_time(e[1]) for e in nf_ev), sum(e[1].elapsed_time(e[2]) for e in nf_ev)],
                            world, dev)
    if world > 1:
        dist.barrier()
    no_flush = {"value": whole_job_tflops(world, args.steps, f_fwd + f_bwd, nf_f + nf_b),
                "fwd_tflops": whole_job_tflops(world, args.steps, f_fwd, nf_f),
                "bwd_tflops": whole_job_tflops(world, args.steps, f_bwd, nf_b), "unit": "TFLOPS",
                "note": "the same steps back to back, L2 not flushed between them"}

    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])  # fp16 and bf16 run at the same dense tensor rate
    dominant = "fa_bwd_dkdv" if bwd_sum >= fwd_sum else "fa_fwd"
    achieved = bwd_tflops if dominant == "fa_bwd_dkdv" else fwd_tflops
    traffic = NCU_TRAFFIC_BYTES.get((args.workload, dominant))

    # ---- the workloads the stated targets are quoted on (N >= 4096, d = 128):
    # same timing protocol, fewer steps, reported beside the headline.
    extra = {}
    if not args.no_extra and args.workload == DEFAULT_WORKLOAD:
        for name in EXTRA_WORKLOADS:
            extra[name] = time_workload(WORKLOADS[name], args.extra_steps, 3, dev, stream, flush, world, rank)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16" if dtype == "fp16" else "bf16",
            "data": "synthetic", "config": config_dict(args.workload, workload),
            "fwd_tflops": fwd_tflops, "bwd_tflops": bwd_tflops,
            "fwd_ms": fwd_sum / args.steps, "bwd_ms": bwd_sum / args.steps,
            "frac_of_peak": {"fwd": fwd_tflops / world / peak, "fwd_bwd": value / world / peak,
                             "peak_tflops": peak, "peak_kind": peak_kind + " bf16 dense (cuBLAS burst)",
                             "fwd_spec": fwd_tflops / world / SPEC_TFLOPS, "fwd_bwd_spec": value / world / SPEC_TFLOPS,
                             "spec_tflops": SPEC_TFLOPS},
            "no_l2_flush": no_flush,
            "roofline": {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "note": ("fa_bwd timed as one call: prep + dkdv + dq launches" if dominant == "fa_bwd_dkdv"
                                  else "one launch per call") + f"; peak {peak_kind}"},
            "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": 4 * tensor_bytes,
                    "d2h_bytes_per_step": 4 * tensor_bytes},
            "gpu_launches": 4 * args.steps,
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
            line["target_workloads"] = extra
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
