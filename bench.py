"""Throughput of the Wan full self-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one full forward call (QK^T, online softmax, PV, epilogue) over the
workload's whole batch: by default the 14B-shaped 720p clip (B=1, S=75600
tokens, H=40 heads, D=128).  The metric is attention TFLOP/s counted as
4*B*H*S^2*D per forward.  Multi-GPU (torchrun, one rank per GPU): every rank
runs its own full problem (weak scaling, no collective on the data path); the
value is the sum of all ranks' FLOPs over the slowest rank's device time.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle (fp64)
on a bounded sample of the same workload on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "attention TFLOP/s (4*B*H*S^2*D fwd)"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"bf16": d.get("bf16_tflops"), "bf16_sustained": d.get("bf16_tflops_sustained"),
                "hbm": d.get("hbm_gbs"), "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"wan_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def nvsmi_id(dev, local: int) -> str:
    """The id nvidia-smi knows this device by: its PCI bus id when torch reports one."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    bus = getattr(props, "pci_bus_id", None)
    dom = getattr(props, "pci_domain_id", None)
    dv = getattr(props, "pci_device_id", None)
    if bus is not None and dom is not None and dv is not None:
        return "%08X:%02X:%02X.0" % (dom, bus, dv)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x for x in vis.split(",") if x.strip().isdigit()]
    return ids[local] if local < len(ids) else str(local)


def cpu_baseline(w, rows_per_head: int, seed: int = 0, x=None):
    """Time the fp64 oracle on `rows_per_head` query rows of every (batch, head)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max(int(i.get("num_threads", 1)) for i in threadpool_info()) if threadpool_info() else 1
    except Exception:
        cores = os.cpu_count() or 1
    if x is None:
        x = synth.make_inputs(w, seed)
    rows = synth.sample_rows(w.S, rows_per_head, seed=seed)
    t0 = time.perf_counter()
    oracle.attn_fwd(x["q"], x["k"], x["v"], rows=rows)
    dt = time.perf_counter() - t0
    flop = 4.0 * w.B * w.H * len(rows) * w.S * w.D
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} query rows x {w.B * w.H} (batch, head) pairs of {w.name} "
                      f"against all {w.S} keys, fp64 numpy/BLAS, {dt:.2f} s"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = synth.make_inputs(w)
    rows_per_step = max(1, args.ref_rows)
    for _ in range(args.warmup):
        cpu_baseline(w, rows_per_step, x=x)
    vals = [cpu_baseline(w, rows_per_step, x=x) for _ in range(args.steps)]
    v = statistics.median(r["value"] for r in vals)
    flop_step = 4.0 * w.B * w.H * rows_per_step * w.S * w.D
    line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": flop_step / (v * 1e12) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "S": w.S, "H": w.H, "D": w.D,
                       "sample_rows_per_head": rows_per_step},
            "cpu_baseline": {**vals[0], "value": v},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import torch
    import video_dit_full_b200 as wa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wa.lib()

    # each rank gets its own seeded problem (seed = rank): weak scaling
    x = synth.make_inputs(w, seed=rank)
    shape = (w.B, w.S, w.H, w.D)

    def host_pinned(bits):
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv = (host_pinned(x[n]) for n in "qkv")
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    o = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ------------------------ device-resident timing ------------------------
    for _ in range(args.warmup):
        wa.fwd(q, k, v, o, lse)
    wa.check_status()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(nvsmi_id(dev, local))
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        wa.fwd(q, k, v, o, lse)
        ev[s][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier()
    status = wa.sync_status()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    if dist is not None:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * w.fwd_flop * args.steps / (total_ms * 1e-3) / 1e12

    # ------------------- end to end through host buffers ---------------------
    ho = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty((w.B, w.H, w.S), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        wa.fwd(q, k, v, o, lse)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if dist is not None:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * w.fwd_flop * e2e_steps / (e2e_ms * 1e-3) / 1e12
    status = status or wa.sync_status()

    if rank == 0:
        peaks = load_peaks()
        mean_launch_ms = sum(launch_ms) / len(launch_ms)
        achieved = w.fwd_flop / (mean_launch_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "S": w.S, "H": w.H, "D": w.D,
                       "fwd_flop_per_step": w.fwd_flop, "parallelism": f"replicas{world}",
                       "l2": "inputs (Q, K, V: %.2f GB) exceed the 126 MB L2; no flush" % (3 * w.B * w.S * w.H * w.D * 2 / 1e9)},
            "gpu_launches": args.steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16"], "traffic": None,
                         "peak_source": f"{peaks['source']} bf16 dense (burst)",
                         "frac_of_sustained": achieved / peaks["bf16_sustained"],
                         "kernel": "wan::fwd::attn_fwd_kernel",
                         "launch_ms": {"mean": mean_launch_ms, "min": min(launch_ms), "max": max(launch_ms)}},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 3 * w.B * w.S * w.H * w.D * 2,
                    "d2h_bytes_per_step": w.B * w.S * w.H * w.D * 2 + w.B * w.H * w.S * 4,
                    "steps": e2e_steps},
            "clocks": clocks,
            "device_status": status,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_rows, x=x)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan14b_720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-rows", type=int, default=128, help="query rows per head timed for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=8, help="query rows per head per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
