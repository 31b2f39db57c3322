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

# DRAM bytes (read + write) of one launch of the dominant kernel from an ncu capture of the
# current kernel on a smaller case (one kernel, one launch), scaled to the workload by S*H;
# absent where the kernel changed since its last capture.  The captures are summarised in
# profiles/.
TRAFFIC = {"wan14b_720p": 2.948e9, "train_480p_fwd_bwd": 3.714e9, "q8_720p": 1.599e9, "sparse8_720p": 2.927e9,
           "fp8_qkv_720p": 5.028e9}


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


def host_cores() -> dict:
    """Threads the oracle's BLAS runs on, the host's CPU count and the CPUs this process may use."""
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        blas = max(int(i.get("num_threads", 1)) for i in info) if info else 1
    except Exception:  # noqa: BLE001
        blas = os.cpu_count() or 1
    try:
        allowed = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        allowed = os.cpu_count() or 1
    return {"cores": blas, "nproc": os.cpu_count() or 1, "cpus_allowed": allowed}


def _baseline(flop, dt, sample, full_flop, cores) -> dict:
    rate = flop / dt
    rec = {"value": rate / 1e12, "unit": "TFLOP/s", **cores, "kind": "oracle", "sample": sample,
           "sample_s": dt, "_flop": flop}
    if flop >= full_flop * (1 - 1e-12):
        rec["full_problem_s"] = dt
    else:
        rec["full_problem_s_extrapolated"] = full_flop / rate
        rec["extrapolation"] = "the workload's full count of the metric's FLOPs at the sample's measured rate"
    return rec


def cpu_baseline(w, rows_per_head: int, seed: int = 0, x=None):
    """Time the fp64 oracle on `rows_per_head` query rows of every (batch, head): a bounded
    sample of the workload, with the full problem's time extrapolated from its rate."""
    import oracle
    cores = host_cores()
    if w.gemm:
        from oracle import fp8_gemm
        M, N, K = w.gemm
        if x is None:
            x = gemm_inputs(w, seed)
        rows = synth.sample_rows(M, rows_per_head, seed=seed)
        t0 = time.perf_counter()
        _, xv, sx = fp8_gemm.quant_rows(x["x"][rows])        # per-token: each row on its own
        _, wv, sw = fp8_gemm.quant_tensor(x["w"])
        fp8_gemm.gemm_from_codes(xv, sx, wv, sw)
        dt = time.perf_counter() - t0
        flop = 2.0 * len(rows) * N * K
        return _baseline(flop, dt, f"{len(rows)} token rows of {w.name} (quantised) against the whole quantised "
                                   f"{N} x {K} weight, fp64 numpy/BLAS, {dt:.2f} s", w.fwd_flop, cores)
    if w.sparse_keep:
        from oracle import block_sparse
        if x is None:
            x = synth.make_inputs(w, seed)
        nb = (w.S + 63) // 64
        mask = synth.block_mask(w.B, w.H, nb, nb, w.sparse_keep, seed=seed)
        rows = synth.sample_rows(w.S, rows_per_head, seed=seed)
        size = np.minimum(64, w.S - 64 * np.arange(nb)).astype(np.float64)
        t0 = time.perf_counter()
        block_sparse.attn_fwd_block_sparse(x["q"], x["k"], x["v"], mask, rows=rows)
        dt = time.perf_counter() - t0
        flop = float(4.0 * w.D * (mask[:, :, rows // 64, :].astype(np.float64) @ size).sum())
        full = float(4.0 * w.D * np.einsum("bhij,i,j->", mask.astype(np.float64), size, size))
        return _baseline(flop, dt, f"{len(rows)} query rows x {w.B * w.H} (batch, head) pairs of {w.name} against "
                                   f"their allowed key blocks (fp64, masked dense rows), {dt:.2f} s", full, cores)
    if x is None:
        x = synth.make_inputs(w, seed)
    rows = synth.sample_rows(w.S, rows_per_head, seed=seed)
    full = w.fwd_flop * (3.5 if w.backward else 1.0)
    if w.backward:
        # the rows' forward and their dQ (scores recomputed, dP, dS K): 10 * Skv * D per row
        t0 = time.perf_counter()
        oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], q_rows=rows, k_rows=[])
        dt = time.perf_counter() - t0
        flop = 10.0 * w.B * w.H * len(rows) * w.kv_len * w.D
        return _baseline(flop, dt, f"forward + dQ of {len(rows)} query rows x {w.B * w.H} (batch, head) pairs of "
                                   f"{w.name} against all {w.kv_len} keys, fp64 numpy/BLAS, {dt:.2f} s", full, cores)
    t0 = time.perf_counter()
    oracle.attn_fwd(x["q"], x["k"], x["v"], rows=rows)
    dt = time.perf_counter() - t0
    flop = 4.0 * w.B * w.H * len(rows) * w.kv_len * w.D
    what = "exact (unquantised) forward" if w.q8 else "forward"
    return _baseline(flop, dt, f"{what} of {len(rows)} query rows x {w.B * w.H} (batch, head) pairs of {w.name} "
                               f"against all {w.kv_len} keys, fp64 numpy/BLAS, {dt:.2f} s", full, cores)


def metric_of(w) -> str:
    if w.sparse_keep:
        return "block-sparse attention TFLOP/s (4*D*64*64 per allowed 64x64 block)"
    if w.gemm:
        return "FP8 GEMM TFLOP/s (2*M*N*K, e4m3 x e4m3 -> fp32)"
    if w.cp:
        return f"{w.cp} context-parallel attention TFLOP/s per rank (4*B*H*S^2*D / {w.cp_ranks})"
    if w.cross:
        return ("cross-attention TFLOP/s (fwd 4*B*H*S*Skv*D + bwd 2.5x fwd)" if w.backward
                else "cross-attention TFLOP/s (4*B*H*S*Skv*D)")
    return METRIC if not w.backward else "attention TFLOP/s (fwd 4*B*H*S^2*D + bwd 2.5x fwd)"


def workload_config(w) -> dict:
    c = {"workload": w.name, "B": w.B, "S": w.S, "H": w.H, "D": w.D}
    if w.cross:
        c["Skv"] = w.kv_len
    if w.cp:
        c.update(cp=w.cp, cp_ranks=w.cp_ranks, cp_note="one rank's kernels; the exchanges are not run")
    if w.gemm:
        c = {"workload": w.name, "M": w.gemm[0], "N": w.gemm[1], "K": w.gemm[2]}
    return c


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = gemm_inputs(w, 0) if w.gemm else synth.make_inputs(w)
    rows_per_step = max(1, args.ref_rows)
    for _ in range(args.warmup):
        cpu_baseline(w, rows_per_step, x=x)
    vals = [cpu_baseline(w, rows_per_step, x=x) for _ in range(args.steps)]
    v = statistics.median(r["value"] for r in vals)
    flop_step = vals[0].pop("_flop")
    for r in vals[1:]:
        r.pop("_flop")
    line = {"metric": metric_of(w), "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": flop_step / (v * 1e12) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {**workload_config(w), "sample_rows_per_head": rows_per_step},
            "cpu_baseline": {**vals[0], "value": v},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """The largest of every rank's device-timed milliseconds (all ranks take part)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flop_per_rank_step: float, steps: int, slowest_ms: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time (weak scaling)."""
    return world * flop_per_rank_step * steps / (slowest_ms * 1e-3) / 1e12


def bwd_splits(w, dev) -> bool:
    """Whether the cross-attention backward spreads each key tile over several CTAs: it does
    when the key tiles alone give fewer than 4 waves of CTAs on the device's SMs."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return -(-w.kv_len // 128) * w.H * w.B < 4 * sms


class Path:
    """The calls one bench step makes for a workload, with their buffers.

    fwd workloads: one wan_attn_fwd; the training workload: wan_attn_fwd then
    wan_attn_bwd; the 8-bit workload: one wan_attn_fwd_q8 (quantise + attend);
    the cross-attention workloads: wan_attn_cross_fwd (then wan_attn_cross_bwd).
    """

    def __init__(self, wa, w, dev, x):
        import torch
        self.wa, self.w = wa, w
        shape = (w.B, w.S, w.H, w.D)
        kv_shape = (w.B, w.kv_len, w.H, w.D)

        def pinned(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

        names = ["q", "k", "v"] + (["do"] if w.backward else [])
        self.host_in = [pinned(x[n]) for n in names]
        self.dev_in = [t.to(dev) for t in self.host_in]
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.o = torch.empty(shape, **bf)
        self.lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
        self.outs = [self.o, self.lse]
        self.ws = None
        if w.backward:
            self.grads = [torch.empty(shape, **bf), torch.empty(kv_shape, **bf), torch.empty(kv_shape, **bf)]
            ws_bytes = (wa.cross_bwd_workspace_size(w.B, w.S, w.kv_len, w.H, w.D) if w.cross
                        else wa.bwd_workspace_size(w.B, w.S, w.H, w.D))
            self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            self.outs = self.outs + self.grads
            self.flop = 3.5 * w.fwd_flop                   # forward + 2.5x forward for the backward
            self.dominant_flop = 2.5 * w.fwd_flop
            call = "wan_attn_cross_bwd" if w.cross else "wan_attn_bwd"
            self.kernel = f"wan::bwd::bwd_main_kernel (timed with its prep and finalise kernels: one {call} call)"
            # fwd + prep + main + dQ; a split key tile adds the dK and dV finalise kernels
            self.launches_per_step = 4 + (2 if w.cross and bwd_splits(w, dev) else 0)
            self.peak_key, self.dtype = "bf16", "bf16"
        elif w.q8:
            self.ws = torch.empty(wa.fwd_q8_workspace_size(w.B, w.S, w.H, w.D), dtype=torch.uint8, device=dev)
            self.flop = w.fwd_flop
            self.dominant_flop = w.fwd_flop
            self.kernel = "wan::q8::q8_attn_kernel (timed with its quantise kernel: one wan_attn_fwd_q8 call)"
            self.launches_per_step = 2
            self.peak_key, self.dtype = "fp8", "int8/e4m3"
        else:
            self.flop = w.fwd_flop
            self.dominant_flop = w.fwd_flop
            if w.cross and w.kv_len != w.S and w.kv_len <= 1024:   # the short-key cross forward's kernel
                self.kernel = "wan::sparse::pair::attn_fwd_pair_kernel<true, true>, every key block (wan_attn_cross_fwd)"
            else:
                self.kernel = "wan::fwd::attn_fwd_kernel" + (" (wan_attn_cross_fwd)" if w.cross else "")
            self.launches_per_step = 1
            self.peak_key, self.dtype = "bf16", "bf16"
        self.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host_in)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.host_out)

    def step(self, dom_events=None, fwd_event=None):
        wa, (q, k, v) = self.wa, self.dev_in[:3]
        fwd = wa.cross_fwd if self.w.cross else wa.fwd
        if self.w.backward:
            if fwd_event is not None:
                fwd_event.record()
            fwd(q, k, v, self.o, self.lse)
            if dom_events:
                dom_events[0].record()
            bwd = wa.cross_bwd if self.w.cross else wa.bwd
            bwd(q, k, v, self.o, self.dev_in[3], self.lse, *self.grads, workspace=self.ws)
        else:
            if dom_events:
                dom_events[0].record()
            if self.w.q8:
                wa.fwd_q8(q, k, v, self.o, self.lse, workspace=self.ws)
            else:
                fwd(q, k, v, self.o, self.lse)
        if dom_events:
            dom_events[1].record()

    def h2d(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)

    def d2h(self):
        for h, d in zip(self.host_out, self.outs):
            h.copy_(d, non_blocking=True)

    def share_host(self, other):
        """Use another instance's pinned host buffers (the same inputs; outputs land in one place)."""
        self.host_in, self.host_out = other.host_in, other.host_out


class CpPath:
    """One rank's compute of a G-way context split (Ring or Ulysses) on this GPU.

    The other ranks' shards are already resident, so the exchanges (NCCL on a real
    split) are not part of the step: it is the per-rank kernel work only.
    ring:    G x (wan_attn_cross_fwd of the rank's S/G queries against one key block
             + wan_attn_cp_merge into the fp32 running result).
    ulysses: wan_attn_cp_layout of the q, k, v shards into send order, wan_attn_fwd on
             all S tokens of the rank's H/G heads, wan_attn_cp_layout of O back into
             sequence order (B = 1: the head-side permutations are identities).
    """

    def __init__(self, wa, w, dev, x):
        import torch
        self.wa, self.w = wa, w
        G, B, S, H, D = w.cp_ranks, w.B, w.S, w.H, w.D
        if B != 1 or S % G or H % G:
            raise ValueError("context-parallel workloads need B = 1, S and H divisible by the ranks")
        self.G, self.S_loc, self.Hg = G, S // G, H // G

        def dev_bf16(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

        full = [dev_bf16(x[n]) for n in ("q", "k", "v")]
        sl = slice(0, self.S_loc)
        # this rank's own shards (its tokens 0..S/G-1 with every head): what e2e copies in
        self.host_in = [torch.from_numpy(np.ascontiguousarray(x[n][:, sl]).view(np.int16)).view(torch.bfloat16)
                        .pin_memory() for n in ("q", "k", "v")]
        bf = dict(dtype=torch.bfloat16, device=dev)
        if w.cp == "ring":
            self.dev_in = [t[:, sl] for t in full]           # views of the resident tensors (B = 1)
            self.blocks = [(full[1][:, j * self.S_loc:(j + 1) * self.S_loc],
                            full[2][:, j * self.S_loc:(j + 1) * self.S_loc]) for j in range(G)]
            self.o = torch.empty((B, self.S_loc, H, D), **bf)
            self.o_acc = torch.empty(self.o.shape, dtype=torch.float32, device=dev)
            self.lse = torch.empty((B, H, self.S_loc), dtype=torch.float32, device=dev)
            self.outs = [self.o, self.lse]
            self.kernel = ("wan::fwd::attn_fwd_kernel + wan::cp::cp_merge_kernel (one rank's 8 key blocks: "
                           "wan_attn_cross_fwd + wan_attn_cp_merge each)")
            self.launches_per_step = 2 * G
        else:
            self.dev_in = [t[:, sl].contiguous() for t in full]   # own shards, [B, S/G, H, D]
            # all tokens of this rank's head group, as the all-to-all would deliver them
            self.heads = [t[:, :, :self.Hg].contiguous() for t in full]
            self.send = [torch.empty((G, B, self.S_loc, self.Hg, D), **bf) for _ in range(3)]
            self.o_heads = torch.empty((B, S, self.Hg, D), **bf)
            self.lse_h = torch.empty((B, self.Hg, S), dtype=torch.float32, device=dev)
            self.o = torch.empty((B, self.S_loc, H, D), **bf)
            self.outs = [self.o]
            self.kernel = ("wan::fwd::attn_fwd_kernel + wan::cp::cp_layout_kernel (one rank: 3 layouts in, "
                           "attention on its 5 heads x all tokens, 1 layout out)")
            self.launches_per_step = 5
        del full
        self.flop = w.fwd_flop
        self.dominant_flop = w.fwd_flop
        self.peak_key, self.dtype = "bf16", "bf16"
        self.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host_in)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.host_out)

    def step(self, dom_events=None):
        wa = self.wa
        if dom_events:
            dom_events[0].record()
        if self.w.cp == "ring":
            q = self.dev_in[0]
            for j, (k, v) in enumerate(self.blocks):
                o_t, lse_t = wa.cross_fwd(q, k, v)
                wa.cp_merge(self.o_acc, self.lse, o_t, lse_t, j == 0, self.o if j + 1 == self.G else None)
        else:
            G, B, S_loc, Hg = self.G, self.w.B, self.S_loc, self.Hg
            for send, shard in zip(self.send, self.dev_in):
                wa.cp_layout(send, shard, B, S_loc, G, Hg, wa.CP_SEQ_TO_SEND)
            wa.fwd(*self.heads, self.o_heads, self.lse_h)
            # o_heads in [B, G*S_loc, Hg, D] is already the send order for B = 1
            wa.cp_layout(self.o, self.o_heads, B, S_loc, G, Hg, wa.CP_RECV_TO_SEQ)
        if dom_events:
            dom_events[1].record()

    def h2d(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)

    def d2h(self):
        for h, d in zip(self.host_out, self.outs):
            h.copy_(d, non_blocking=True)

    def share_host(self, other):
        """Use another instance's pinned host buffers (the same inputs; outputs land in one place)."""
        self.host_in, self.host_out = other.host_in, other.host_out


class GemmPath:
    """The FP8 linear layer: wan_fp8_quantize_rows of the bf16 activations X [M, K] (per token),
    then wan_fp8_gemm with a weight W [N, K] quantised once beforehand (per tensor), as at
    inference time."""

    def __init__(self, wa, w, dev, x):
        import torch
        self.wa, self.w = wa, w
        M, N, K = w.gemm

        def pinned(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

        self.host_in = [pinned(x["x"])]
        self.dev_in = [t.to(dev) for t in self.host_in]
        self.w_codes, self.w_scale2 = wa.fp8_quantize_tensor(pinned(x["w"]).to(dev))
        self.codes = torch.empty((M, K), dtype=torch.uint8, device=dev)
        self.scales = torch.empty(M, dtype=torch.float32, device=dev)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.outs = [self.y]
        self.flop = w.fwd_flop
        self.dominant_flop = w.fwd_flop
        self.kernel = "wan::fp8::fp8_gemm_pair_kernel (timed with the per-token quantiser: one FP8 linear layer)"
        self.launches_per_step = 2
        self.peak_key, self.dtype = "fp8", "e4m3"
        self.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host_in)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.host_out)

    def step(self, dom_events=None):
        wa = self.wa
        if dom_events:
            dom_events[0].record()
        wa.fp8_quantize_rows(self.dev_in[0], self.codes, self.scales)
        wa.fp8_gemm(self.codes, self.scales, self.w_codes, self.w_scale2[:1], self.y)
        if dom_events:
            dom_events[1].record()

    def h2d(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)

    def d2h(self):
        for h, d in zip(self.host_out, self.outs):
            h.copy_(d, non_blocking=True)

    def share_host(self, other):
        """Use another instance's pinned host buffers (the same inputs; outputs land in one place)."""
        self.host_in, self.host_out = other.host_in, other.host_out


def union_fraction(mask):
    """Fraction of (Q tile, key block) pairs a CTA computes: each 128-row Q tile walks the union of
    the key blocks its two 64-row query blocks attend (a short last tile has one)."""
    nqb = mask.shape[2]
    m2 = np.pad(mask, ((0, 0), (0, 0), (0, nqb % 2), (0, 0)))
    return float(m2.reshape(mask.shape[0], mask.shape[1], -1, 2, mask.shape[3]).max(axis=3).mean())


class SparsePath:
    """Block-sparse attention: one wan_attn_fwd_block_sparse over a seeded 64 x 64 block mask.
    `flop` counts only the allowed blocks (4 * D * |query block| * |key block| each); the
    dense-equivalent count and the fraction of key blocks the CTAs' unions cover are reported
    beside it."""

    def __init__(self, wa, w, dev, x):
        import torch
        self.wa, self.w = wa, w
        shape = (w.B, w.S, w.H, w.D)

        def pinned(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

        nb = (w.S + 63) // 64
        self.mask_host = synth.block_mask(w.B, w.H, nb, nb, w.sparse_keep, seed=x["seed"])
        size = np.minimum(64, w.S - 64 * np.arange(nb)).astype(np.float64)
        self.flop = float(4.0 * w.D * np.einsum("bhij,i,j->", self.mask_host.astype(np.float64), size, size))
        self.dense_flop = w.fwd_flop
        self.union_frac = union_fraction(self.mask_host)
        self.host_in = [pinned(x[n]) for n in ("q", "k", "v")]
        self.dev_in = [t.to(dev) for t in self.host_in]
        self.mask = torch.from_numpy(self.mask_host).to(dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.o = torch.empty(shape, **bf)
        self.lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
        self.ws = torch.empty(wa.block_sparse_workspace_size(w.B, w.S, w.S, w.H, w.D), dtype=torch.uint8,
                              device=dev)
        self.outs = [self.o, self.lse]
        self.dominant_flop = self.flop
        self.kernel = ("wan::sparse::pair::attn_fwd_pair_kernel<false, false> (with its per-tile key-block list "
                       "kernel: one wan_attn_fwd_block_sparse)")
        self.launches_per_step = 2
        self.peak_key, self.dtype = "bf16", "bf16"
        self.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host_in)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.host_out)

    def step(self, dom_events=None):
        if dom_events:
            dom_events[0].record()
        q, k, v = self.dev_in
        self.wa.fwd_block_sparse(q, k, v, self.mask, self.o, self.lse, workspace=self.ws)
        if dom_events:
            dom_events[1].record()

    def h2d(self):
        for d, h in zip(self.dev_in, self.host_in):
            d.copy_(h, non_blocking=True)

    def d2h(self):
        for h, d in zip(self.host_out, self.outs):
            h.copy_(d, non_blocking=True)

    def share_host(self, other):
        """Use another instance's pinned host buffers (the same inputs; outputs land in one place)."""
        self.host_in, self.host_out = other.host_in, other.host_out


def e2e_pipelined(paths, steps, dev) -> float:
    """Device milliseconds of `steps` end-to-end steps over the two buffer sets in `paths`:
    host-to-device copy (stream 1), the step's kernels (stream 2), device-to-host copy (stream 3);
    a buffer set is refilled only after its previous step's kernels and read-back are done."""
    import torch
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    cmp_done, out_done = [None] * steps, [None] * steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        p = paths[i % 2]
        if i >= 2:
            s_in.wait_event(cmp_done[i - 2])           # the set's inputs are free again
        with torch.cuda.stream(s_in):
            p.h2d()
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        s_cmp.wait_event(in_done)
        if i >= 2:
            s_cmp.wait_event(out_done[i - 2])          # the set's outputs have been read back
        with torch.cuda.stream(s_cmp):
            p.step()
        cmp_done[i] = torch.cuda.Event()
        cmp_done[i].record(s_cmp)
        s_out.wait_event(cmp_done[i])
        with torch.cuda.stream(s_out):
            p.d2h()
        out_done[i] = torch.cuda.Event()
        out_done[i].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1)


def make_path(wa, w, dev, x):
    if w.sparse_keep:
        return SparsePath(wa, w, dev, x)
    if w.gemm:
        return GemmPath(wa, w, dev, x)
    if w.cp:
        return CpPath(wa, w, dev, x)
    return Path(wa, w, dev, x)


def gemm_inputs(w, seed):
    M, N, K = w.gemm
    return {"x": synth.make_tensor((M, K), seed, synth.STREAM_Q), "w": synth.make_tensor((N, K), seed, synth.STREAM_K)}


# The configurations quoted beside the headline one: each gets its own record in the
# line's "extra" object (timed on its own, with its own clocks and CPU-oracle sample).
# Values: (timed steps, oracle query rows per (batch, head) for its cpu_baseline).
EXTRA_WORKLOADS = {"oracle_1280": (200, 1280), "wan1.3b_480p_cfg": (20, 16),
                   "train_480p_fwd_bwd": (8, 16), "q8_720p": (10, 16)}


def measure_8bit_peaks(dev, n: int = 8192, reps: int = 10) -> dict:
    """Dense 8-bit tensor throughput of this GPU through the vendor library, as the bf16 peak
    beside it was measured: an e4m3 x e4m3 -> bf16 torch._scaled_mm and an int8 x int8 -> int32
    torch._int_mm of n^3 (2 n^3 operations), best of `reps` launches after warm-up, CUDA events."""
    import torch
    out = {"shape": f"{n}x{n}x{n}", "how": f"best of {reps} launches after 3 warm-ups, CUDA events"}

    def best_rate(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12

    g = torch.Generator(device=dev)
    g.manual_seed(0)
    try:
        a = (torch.randn(n, n, device=dev, generator=g)).to(torch.float8_e4m3fn)
        b = (torch.randn(n, n, device=dev, generator=g)).to(torch.float8_e4m3fn).t()   # column-major
        one = torch.ones((), device=dev)
        out["fp8_e4m3_tflops"] = best_rate(lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,
                                                                     out_dtype=torch.bfloat16))
        del a, b
    except Exception as e:  # noqa: BLE001 - report, do not fail the bench
        out["fp8_e4m3_error"] = f"{type(e).__name__}: {e}"[:200]
    try:
        ai = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
        bi = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
        rates = {"row_major_b": best_rate(lambda: torch._int_mm(ai, bi))}
        bt = bi.t().contiguous().t()                                                    # column-major
        rates["col_major_b"] = best_rate(lambda: torch._int_mm(ai, bt))
        out["int8_tops"] = max(rates.values())
        out["int8_by_layout"] = rates
        del ai, bi, bt
    except Exception as e:  # noqa: BLE001
        out["int8_error"] = f"{type(e).__name__}: {e}"[:200]
    torch.cuda.empty_cache()
    return out


def peak_for(path, peaks, p8) -> tuple:
    """(burst peak, sustained peak or None, description) for the path's dominant kernel."""
    if path.peak_key != "fp8":
        return peaks["bf16"], peaks["bf16_sustained"], f"{peaks['source']} bf16 dense (burst)"
    fp8, i8 = p8.get("fp8_e4m3_tflops"), p8.get("int8_tops")
    if isinstance(path, GemmPath):
        if fp8:
            return fp8, None, "measured e4m3 torch._scaled_mm 8192^3 (burst), this run"
    elif fp8 and i8:
        # half of the 8-bit forward's operations are int8 (Q K^T), half e4m3 (P V): time adds
        eff = 2.0 / (1.0 / i8 + 1.0 / fp8)
        return eff, None, ("measured, this run: 2 / (1/int8 + 1/e4m3) of torch._int_mm and "
                           "torch._scaled_mm 8192^3 (burst); half the operations are int8 Q K^T, half e4m3 P V")
    return (2.0 * peaks["bf16"], 2.0 * peaks["bf16_sustained"],
            f"{peaks['source']} bf16 dense burst x 2 (nominal 8-bit : bf16 ratio; no 8-bit peak measured)")


def time_device(path, steps, warmup, dev, wa, gpu_id, barrier=lambda: None, flush=None) -> dict:
    """Warm-up, then `steps` steps between CUDA events on the launching stream (synchronised
    on both sides), the dominant call timed per step, clocks sampled during the timed region.
    `flush`: a device buffer larger than the L2, overwritten between steps (outside the
    per-step events) when the workload's inputs would otherwise stay in the L2."""
    import torch
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        path.step()
    status = wa.sync_status()
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [(mk(), mk()) for _ in range(steps)]
    fwd_ev = [mk() for _ in range(steps)] if isinstance(path, Path) and path.w.backward else None
    sampler = ClockSampler(gpu_id)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    t_start, t_end = mk(), mk()
    t_start.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        if fwd_ev:
            path.step(ev[i], fwd_ev[i])
        else:
            path.step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier()
    status = status or wa.sync_status()
    return {"total_ms": t_start.elapsed_time(t_end), "dom_ms": [a.elapsed_time(b) for a, b in ev],
            "fwd_ms": [f.elapsed_time(a) for f, (a, _) in zip(fwd_ev, ev)] if fwd_ev else None,
            "clocks": clocks, "status": status}


def roofline_of(path, w, t, peaks, p8) -> dict:
    mean_ms = sum(t["dom_ms"]) / len(t["dom_ms"])
    achieved = path.dominant_flop / (mean_ms * 1e-3) / 1e12
    peak, sustained, src = peak_for(path, peaks, p8)
    r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
         "traffic": TRAFFIC.get(w.name), "peak_source": src}
    if sustained:
        r["frac_of_sustained"] = achieved / sustained
    r["kernel"] = path.kernel
    r["launch_ms"] = {"mean": mean_ms, "min": min(t["dom_ms"]), "max": max(t["dom_ms"])}
    return r


def extra_record(wa, name, dev, gpu_id, peaks, p8, warmup, no_cpu) -> dict:
    """One configuration beside the headline: timed alone, with its own roofline, clocks and
    a bounded CPU-oracle sample."""
    import torch
    w = synth.WORKLOADS[name]
    steps, cpu_rows = EXTRA_WORKLOADS[name]
    x = synth.make_inputs(w, seed=0)
    x["seed"] = 0
    path = make_path(wa, w, dev, x)
    in_bytes = sum(t_.numel() * t_.element_size() for t_ in path.dev_in)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < 126e6 else None
    t = time_device(path, steps, max(3, warmup), dev, wa, gpu_id, flush=flush)
    # with an L2 flush between steps, a step's time is its own events' (the flush is outside them)
    step_ms = sum(t["dom_ms"]) / steps if flush is not None else t["total_ms"] / steps
    rec = {"metric": metric_of(w), "value": path.flop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "steps": steps, "warmup": max(3, warmup), "ms_per_step": step_ms, "dtype": path.dtype,
           "config": {**workload_config(w), "flop_per_step": path.flop}, "gpu_launches": steps * path.launches_per_step,
           "roofline": roofline_of(path, w, t, peaks, p8), "clocks": t["clocks"], "device_status": t["status"]}
    if t["fwd_ms"]:
        fwd_ms = sum(t["fwd_ms"]) / len(t["fwd_ms"])
        bwd_ms = rec["roofline"]["launch_ms"]["mean"]
        rec["split"] = {"fwd_ms": fwd_ms, "fwd_tflops": w.fwd_flop / (fwd_ms * 1e-3) / 1e12,
                        "bwd_ms": bwd_ms, "bwd_tflops": 2.5 * w.fwd_flop / (bwd_ms * 1e-3) / 1e12,
                        "bwd_flop_count": "2.5 x the forward's 4*B*H*S^2*D (the pages' beta: 2x)"}
    if w.S < 148 * 256:
        rec["config"]["note"] = "latency-bound: fewer Q-tile CTAs than one wave of the 148 SMs"
    rec["config"]["l2"] = ("inputs (%.1f MB) fit in the 126 MB L2: a 256 MB buffer is overwritten between "
                           "steps, outside each step's events" % (in_bytes / 1e6) if flush is not None
                           else "inputs (%.2f GB) exceed the 126 MB L2; no flush" % (in_bytes / 1e9))
    del path, flush
    torch.cuda.empty_cache()
    if not no_cpu:
        cb = cpu_baseline(w, cpu_rows, x=x)
        cb.pop("_flop")
        rec["cpu_baseline"] = cb
    return rec


def run_ours(args, w):
    import torch
    import video_dit_full_b200 as wa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    wa.lib()
    gpu_id = nvsmi_id(dev, local)

    # each rank gets its own seeded problem (seed = rank): weak scaling
    x = gemm_inputs(w, rank) if w.gemm else synth.make_inputs(w, seed=rank)
    x["seed"] = rank
    path = make_path(wa, w, dev, x)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ------------------------ device-resident timing ------------------------
    t = time_device(path, args.steps, args.warmup, dev, wa, gpu_id, barrier)
    status = t["status"]
    total_ms = max_over_ranks(t["total_ms"], dist, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(world, path.flop, args.steps, total_ms)

    # ------------------- end to end through host buffers ---------------------
    # Every step copies its inputs from pinned host memory and its outputs back.  Two device
    # buffer sets alternate, so step i's kernels overlap step i+1's host-to-device copy and step
    # i-1's device-to-host copy (three streams, ordered by events).
    e2e_steps = max(2, args.steps)                    # as many steps as the device-resident timing
    twin = make_path(wa, w, dev, x)
    twin.share_host(path)
    paths = (path, twin)
    e2e_pipelined(paths, 2, dev)                       # warm-up of the streams and buffers
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e2e_pipelined(paths, e2e_steps, dev), dist, dev)
    del twin, paths
    e2e_value = whole_job_tflops(world, path.flop, e2e_steps, e2e_ms)
    status = status or wa.sync_status()

    if rank == 0:
        peaks = load_peaks()
        p8 = measure_8bit_peaks(dev) if world == 1 and (path.peak_key == "fp8" or not args.no_extra) else {}
        in_gb = sum(t_.numel() * t_.element_size() for t_ in path.dev_in) / 1e9
        line = {
            "metric": metric_of(w),
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": path.dtype, "data": "synthetic",
            "config": {**workload_config(w),
                       "flop_per_step": path.flop, "parallelism": f"replicas{world}",
                       "l2": "inputs (%.2f GB) exceed the 126 MB L2; no flush" % in_gb},
            "gpu_launches": args.steps * path.launches_per_step,
            **({"sparse": {"keep": w.sparse_keep, "union_fraction_computed": path.union_frac,
                           "dense_equivalent_tflops": whole_job_tflops(world, path.dense_flop, args.steps, total_ms),
                           # the rate of the tensor work the tiles do: every key block of a tile's union
                           "union_tflops": whole_job_tflops(world, path.union_frac * path.dense_flop, args.steps,
                                                            total_ms)}}
               if w.sparse_keep else {}),
            "roofline": roofline_of(path, w, t, peaks, p8),
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": path.h2d_bytes,
                    "d2h_bytes_per_step": path.d2h_bytes, "steps": e2e_steps,
                    "pipelined": "two buffer sets; each step's copies overlap the neighbouring steps' kernels; "
                                 "the first step's input copy and the last step's read-back are not overlapped"},
            "clocks": t["clocks"],
            "device_status": status,
        }
        if p8:
            line["peaks_8bit"] = p8
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_rows, x=x)
            line["cpu_baseline"].pop("_flop")
        if world == 1 and not args.no_extra:
            del path
            x = None
            torch.cuda.empty_cache()
            line["extra"] = {}
            for name in EXTRA_WORKLOADS:
                if name == w.name:
                    continue
                rec = extra_record(wa, name, dev, gpu_id, peaks, p8, args.warmup, args.no_cpu_baseline)
                status = status or rec["device_status"]
                line["extra"][name] = rec
            line["device_status"] = status
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
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations' records (and the 8-bit peak measurement)")
    ap.add_argument("--S", type=int, default=None, help="override the token count (small profiling cases)")
    ap.add_argument("--H", type=int, default=None, help="override the head count (small profiling cases)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.S or args.H:
        import dataclasses
        gemm = (args.S or w.gemm[0],) + tuple(w.gemm[1:]) if w.gemm else None   # --S sets a GEMM's M
        w = dataclasses.replace(w, S=args.S or w.S, H=args.H or w.H, gemm=gemm,
                                name=f"{w.name}@S{args.S or w.S}H{args.H or w.H}")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
