#!/usr/bin/env python
"""Benchmark of the SLA2 inference forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one sla2_forward call (router, linear state, sparse branch,
epilogue) on the Wan2.1-1.3B-480P attention shape: B=1, H=12, N=32768, d=128,
k% = 3 (97% sparse), seeded synthetic bf16 inputs resident in HBM. Q/K/V are
302 MB together, larger than the 126 MB L2, so no flush is needed between
steps. `value` is the dense-equivalent throughput 4 B H N^2 d / t (TOPS),
summed over ranks; each rank runs its own replica (the pass needs no
collective). Per-stage times come from CUDA events recorded by the library
on the launch stream at stage boundaries.

--impl reference times the CPU oracle (the reference arm of this build) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SLA2 fwd ms & effective TOPS @N=32768,H=12,d=128,97% sparse; % of roofline"
WORKLOAD = "wan1.3b"

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_8BIT_OVER_BF16 = 4.5 / 2.25   # dense FP8/INT8 : dense bf16 (nominal ratio)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def work_model(w, k):
    """Algorithmic work of one forward pass: bytes of the HBM-bound stages, 8-bit ops
    of the sparse branch and fp16 flops of the epilogue, per the definitions below."""
    B, H, N, d = w.B, w.H, w.N, w.d
    BH, nq, nk = B * H, N // 128, N // 64
    E = BH * N * d
    pairs = BH * nq * k
    return {
        "pairs": pairs,
        "sparse_ops": pairs * 4 * 128 * 64 * d,
        "effective_ops": 4 * B * H * N * N * d,
        # router: read Q, K, V (bf16), write Q-hat (int8)
        "router_bytes": 2 * E * 3 + E,
        # linear state: read K, V (bf16), write K-hat, V-hat^T (8-bit), h_j^T tiles (fp16), z_j (fp32)
        "linear_bytes": 2 * E * 2 + 2 * E + BH * nk * d * d * 2 + BH * nk * d * 4,
        # epilogue: read Q (bf16), O_s (fp32), h_j^T tiles once (fp16), write out (bf16); the
        # repeated tile gather (k + 1 per query block) is L2 traffic, reported separately
        "epilogue_bytes": 2 * E + 4 * E + 2 * E + BH * nk * d * d * 2,
        "gather_bytes": BH * nq * (k + 1) * d * d * 2,   # per query block: H_total and the k selected h_j tiles
        # epilogue MMAs: phi(Q_i) (128 x d) times k + 1 tiles (d x d), fp16 in, fp32 accumulate
        "epilogue_flops": BH * nq * (k + 1) * 2 * 128 * d * d if k < nk else 0,
    }


# DRAM bytes per launch measured by ncu (summaries under profiles/), valid only for the
# kernel source they were taken on: sha256 prefix of the kernel file + device.cuh + kernels.cuh.
MEASURED_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum, --set full capture
    "sparse": ("sparse.cu", "3a73ccef7b0d189c", 298.1e6, "ncu dram__bytes_read.sum + dram__bytes_write.sum"),
    # dram__bytes.sum.per_second x gpu__time_duration.sum, section captures
    "epilogue": ("epilogue.cu", "1b0cc1424c18eeed", 596.3e6, "ncu dram__bytes.sum.per_second x duration"),
    "linear_state": ("linear.cu", "67c76cddfc1bdc85", 471.3e6, "ncu dram__bytes.sum.per_second x duration"),
    "router": ("router.cu", "4eadfd52602acf06", 345.5e6, "ncu dram__bytes.sum.per_second x duration (pool_kernel)"),
}


def measured_traffic(name):
    """(bytes, source) of the ncu capture for this stage's kernel, or (None, None) once the
    kernel source differs from the one that was profiled."""
    import hashlib
    if name not in MEASURED_TRAFFIC:
        return None, None
    f, sha, b, src = MEASURED_TRAFFIC[name]
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_linear_router_b200", "csrc")
    h = hashlib.sha256()
    try:
        for part in (f, "device.cuh", "kernels.cuh"):
            with open(os.path.join(csrc, part), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None, None
    return (b, src) if h.hexdigest()[:16] == sha else (None, None)


def launches_per_forward(w, k):
    """Kernels one forward launches: router 5 (pool, column means, both projections in
    one launch, logits, top-k), linear state 2, sparse 1, Z_i 1 and epilogue 1 (no Z_i
    pass when every key block is selected)."""
    return 5 + 2 + 1 + (2 if k < w.N // 64 else 1)


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(x, dist, device):
    """The slowest rank's value: a MAX all-reduce that every rank takes part in (the
    job's time is the time of its slowest rank)."""
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ops_per_step, ms_per_step, world_size):
    """Whole-job throughput in TOPS: every rank runs one replica of the workload per
    step, and the step time is the slowest rank's."""
    return ops_per_step / (ms_per_step * 1e-3) / 1e12 * world_size


def bench_config(w, k, world_size):
    """The `config` object of a bench line (both arms): the workload, how L2 is
    handled between steps and the parallelism."""
    qkv_mb = 3 * 2 * w.B * w.H * w.N * w.d / 1e6
    return {"workload": f"{w.name} B={w.B} H={w.H} N={w.N} d={w.d} k%={w.topk_frac * 100:g} (k={k} of {w.nk})",
            "l2": (f"no flush: Q/K/V {qkv_mb:.0f} MB > 126 MB L2" if qkv_mb > 126 else
                   f"no flush: Q/K/V {qkv_mb:.0f} MB fit in the 126 MB L2 (warm-cache timing)"),
            "parallelism": f"replicas x{world_size}"}


def dist_setup():
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    return ws, rank, local


def cpu_oracle_sample(w, blocks_per_head=16):
    """Time the oracle on a bounded sample of the workload: one head's set-up
    (router, quantisation, linear states) plus `blocks_per_head` query blocks,
    extrapolated to the whole workload. Returns (effective TOPS, description)."""
    import numpy as np
    from oracle import sla2_oracle as O
    from block_sparse_linear_router_b200.inputs import make_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    inp = make_inputs(w, heads=1)
    Q, K, V = (t[0, 0].double().numpy() for t in (inp.q, inp.k, inp.v))
    Wq, Wk, al = inp.proj_q[0].double().numpy(), inp.proj_k[0].double().numpy(), inp.alpha[0].double().numpy()
    t0 = time.perf_counter()
    O.head_forward(Q, K, V, Wq, Wk, al, w.topk_frac, mode="qa", blocks=[])
    t_setup = time.perf_counter() - t0
    nb = blocks_per_head
    t0 = time.perf_counter()
    O.head_forward(Q, K, V, Wq, Wk, al, w.topk_frac, mode="qa", blocks=list(range(nb)))
    t_blocks = max(time.perf_counter() - t0 - t_setup, 1e-9)
    per_block = t_blocks / nb
    nq = w.N // 128
    t_full = w.B * w.H * (t_setup + nq * per_block)
    eff = 4 * w.B * w.H * w.N * w.N * w.d / t_full / 1e12
    sample = (f"oracle mode qa, 1 head: set-up {t_setup:.2f} s + {nb} query blocks {t_blocks:.2f} s, "
              f"extrapolated to {w.B * w.H} heads x {nq} query blocks = {t_full:.0f} s per forward")
    return eff, sample, cores, t_full


def run_reference(args):
    """--impl reference: the CPU oracle, rank 0 only."""
    from block_sparse_linear_router_b200.inputs import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import sla2_oracle as O
    w = WORKLOADS[args.workload]
    if args.frac is not None:
        w = w.with_frac(args.frac, alpha_one=(args.frac == 1.0))
    k = O.topk_count(w.nk, w.topk_frac)
    vals, samples = [], []
    for _ in range(max(args.warmup, 0)):
        cpu_oracle_sample(w, blocks_per_head=8)
    for _ in range(args.steps):
        eff, sample, cores, t_full = cpu_oracle_sample(w, blocks_per_head=8)
        vals.append(eff)
        samples.append(sample)
    v = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 4 * w.B * w.H * w.N * w.N * w.d / v / 1e9,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(w, k, args.gpus),
        "cpu_baseline": {"value": v, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": samples[-1]},
        "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--frac", type=float, default=None, help="override k% (sweep)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from block_sparse_linear_router_b200 import build as B
    from block_sparse_linear_router_b200 import sla2
    from block_sparse_linear_router_b200.inputs import WORKLOADS, make_inputs

    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        B.build()
    if ws > 1:
        dist.barrier()
    sla2.load_library()

    w = WORKLOADS[args.workload]
    if args.frac is not None:
        w = w.with_frac(args.frac, alpha_one=(args.frac == 1.0))
    inp = make_inputs(w)
    t = {n: getattr(inp, n).to(dev) for n in ("q", "k", "v", "proj_q", "proj_k", "alpha")}
    k = sla2.topk_count(w.nk, w.topk_frac)
    wsp = sla2.Workspace.for_shape(w.B, w.H, w.N, w.d, w.topk_frac, 1, dev)
    out = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    import ctypes
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(sla2.STAGE_EVENTS)] for _ in range(K)]
    for row in evs:                      # materialise the lazily created events
        for e in row:
            e.record(stream)
    handles = [(ctypes.c_void_p * sla2.STAGE_EVENTS)(*[e.cuda_event for e in row]) for row in evs]

    def step(h=None):
        sla2.forward(t["q"], t["k"], t["v"], t["proj_q"], t["proj_k"], t["alpha"], w.topk_frac, quantize=1,
                     workspace=wsp, out=out, stream=stream, stage_events=h)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        step(handles[i])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if ws > 1:
        dist.barrier()
    ms_total = e0.elapsed_time(e1)
    clk = clocks.stop()

    stage_ms = [0.0] * 4
    for row in evs:
        for s in range(4):
            stage_ms[s] += row[s].elapsed_time(row[s + 1]) / K
    ms_step = ms_total / K
    if ws > 1:
        ms_step = max_over_ranks(ms_step, dist, dev)

    wm = work_model(w, k)
    eff_tops = job_throughput(wm["effective_ops"], ms_step, ws)

    # ---- end to end through the public API: pinned host inputs -> device -> forward -> host output
    e2e = None
    if not args.no_e2e:
        host = {n: getattr(inp, n).pin_memory() for n in ("q", "k", "v", "proj_q", "proj_k", "alpha")}
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dbuf = {n: torch.empty_like(t[n]) for n in t}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            for n in host:
                dbuf[n].copy_(host[n], non_blocking=True)
            sla2.forward(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["proj_q"], dbuf["proj_k"], dbuf["alpha"],
                         w.topk_frac, quantize=1, workspace=wsp, out=out, stream=stream)
            hout.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        if ws > 1:
            dist.barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        ke = max(3, K // 4)
        f0.record(stream)
        for _ in range(ke):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = f0.elapsed_time(f1) / ke
        if ws > 1:
            ms_e2e = max_over_ranks(ms_e2e, dist, dev)
        e2e = {"value": job_throughput(wm["effective_ops"], ms_e2e, ws), "unit": "TOPS",
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank != 0:
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    p8 = peaks["bf16_tflops"] * NOMINAL_8BIT_OVER_BF16
    names = ["router", "linear_state", "sparse", "epilogue"]
    kern = {}
    p16 = peaks["bf16_tflops"]   # fp16 and bf16 run at the same dense rate
    for n, msv in zip(names, stage_ms):
        if n == "sparse":
            ach = wm["sparse_ops"] / (msv * 1e-3) / 1e12
            kern[n] = {"ms": msv, "bound": "tensor", "achieved": ach, "peak": p8, "unit": "TOPS", "frac": ach / p8}
        elif n == "epilogue" and wm["epilogue_flops"] > 0:
            # tensor-bound when its MMA time exceeds its HBM time (206 GFLOP vs 604 MB here)
            ach = wm["epilogue_flops"] / (msv * 1e-3) / 1e12
            hb = wm["epilogue_bytes"] / (msv * 1e-3) / 1e9
            kern[n] = {"ms": msv, "bound": "tensor", "achieved": ach, "peak": p16, "unit": "TFLOP/s",
                       "frac": ach / p16, "hbm_achieved_gbs": hb, "hbm_frac": hb / hbm,
                       "algorithmic_bytes": wm["epilogue_bytes"], "flops": wm["epilogue_flops"]}
        else:
            b = wm[f"{n.split('_')[0]}_bytes"] if n != "linear_state" else wm["linear_bytes"]
            ach = b / (msv * 1e-3) / 1e9
            kern[n] = {"ms": msv, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                       "algorithmic_bytes": b}
    for n in names:
        tb, tsrc = measured_traffic(n)
        kern[n]["traffic"] = tb
        if tb is not None:
            kern[n]["traffic_source"] = tsrc
    dom = max(names, key=lambda n: kern[n]["ms"])
    dk = kern[dom]
    psrc = {"sparse": "8-bit = bf16 burst x 2 nominal ratio", "epilogue": "fp16 = bf16 burst (same dense rate)"}
    roofline = {"bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"], "unit": dk["unit"],
                "frac": dk["frac"], "traffic": dk["traffic"], "kernel": dom,
                "peak_source": f"{peak_src} ({psrc.get(dom, 'HBM copy') if dk['bound'] == 'tensor' else 'HBM copy'})"}

    cpu = None
    if not args.no_cpu_baseline:
        eff, sample, cores, _ = cpu_oracle_sample(w)
        cpu = {"value": eff, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample}

    line = {
        "metric": METRIC, "value": eff_tops, "unit": "TOPS", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8+e4m3",
        "data": "synthetic",
        "config": bench_config(w, k, ws),
        "roofline": roofline, "kernels": kern,
        "stages": "router = pass over Q/K/V + column means; linear_state = linear state + reduce on a second "
                  "stream, with the router's projections / logits / top-k concurrent on the caller's stream; "
                  "sparse = sparse branch (Z_i concurrent); epilogue = linear apply + mix",
        "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_forward(w, k) * K, "clocks": clk,
        "sparse_issued_tops": kern["sparse"]["achieved"],
    }
    print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
