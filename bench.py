#!/usr/bin/env python
"""Benchmark of the quantized MoE expert step on B200.

Default workload (one decode MoE layer shaped like the Flash-MoE pages'
model): hidden 4096, 512 experts, top-4 renormalised, expert intermediate
1024, 4-bit affine group-64 experts (bf16 scale/bias), SwiGLU, batch 1 token
fp32, all experts resident in HBM.  One step = one token through the whole
layer (RMSNorm, router, top-K, 4 expert FFNs, combine) = one launch of the
fused kernel.  Tokens are distinct (a stream of seeded N(0,1) vectors), so the
routing scatters over the 3.6 GB expert pool, far larger than L2.

Prints one JSON line (see the design doc for every key).  ``--impl reference``
times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402

WORKLOADS = {
    "c1": dict(H=4096, E=512, K=4, I=1024, bits=4,
               name="one decode MoE layer: hidden 4096, 512 experts, top-4 renormalised, intermediate 1024, "
                    "4-bit affine g64 bf16 scale/bias, SwiGLU, batch 1 token fp32, all experts in HBM"),
    "c0": dict(H=256, E=16, K=2, I=64, bits=4,
               name="tiny MoE FFN: hidden 256, 16 experts, top-2, intermediate 64, 4-bit g64, 1 token"),
}

METRIC = "MoE-layer decode tokens/s at 1 B200"
UNIT = "tokens/s"
EPS32 = float(np.float32(1e-6))
KERNEL_NAME = "qe_fused_layer_kernel"


def expert_bytes(H, I, bits):
    n = 3 * H * I
    return n * bits // 8 + 2 * 2 * n // 64


def algorithmic_bytes(wl):
    """Bytes one fused launch must move: K experts' packed weights and
    scales/biases, the fp32 router, x in and out."""
    H, E, K, I, bits = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"]
    experts = K * expert_bytes(H, I, bits)
    router = E * H * 4
    act = 2 * H * 4
    return experts, router, act


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_expert_matvec_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic(workload):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", f"fused_layer_{workload}_traffic.json")
    try:
        d = json.load(open(path))
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("traffic_bytes_per_launch")


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": sorted(reasons),
                "samples": len(rows)}


# --------------------------------------------------------------------------
# oracle timing (the CPU baseline and the reference arm)
# --------------------------------------------------------------------------

def oracle_token_time(wl, seed, tokens, row_fraction=1.0, nthreads=None):
    """Time the fp64 oracle on `tokens` tokens of the workload: routing in
    full, expert matvecs on a leading fraction of the rows.  Expert weights
    are regenerated before the timed calls.  Returns (seconds per token
    extrapolated to all rows, threads, seconds measured)."""
    import oracle
    import synth
    H, E, K, I, bits = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"]
    nthreads = nthreads or os.cpu_count() or 1
    W = synth.host_router(seed, 0, E, H)
    xs = [synth.host_tokens(seed, t, 1, H)[0].astype(np.float64) for t in tokens]
    # untimed: find the experts, regenerate them
    cache = {}
    for x in xs:
        idx, _ = oracle.topk(oracle.router(W, oracle.rmsnorm(x, None, EPS32), None, nthreads), K)
        for e in idx:
            if int(e) not in cache:
                cache[int(e)] = synth.host_expert(seed, 0, int(e), H, I, bits)
    nr_i = max(1, int(round(I * row_fraction)))
    nr_h = max(1, int(round(H * row_fraction)))
    t_route = 0.0
    t_exp = 0.0
    for x in xs:
        t0 = time.perf_counter()
        xn = oracle.rmsnorm(x, None, EPS32)
        lg = oracle.router(W, xn, None, nthreads)
        idx, w = oracle.topk(lg, K)
        t1 = time.perf_counter()
        ys = []
        for e in idx:
            ex = cache[int(e)]
            g = oracle.qmatvec(ex["gate_wq"][:nr_i], ex["gate_s"][:nr_i], ex["gate_b"][:nr_i], bits, xn, nthreads)
            u = oracle.qmatvec(ex["up_wq"][:nr_i], ex["up_s"][:nr_i], ex["up_b"][:nr_i], bits, xn, nthreads)
            h = np.zeros(I)
            h[:nr_i] = oracle.swiglu(g, u)
            ys.append(oracle.qmatvec(ex["down_wq"][:nr_h], ex["down_s"][:nr_h], ex["down_b"][:nr_h], bits, h,
                                     nthreads))
        yfull = np.zeros((K, H))
        for k in range(K):
            yfull[k, :nr_h] = ys[k]
        oracle.combine(yfull, w, x)
        t2 = time.perf_counter()
        t_route += t1 - t0
        t_exp += t2 - t1
    n = len(xs)
    per_token = t_route / n + (t_exp / n) / (nr_h / H if row_fraction < 1.0 else 1.0)
    return per_token, nthreads, t_route + t_exp


def cpu_baseline(wl, seed, budget_s=15.0):
    """The oracle on a bounded sample of the workload (whole tokens)."""
    per1, nth, spent = oracle_token_time(wl, seed, [1_000_000])
    n = max(1, min(64, int(budget_s / max(per1, 1e-9))))
    per, nth, spent2 = oracle_token_time(wl, seed, list(range(1_000_001, 1_000_001 + n)))
    return {"value": 1.0 / per, "unit": UNIT, "cores": nth, "kind": "oracle",
            "sample": f"{n} whole tokens of the workload (fp64 oracle, OpenMP over rows, {nth} threads), "
                      f"{spent2:.1f} s of CPU time"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    per_full, nth, _ = oracle_token_time(wl, args.seed, [2_000_000])
    budget = 150.0  # seconds for all K + W steps
    frac = min(1.0, max(1.0 / 256, (budget / (K + W)) / max(per_full, 1e-9)))
    for t in range(W):
        oracle_token_time(wl, args.seed, [3_000_000 + t], frac, nth)
    t0 = time.perf_counter()
    per = []
    for t in range(K):
        p, _, _ = oracle_token_time(wl, args.seed, [4_000_000 + t], frac, nth)
        per.append(p)
    wall = time.perf_counter() - t0
    value = K / sum(per)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": 1000.0 * sum(per) / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl["name"], "tokens": "distinct seeded N(0,1) tokens"},
            "cpu_baseline": {"kind": "oracle", "cores": nth, "value": value, "unit": UNIT,
                             "sample": f"each step: one token, routing in full, expert rows sampled at fraction "
                                       f"{frac:.4f} and extrapolated; {wall:.1f} s wall"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def run_ours(args, wl, rank, world, local_rank):
    import torch
    import quantized_expert_matvec_b200 as q
    from _util import dev_router, dev_tokens, fill_pool
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H, E, K, I, bits = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"]
    cfg = q.Cfg(H, E, K, I, 64, EPS32)
    seed = args.seed
    pool = q.ExpertPool(cfg, E, bits, device=dev)
    fill_pool(pool, seed, 0)
    Wr = dev_router(seed, 0, E, H, device=dev)
    layer = q.Layer(Wr.data_ptr(), None, None, pool.table.data_ptr())
    ws = q.workspace(cfg, 1, device=dev)
    chunk = 1024
    n_chunks = 8
    n_tok = chunk * n_chunks
    tok0 = 10_000_000 * (rank + 1)
    x = dev_tokens(seed, tok0, n_tok, H, device=dev)
    out = torch.empty((n_tok, H), dtype=torch.float32, device=dev)
    idx = torch.empty((n_tok, K), dtype=torch.int32, device=dev)
    wts = torch.empty((n_tok, K), dtype=torch.float32, device=dev)
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def step(t, stream):
        q.moe_layer_step(cfg, layer, x[t:t + 1], out[t:t + 1], False, idx[t:t + 1], wts[t:t + 1], ws,
                         stream=stream)

    def capture(first, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(count):
                step((first + i) % n_tok, s)
        return g

    with torch.cuda.stream(s):
        step(0, s)
        s.synchronize()
        graphs = [capture(c * chunk, chunk) for c in range(n_chunks)]
        rem = args.steps % chunk
        rem_graph = capture(0, rem) if rem else None
        warm_graph = capture(0, args.warmup) if args.warmup else None
    torch.cuda.synchronize()
    if q.qe_workspace_status(ws, s) != q.QE_OK:
        raise RuntimeError("device status after capture: " + q.qe_last_error())

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # warm-up
    with torch.cuda.stream(s):
        if warm_graph is not None:
            warm_graph.replay()
    s.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    full = args.steps // chunk
    with torch.cuda.stream(s):
        ev0.record(s)
        for i in range(full):
            graphs[i % n_chunks].replay()
        if rem_graph is not None:
            rem_graph.replay()
        ev1.record(s)
    s.synchronize()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1)
    status = q.qe_workspace_status(ws, s)
    if status != q.QE_OK:
        raise RuntimeError("device status after timing: " + q.qe_last_error())
    ms_max = ms
    if world > 1:
        import torch.distributed as dist
        tt = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_max = float(tt.item())
    value = world * args.steps / (ms_max / 1000.0)

    # ---------------------------------------------------------------- e2e
    n_e2e = min(args.steps, 2048)
    x_host = x[:n_e2e].cpu().pin_memory()
    out_host = torch.empty((n_e2e, H), dtype=torch.float32).pin_memory()
    xin = torch.empty((1, H), dtype=torch.float32, device=dev)
    res = torch.empty((1, H), dtype=torch.float32, device=dev)
    with torch.cuda.stream(s):
        for t in range(8):
            xin.copy_(x_host[t:t + 1], non_blocking=True)
            q.moe_layer_step(cfg, layer, xin, res, False, None, None, ws, stream=s)
            out_host[t:t + 1].copy_(res, non_blocking=True)
            s.synchronize()
    barrier()
    t0 = time.perf_counter()
    with torch.cuda.stream(s):
        for t in range(n_e2e):
            xin.copy_(x_host[t:t + 1], non_blocking=True)
            q.moe_layer_step(cfg, layer, xin, res, False, None, None, ws, stream=s)
            out_host[t:t + 1].copy_(res, non_blocking=True)
            s.synchronize()
    e2e_s = time.perf_counter() - t0
    if world > 1:
        import torch.distributed as dist
        tt = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_s = float(tt.item())
    e2e_value = world * n_e2e / e2e_s

    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    exp_b, rout_b, act_b = algorithmic_bytes(wl)
    per_launch_s = (ms / 1000.0) / args.steps
    alg = exp_b + rout_b + act_b
    achieved = alg / per_launch_s / 1e9
    peak = float(peaks["hbm_gbs"])
    traffic = load_traffic(args.workload)
    cpu = None if args.no_cpu_baseline else cpu_baseline(wl, seed)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "batch": 1, "tokens_distinct": n_tok,
                   "l2": "inputs larger than L2: 3.6 GB expert pool, routing scatters over all 512 experts",
                   "launch": "CUDA graphs of 1024 single-token layer steps, one fused persistent kernel each",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                     "kernel": KERNEL_NAME, "algorithmic_bytes_per_launch": alg},
        "expert_gbs": exp_b / per_launch_s / 1e9,
        "expert_frac": exp_b / per_launch_s / 1e9 / peak,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
                "steps": n_e2e, "how": "per token: pinned H2D of x, moe_layer_step, D2H of out, stream sync"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=65536)
    ap.add_argument("--warmup", type=int, default=1024)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c1", choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
