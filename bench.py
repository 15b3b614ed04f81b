#!/usr/bin/env python
"""Benchmark of the quantized MoE expert step on B200.

Default workload (the configuration the headline metric is quoted on): one
decode MoE layer shaped like the Flash-MoE pages' model, hidden 4096, 512
experts, top-4 renormalised, expert intermediate 1024, 4-bit affine group-64
experts (bf16 scale/bias), SwiGLU, batch 1 token fp32, all experts resident
in HBM.  One step = one token through the whole layer (RMSNorm, router,
top-K, 4 expert FFNs, combine) = one launch of the fused kernel.  Tokens are
distinct seeded N(0,1) vectors, so routing scatters over the 3.6 GB expert
pool, far larger than L2.

Other workloads (--workload): c0 tiny layer, c4 batched decode (256 tokens
per step, grouped experts).  Prints one JSON line; ``--impl reference`` times
the fp64 CPU oracle on the host cores instead.
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

EPS32 = float(np.float32(1e-6))

WORKLOADS = {
    "c1": dict(H=4096, E=512, K=4, I=1024, bits=4, T=1,
               name="one decode MoE layer: hidden 4096, 512 experts, top-4 renormalised, intermediate 1024, "
                    "4-bit affine g64 bf16 scale/bias, SwiGLU, batch 1 token fp32, all experts in HBM",
               metric="MoE-layer decode tokens/s at 1 B200"),
    "c0": dict(H=256, E=16, K=2, I=64, bits=4, T=1,
               name="tiny MoE FFN: hidden 256, 16 experts, top-2, intermediate 64, 4-bit g64, 1 token",
               metric="MoE-layer decode tokens/s at 1 B200 (tiny layer)"),
    "c4": dict(H=4096, E=512, K=4, I=1024, bits=4, T=256,
               name="batched decode of the one-layer workload: 256 bf16 tokens per step, own top-4 of 512 each, "
                    "grouped per expert, 4-bit g64 experts in HBM, uniform routing",
               metric="MoE-layer batched decode tokens/s at 1 B200"),
}

UNIT = "tokens/s"


def expert_bytes(H, I, bits):
    n = 3 * H * I
    return n * bits // 8 + 2 * 2 * n // 64


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
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
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
    """Time the fp64 oracle on whole tokens of the workload's layer: routing
    in full, expert matvecs on a leading fraction of the rows (extrapolated).
    Expert weights are regenerated before the timed calls.  Returns (seconds
    per token, threads, seconds measured)."""
    import oracle
    import synth
    H, E, K, I, bits = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"]
    bf16 = wl["T"] > 1
    nthreads = nthreads or os.cpu_count() or 1
    W = synth.host_router(seed, 0, E, H)

    def tok(t):
        x = synth.host_tokens(seed, t, 1, H, bf16=bf16)[0]
        if bf16:
            return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return x.astype(np.float64)

    xs = [tok(t) for t in tokens]
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
    per1, nth, _ = oracle_token_time(wl, seed, [1_000_000])
    n = max(1, min(64, int(budget_s / max(per1, 1e-9))))
    per, nth, spent = oracle_token_time(wl, seed, list(range(1_000_001, 1_000_001 + n)))
    return {"value": 1.0 / per, "unit": UNIT, "cores": nth, "kind": "oracle",
            "sample": f"{n} whole tokens of the workload (fp64 oracle, OpenMP over rows, {nth} threads), "
                      f"{spent:.1f} s of CPU time"}


class OracleSample:
    """The oracle on a fixed pool of distinct tokens of the workload: routing
    in full every time, expert matvecs on a leading fraction of the rows
    (their time extrapolated to the full rows).  Experts are generated once,
    outside the timed calls, and kept cut to the sampled rows."""

    def __init__(self, wl, seed, frac, n_pool=32, nthreads=None):
        import oracle
        import synth
        self.oracle = oracle
        H, E, K, I, bits = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"]
        self.K, self.bits, self.H, self.I = K, bits, H, I
        self.nthreads = nthreads or os.cpu_count() or 1
        self.frac = frac
        self.nr_i = max(1, int(round(I * frac)))
        self.nr_h = max(1, int(round(H * frac)))
        self.W = synth.host_router(seed, 0, E, H)
        bf16 = wl["T"] > 1
        self.xs = []
        self.experts = {}
        for t in range(n_pool):
            x = synth.host_tokens(seed, 4_000_000 + t, 1, H, bf16=bf16)[0]
            x = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if bf16 else x.astype(np.float64)
            self.xs.append(x)
            idx, _ = oracle.topk(oracle.router(self.W, oracle.rmsnorm(x, None, EPS32), None, self.nthreads), K)
            for e in idx:
                e = int(e)
                if e not in self.experts:
                    ex = synth.host_expert(seed, 0, e, H, I, bits)
                    cut = {}
                    for m, nr in (("gate", self.nr_i), ("up", self.nr_i), ("down", self.nr_h)):
                        for f in ("wq", "s", "b"):
                            cut[f"{m}_{f}"] = np.ascontiguousarray(ex[f"{m}_{f}"][:nr])
                    self.experts[e] = cut

    def token_seconds(self, t):
        """Oracle time of pool token t, extrapolated to the full rows."""
        o, nth, bits = self.oracle, self.nthreads, self.bits
        x = self.xs[t % len(self.xs)]
        t0 = time.perf_counter()
        xn = o.rmsnorm(x, None, EPS32)
        idx, w = o.topk(o.router(self.W, xn, None, nth), self.K)
        t1 = time.perf_counter()
        yfull = np.zeros((self.K, self.H))
        for k, e in enumerate(idx):
            ex = self.experts[int(e)]
            g = o.qmatvec(ex["gate_wq"], ex["gate_s"], ex["gate_b"], bits, xn, nth)
            u = o.qmatvec(ex["up_wq"], ex["up_s"], ex["up_b"], bits, xn, nth)
            h = np.zeros(self.I)
            h[: self.nr_i] = o.swiglu(g, u)
            yfull[k, : self.nr_h] = o.qmatvec(ex["down_wq"], ex["down_s"], ex["down_b"], bits, h, nth)
        o.combine(yfull, w, x)
        t2 = time.perf_counter()
        return (t1 - t0) + (t2 - t1) / self.frac


def run_reference(args, wl, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores.
    Each step is one token (T tokens for a batched workload, of which at
    most 4 are timed and the rest extrapolated), on a bounded sample sized so
    that all warm-up and timed steps take about 150 s."""
    if rank != 0:
        return
    K, W, T = args.steps, args.warmup, wl["T"]
    probe = OracleSample(wl, args.seed, 1.0, n_pool=1)
    per_full = min(probe.token_seconds(0) for _ in range(2))
    t_timed = min(T, 4)
    frac = min(1.0, max(1.0 / 512, (150.0 / (K + W)) / max(per_full * t_timed, 1e-9)))
    smp = OracleSample(wl, args.seed, frac)
    i = 0
    for _ in range(W):
        for _ in range(t_timed):
            smp.token_seconds(i)
            i += 1
    t0 = time.perf_counter()
    total = 0.0
    for _ in range(K):
        st = 0.0
        for _ in range(t_timed):
            st += smp.token_seconds(i)
            i += 1
        total += st * (T / t_timed)
    wall = time.perf_counter() - t0
    value = K * T / total
    line = {"metric": wl["metric"], "value": value, "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": 1000.0 * total / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl["name"], "tokens_per_step": T,
                       "tokens": "a pool of 32 distinct seeded N(0,1) tokens, cycled"},
            "cpu_baseline": {"kind": "oracle", "cores": smp.nthreads, "value": value, "unit": UNIT,
                             "sample": f"each step: {t_timed} of its {T} token(s) timed, routing in full, expert "
                                       f"rows sampled at fraction {frac:.4f} and extrapolated; "
                                       f"{wall:.1f} s wall for the timed steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

class LayerSetup:
    """One resident layer (pool, router, workspace) and a token stream."""

    def __init__(self, q, wl, seed, dev, n_tok, tok0):
        import torch
        from _util import dev_router, dev_tokens, fill_pool
        H, E, K, I, bits, T = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"], wl["T"]
        self.wl = wl
        self.cfg = q.Cfg(H, E, K, I, 64, EPS32)
        self.pool = q.ExpertPool(self.cfg, E, bits, device=dev)
        fill_pool(self.pool, seed, 0)
        self.W = dev_router(seed, 0, E, H, device=dev)
        self.layer = q.Layer(self.W.data_ptr(), None, None, self.pool.table.data_ptr())
        self.ws = q.workspace(self.cfg, T, device=dev)
        self.x = dev_tokens(seed, tok0, n_tok, H, bf16=T > 1, device=dev)
        self.out = torch.empty((n_tok, H), dtype=torch.float32, device=dev)
        self.idx = torch.empty((n_tok, K), dtype=torch.int32, device=dev)
        self.w = torch.empty((n_tok, K), dtype=torch.float32, device=dev)
        self.n_tok = n_tok
        self.T = T


def run_ours(args, wl, rank, world, local_rank):
    import torch
    import quantized_expert_matvec_b200 as q
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H, E, K, I, bits, T = wl["H"], wl["E"], wl["K"], wl["I"], wl["bits"], wl["T"]
    seed = args.seed
    chunk = 1024 if T == 1 else 8          # steps per captured graph
    n_chunks = 8 if T == 1 else 4
    n_tok = chunk * n_chunks * T
    ls = LayerSetup(q, wl, seed, dev, n_tok, 10_000_000 * (rank + 1))
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def step(i, stream):
        t0 = (i * T) % n_tok
        q.moe_layer_step(ls.cfg, ls.layer, ls.x[t0:t0 + T], ls.out[t0:t0 + T], False, ls.idx[t0:t0 + T],
                         ls.w[t0:t0 + T], ls.ws, stream=stream)

    def capture(first, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(count):
                step(first + i, s)
        return g

    with torch.cuda.stream(s):
        step(0, s)
        s.synchronize()
        graphs = [capture(c * chunk, chunk) for c in range(n_chunks)]
        rem = args.steps % chunk
        rem_graph = capture(0, rem) if rem else None
        warm_graph = capture(0, min(args.warmup, chunk * n_chunks))
    torch.cuda.synchronize()
    if q.qe_workspace_status(ls.ws, s) != q.QE_OK:
        raise RuntimeError("device status after capture: " + q.qe_last_error())

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    with torch.cuda.stream(s):
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
    if q.qe_workspace_status(ls.ws, s) != q.QE_OK:
        raise RuntimeError("device status after timing: " + q.qe_last_error())
    ms_max = ms
    if world > 1:
        import torch.distributed as dist
        tt = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_max = float(tt.item())
    value = world * args.steps * T / (ms_max / 1000.0)

    # distinct experts touched per step (from the routing of the timed steps)
    idx_h = ls.idx.cpu().numpy().reshape(-1, T * K)
    written = min(len(idx_h), max(args.steps, min(args.warmup, chunk * n_chunks)))  # rows the steps wrote
    distinct = float(np.mean([len(np.unique(r)) for r in idx_h[:written]]))

    # ---------------------------------------------------------------- e2e
    n_e2e = min(args.steps, 2048 if T == 1 else 64)
    x_host = ls.x[: max(T, 1) * min(n_e2e, ls.n_tok // T)].cpu().pin_memory()
    out_host = torch.empty((T, H), dtype=torch.float32).pin_memory()
    xin = torch.empty((T, H), dtype=ls.x.dtype, device=dev)
    res = torch.empty((T, H), dtype=torch.float32, device=dev)
    nb = x_host.shape[0] // T

    def e2e_step(i):
        b = (i % nb) * T
        xin.copy_(x_host[b:b + T], non_blocking=True)
        q.moe_layer_step(ls.cfg, ls.layer, xin, res, False, None, None, ls.ws, stream=s)
        out_host.copy_(res, non_blocking=True)
        s.synchronize()

    with torch.cuda.stream(s):
        for i in range(4):
            e2e_step(i)
    barrier()
    t0 = time.perf_counter()
    with torch.cuda.stream(s):
        for i in range(n_e2e):
            e2e_step(i)
    e2e_s = time.perf_counter() - t0
    if world > 1:
        import torch.distributed as dist
        tt = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_s = float(tt.item())
    e2e_value = world * n_e2e * T / e2e_s

    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    per_step_s = (ms / 1000.0) / args.steps
    exp_b = distinct * expert_bytes(H, I, bits)
    alg = exp_b + E * H * 4 + T * H * (2 if T > 1 else 4) + T * H * 4
    achieved = alg / per_step_s / 1e9
    peak = float(peaks["hbm_gbs"])
    cpu = None if args.no_cpu_baseline else cpu_baseline(wl, seed)
    kern = "qe_fused_layer_kernel" if T == 1 else "grouped_expert_kernel (+ route, group, combine)"
    line = {
        "metric": wl["metric"], "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "tokens_per_step": T, "tokens_distinct": ls.n_tok,
                   "l2": "inputs larger than L2: 3.6 GB expert pool, routing scatters over all 512 experts",
                   "launch": f"CUDA graphs of {chunk} layer steps",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": load_traffic(args.workload), "peak_source": peak_kind,
                     "kernel": kern, "algorithmic_bytes_per_launch": alg,
                     "duration": "whole step (launch gaps included)"},
        "expert_gbs": exp_b / per_step_s / 1e9,
        "expert_frac": exp_b / per_step_s / 1e9 / peak,
        "distinct_experts_per_step": distinct,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * H * ls.x.element_size(),
                "d2h_bytes_per_step": T * H * 4, "steps": n_e2e,
                "how": "per step: pinned H2D of x, moe_layer_step, D2H of out, stream sync"},
        "gpu_launches": args.steps * (1 if T == 1 else 6),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c1", choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.steps is None:
        args.steps = 32768 if wl["T"] == 1 else 64
    if args.warmup is None:
        args.warmup = 256 if wl["T"] == 1 else 8
    args.warmup = max(args.warmup, 3)
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
