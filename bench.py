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

Other workloads (--workload): c0 tiny layer, c2 40-layer stack, c3 tiered
layers, c4 batched decode (256 tokens per step, grouped experts), gdn the
GatedDeltaNet decode step of the same model (45 layers of 64 heads x 128x128
recurrent state).  Prints one JSON line; ``--impl reference`` times
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
    "c2": dict(H=4096, E=512, K=4, I=1024, bits=4, T=1, layers=40, zipf=True,
               name="40-layer stack of the one-layer workload (no attention), 145 GB of 4-bit experts in HBM, "
                    "sequential decode tokens with residual add between layers, Zipf(1.1) popularity logit "
                    "offset per layer (alpha 0.40: about 70% of selections in the hottest 25%)",
               metric="40-layer MoE stack decode tokens/s at 1 B200"),
    "c3": dict(H=4096, E=512, K=4, I=1024, bits=4, T=1, layers=60, zipf=True, hot=128, cache_gb=24.0,
               name="60 tiered layers of the one-layer shape: per layer the 128 most popular experts 4-bit in "
                    "HBM, the other 384 2-bit in pinned host memory behind a 24 GB HBM LRU expert cache "
                    "(misses copied by a kernel from mapped host memory, cache resolved on the device), Zipf routing, "
                    "sequential decode tokens with residual",
               metric="60-layer tiered MoE decode tokens/s at 1 B200"),
    "c4": dict(H=4096, E=512, K=4, I=1024, bits=4, T=256,
               name="batched decode of the one-layer workload: 256 bf16 tokens per step, own top-4 of 512 each, "
                    "grouped per expert, 4-bit g64 experts in HBM, uniform routing",
               metric="MoE-layer batched decode tokens/s at 1 B200"),
    "gdn": dict(heads=64, dk=128, dv=128, layers=45, T=1,
                name="GatedDeltaNet decode: one token through the recurrent state of 45 linear-attention layers, "
                     "64 heads x 128x128 fp32 state per layer (180 MiB of state in HBM, larger than L2), gated "
                     "delta rule (scal, gemv, ger, gemv per head), batch 1 sequence",
                metric="GatedDeltaNet decode tokens/s at 1 B200 (45 layers)"),
    "gdn8": dict(heads=64, dk=128, dv=128, layers=45, T=8, seqs=8,
                 name="GatedDeltaNet batched decode: one token of each of 8 sequences through the recurrent state "
                      "of 45 linear-attention layers, 8 x 64 heads x 128x128 fp32 state per layer (1.4 GiB of "
                      "state in HBM), gated delta rule, one launch per layer for all 8 sequences",
                 metric="GatedDeltaNet batched decode tokens/s at 1 B200 (45 layers, 8 sequences)"),
}

UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal


def expert_bytes(H, I, bits):
    n = 3 * H * I
    return n * bits // 8 + 2 * 2 * n // 64


KERNEL_SOURCES = {  # the sources the dominant kernel of each workload is compiled from
    "c1": ("qe_fused.cu", "qe_device.cuh", "qe_fused_plan.h", "qe_internal.h"),
    "c0": ("qe_fused.cu", "qe_device.cuh", "qe_fused_plan.h", "qe_internal.h"),
    "c2": ("qe_fused.cu", "qe_device.cuh", "qe_fused_plan.h", "qe_internal.h"),
    "c4": ("qe_grouped.cu", "qe_device.cuh", "qe_internal.h"),
    "gdn": ("qe_gdn.cu", "qe_device.cuh", "qe_internal.h"),
    "gdn8": ("qe_gdn.cu", "qe_device.cuh", "qe_internal.h"),
}


def kernel_source_hash(workload="c1"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_expert_matvec_b200", "csrc")
    for f in KERNEL_SOURCES.get(workload, KERNEL_SOURCES["c1"]):
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
    if d.get("kernel_source_hash") != kernel_source_hash(workload):
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

def wl_layers(wl):
    return wl.get("layers", 1)


def wl_bits_of(wl, seed, layer):
    """Bits of each expert of a layer: the tiered workload keeps its hot set
    (most popular ranks) at 4 bits and the rest at 2."""
    import synth
    if wl.get("hot"):
        hot = synth.hot_set(seed, layer, wl["E"], wl["hot"])
        return lambda e: 4 if hot[e] else 2
    return lambda e: wl["bits"]


def wl_offset(wl, seed, layer):
    import synth
    return synth.zipf_logit_offset(seed, layer, wl["E"]) if wl.get("zipf") else None


class OracleSample:
    """The oracle on a pool of (layer, token) layer steps of the workload:
    routing in full every time, expert matvecs on a leading fraction of the
    rows (their time extrapolated to the full rows).  Experts are generated
    once, outside the timed calls, and kept cut to the sampled rows."""

    def __init__(self, wl, seed, frac, n_pool=32, nthreads=None, max_layers=8):
        import oracle
        import synth
        self.oracle = oracle
        H, E, K, I = wl["H"], wl["E"], wl["K"], wl["I"]
        self.K, self.H, self.I = K, H, I
        self.nthreads = nthreads or os.cpu_count() or 1
        self.frac = frac
        self.nr_i = max(1, int(round(I * frac)))
        self.nr_h = max(1, int(round(H * frac)))
        self.residual = wl_layers(wl) > 1
        nl = min(wl_layers(wl), max_layers)
        self.W = [synth.host_router(seed, l, E, H) for l in range(nl)]
        self.off = [wl_offset(wl, seed, l) for l in range(nl)]
        self.bits = [wl_bits_of(wl, seed, l) for l in range(nl)]
        bf16 = wl["T"] > 1
        self.pool = []
        self.experts = {}
        for j in range(n_pool):
            l = j % nl
            x = synth.host_tokens(seed, 4_000_000 + j, 1, H, bf16=bf16)[0]
            x = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if bf16 else x.astype(np.float64)
            self.pool.append((l, x))
            idx, _ = oracle.topk(oracle.router(self.W[l], oracle.rmsnorm(x, None, EPS32), self.off[l],
                                               self.nthreads), K)
            for e in idx:
                e = int(e)
                if (l, e) not in self.experts:
                    b = self.bits[l](e)
                    ex = synth.host_expert(seed, l, e, H, I, b)
                    cut = {"bits": b}
                    for m, nr in (("gate", self.nr_i), ("up", self.nr_i), ("down", self.nr_h)):
                        for f in ("wq", "s", "b"):
                            cut[f"{m}_{f}"] = np.ascontiguousarray(ex[f"{m}_{f}"][:nr])
                    self.experts[(l, e)] = cut

    def step_seconds(self, j):
        """Oracle time of pool layer step j, extrapolated to the full rows."""
        o, nth = self.oracle, self.nthreads
        l, x = self.pool[j % len(self.pool)]
        t0 = time.perf_counter()
        xn = o.rmsnorm(x, None, EPS32)
        idx, w = o.topk(o.router(self.W[l], xn, self.off[l], nth), self.K)
        t1 = time.perf_counter()
        yfull = np.zeros((self.K, self.H))
        for k, e in enumerate(idx):
            ex = self.experts[(l, int(e))]
            b = ex["bits"]
            g = o.qmatvec(ex["gate_wq"], ex["gate_s"], ex["gate_b"], b, xn, nth)
            u = o.qmatvec(ex["up_wq"], ex["up_s"], ex["up_b"], b, xn, nth)
            h = np.zeros(self.I)
            h[: self.nr_i] = o.swiglu(g, u)
            yfull[k, : self.nr_h] = o.qmatvec(ex["down_wq"], ex["down_s"], ex["down_b"], b, h, nth)
        o.combine(yfull, w, x if self.residual else None)
        t2 = time.perf_counter()
        return (t1 - t0) + (t2 - t1) / self.frac


def cpu_baseline(wl, seed, budget_s=15.0):
    """The oracle on a bounded sample of the workload: whole layer steps
    (routing and all expert rows), scaled to tokens."""
    probe = OracleSample(wl, seed, 1.0, n_pool=1)
    per1 = probe.step_seconds(0)
    n = max(2, min(2000, int(budget_s / max(per1, 1e-9))))
    pool = min(n, 32)  # 32 distinct tokens, cycled: their experts far exceed any CPU cache
    smp = OracleSample(wl, seed, 1.0, n_pool=pool)
    t0 = time.perf_counter()
    tot = sum(smp.step_seconds(j) for j in range(n))
    spent = time.perf_counter() - t0
    per_token = tot / n * wl_layers(wl)
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": smp.nthreads, "kind": "oracle",
            "sample": f"{n} whole layer steps over {pool} distinct tokens (routing and all expert rows, fp64 "
                      f"oracle, OpenMP over rows, {smp.nthreads} threads) of {min(wl_layers(wl), 8)} layer(s), "
                      f"scaled to {wl_layers(wl)} layer(s) per token; {spent:.1f} s of CPU time"}


def run_reference(args, wl, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores.
    A step is the workload's step (one token through every layer, or T
    tokens through one layer); at most 4 of its layer steps are timed and the
    rest extrapolated, on a bounded sample sized so that all warm-up and
    timed steps take about 150 s."""
    if rank != 0:
        return
    if "heads" in wl:
        run_reference_gdn(args, wl)
        return
    K, W, T = args.steps, args.warmup, wl["T"]
    per_step_units = T * wl_layers(wl)   # layer steps in one step
    probe = OracleSample(wl, args.seed, 1.0, n_pool=1)
    per_full = min(probe.step_seconds(0) for _ in range(2))
    t_timed = min(per_step_units, 4)
    frac = min(1.0, max(1.0 / 512, (150.0 / (K + W)) / max(per_full * t_timed, 1e-9)))
    smp = OracleSample(wl, args.seed, frac)
    i = 0
    for _ in range(W):
        for _ in range(t_timed):
            smp.step_seconds(i)
            i += 1
    t0 = time.perf_counter()
    total = 0.0
    for _ in range(K):
        st = 0.0
        for _ in range(t_timed):
            st += smp.step_seconds(i)
            i += 1
        total += st * (per_step_units / t_timed)
    wall = time.perf_counter() - t0
    value = K * T / total
    line = {"metric": wl["metric"], "value": value, "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": 1000.0 * total / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl["name"], "tokens_per_step": T, "layers": wl_layers(wl),
                       "tokens": "a pool of 32 distinct seeded N(0,1) tokens, cycled"},
            "cpu_baseline": {"kind": "oracle", "cores": smp.nthreads, "value": value, "unit": UNIT,
                             "sample": f"each step: {t_timed} of its {per_step_units} layer step(s) timed, "
                                       f"routing in full, expert rows sampled at fraction {frac:.4f} and "
                                       f"extrapolated; {wall:.1f} s wall for the timed steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class GdnOracleSample:
    """The oracle's GatedDeltaNet step on a few layers of the workload: fp64
    state per layer, a pool of seeded tokens, one whole layer step per call."""

    def __init__(self, wl, seed, n_layers=2, n_tok=4):
        import oracle
        import synth
        self.oracle = oracle
        nh, dk, dv = wl["heads"], wl["dk"], wl["dv"]
        self.S = [synth.host_gdn_state(seed, l, nh, dk, dv).astype(np.float64) for l in range(n_layers)]
        self.toks = [[synth.host_gdn_token(seed, l, t, nh, dk, dv) for t in range(n_tok)] for l in range(n_layers)]
        self.i = 0

    def layer_step_seconds(self):
        l = self.i % len(self.S)
        tok = self.toks[l][(self.i // len(self.S)) % len(self.toks[l])]
        self.i += 1
        t0 = time.perf_counter()
        self.S[l], _ = self.oracle.gdn_step(self.S[l], tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        return time.perf_counter() - t0


def gdn_cpu_baseline(wl, seed, budget_s=10.0):
    smp = GdnOracleSample(wl, seed)
    per = smp.layer_step_seconds()
    n = max(2, min(4000, int(budget_s / max(per, 1e-9))))
    t0 = time.perf_counter()
    tot = sum(smp.layer_step_seconds() for _ in range(n))
    spent = time.perf_counter() - t0
    per_token = tot / n * wl["layers"]      # one sequence's token; the oracle step is per sequence
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} whole layer steps (64 heads x 128x128, fp64 oracle, one thread) over 2 layers' "
                      f"states and 4 tokens each, scaled to {wl['layers']} layers per token; {spent:.1f} s"}


def run_reference_gdn(args, wl):
    """Reference arm of the GatedDeltaNet workload: the oracle's step, at
    most 4 layer steps timed per step and scaled to the 45 layers."""
    K, W = args.steps, args.warmup
    smp = GdnOracleSample(wl, args.seed)
    per = min(smp.layer_step_seconds() for _ in range(2))
    t_timed = max(1, min(4, int((150.0 / (K + W)) / max(per, 1e-9))))
    for _ in range(W * t_timed):
        smp.layer_step_seconds()
    t0 = time.perf_counter()
    total = 0.0
    seqs = wl.get("seqs", 1)
    for _ in range(K):
        # a step: every sequence's token through every layer (the oracle
        # takes one sequence's layer step at a time)
        total += sum(smp.layer_step_seconds() for _ in range(t_timed)) * (wl["layers"] * seqs / t_timed)
    wall = time.perf_counter() - t0
    value = K * seqs / total
    line = {"metric": wl["metric"], "value": value, "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": 1000.0 * total / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl["name"], "tokens_per_step": seqs, "layers": wl["layers"]},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": UNIT,
                             "sample": f"each step: {t_timed} of its {wl['layers'] * seqs} layer steps timed (fp64 "
                                       f"oracle, one thread), scaled; {wall:.2f} s wall for the timed steps"},
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
    ls = LayerSetup(q, wl, seed, dev, n_tok, rank_token_base(10_000_000, rank))
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
        full = args.steps // chunk
        rem = args.steps % chunk
        # timed steps run the stream in order: full graphs, then the rest
        rem_graph = capture(full * chunk, rem) if rem else None
        # warm-up on the stream's last tokens, which the timed steps reach
        # only after n_tok - warmup steps (never, unless they wrap around)
        n_warm = min(args.warmup, chunk * n_chunks)
        warm_graph = capture(chunk * n_chunks - n_warm, n_warm)
    torch.cuda.synchronize()
    if q.qe_workspace_status(ls.ws, s) != q.QE_OK:
        raise RuntimeError("device status after capture: " + q.qe_last_error())

    with torch.cuda.stream(s):
        warm_graph.replay()
    s.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for i in range(full):
            graphs[i % n_chunks].replay()
        if rem_graph is not None:
            rem_graph.replay()
        ev1.record(s)
    s.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1)
    if q.qe_workspace_status(ls.ws, s) != q.QE_OK:
        raise RuntimeError("device status after timing: " + q.qe_last_error())
    ms_max = sync_max(world, dev, ms)
    value = world * args.steps * T / (ms_max / 1000.0)

    # distinct experts touched per step (from the routing of the timed steps)
    idx_h = ls.idx.cpu().numpy().reshape(-1, T * K)
    written = min(len(idx_h), args.steps)  # rows the timed steps wrote (the stream's first steps)
    distinct = float(np.mean([len(np.unique(r)) for r in idx_h[:written]]))

    # ---------------------------------------------------------------- e2e
    n_e2e = min(args.steps, 2048 if T == 1 else 64)
    x_host = ls.x[: max(T, 1) * min(n_e2e, ls.n_tok // T)].cpu().pin_memory()
    out_host = torch.empty((T, H), dtype=torch.float32).pin_memory()
    nb = x_host.shape[0] // T

    def e2e_step(i):
        # one C-ABI call on host buffers: copy in, layer step, copy out, sync
        b = (i % nb) * T
        q.moe_layer_step_host(ls.cfg, ls.layer, x_host[b:b + T], out_host, False, ls.ws, stream=s)

    with torch.cuda.stream(s):
        for i in range(4):
            e2e_step(i)
    barrier(world)
    t0 = time.perf_counter()
    with torch.cuda.stream(s):
        for i in range(n_e2e):
            e2e_step(i)
    e2e_s = sync_max(world, dev, time.perf_counter() - t0)
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
    kern = ("qe_fused_layer_kernel" if T == 1 else
            "grouped_expert_kernel<0> (gate/up) + grouped_expert_kernel<1> (down) (+ route, group, combine)")
    line = {
        "metric": wl["metric"], "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "tokens_per_step": T,
                   "tokens_distinct": min(args.steps * T, ls.n_tok),
                   "warmup_tokens": f"the stream's last {n_warm * T}, disjoint from the first "
                                    f"{ls.n_tok - n_warm * T} timed tokens",
                   "l2": "inputs larger than L2: 3.6 GB expert pool, routing scatters over all 512 experts",
                   "launch": f"CUDA graphs of {chunk} layer steps",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": load_traffic(args.workload), "peak_source": peak_kind,
                     "kernel": kern, "algorithmic_bytes_per_launch": alg,
                     "duration": "whole step (launch gaps included)",
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "frac_basis": "frac: of the measured copy peak; frac_of_nominal_8tbs: of B200's nominal 8 TB/s"},
        "expert_gbs": exp_b / per_step_s / 1e9,
        "expert_frac": exp_b / per_step_s / 1e9 / peak,
        "distinct_experts_per_step": distinct,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * H * ls.x.element_size(),
                "d2h_bytes_per_step": T * H * 4, "steps": n_e2e,
                "how": "per step: moe_layer_step_host on pinned host buffers (H2D of x, layer step, D2H of "
                       "out, stream sync)"},
        # T == 1: the fused kernel; else route norm, logits, top-K, grouping,
        # gate/up, down and combine
        "gpu_launches": args.steps * (1 if T == 1 else 7),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def rank_token_base(base, rank):
    """First token id of a rank's token stream: replicas draw disjoint
    token streams (each rank's stream holds fewer than 10^7 tokens)."""
    return base * (rank + 1)


def sync_max(world, dev, value):
    """Max of a float over ranks (the slowest rank's time)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    tt = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def finish_line(args, wl, world, ms_max, ms, n_units, alg_bytes_per_step, exp_bytes_per_step, distinct, extra,
                e2e, clocks, launches, kernel, duration_note):
    peaks, peak_kind = measured_peaks()
    per_step_s = (ms / 1000.0) / args.steps
    peak = float(peaks["hbm_gbs"])
    achieved = alg_bytes_per_step / per_step_s / 1e9
    cpu = None if args.no_cpu_baseline else cpu_baseline(wl, args.seed)
    line = {
        "metric": wl["metric"], "value": world * n_units / (ms_max / 1000.0), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "parallelism": "replicas" if world > 1 else "single GPU", **extra},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": load_traffic(args.workload), "peak_source": peak_kind, "kernel": kernel,
                     "algorithmic_bytes_per_launch": alg_bytes_per_step, "duration": duration_note,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "frac_basis": "frac: of the measured copy peak; frac_of_nominal_8tbs: of B200's nominal 8 TB/s"},
        "expert_gbs": exp_bytes_per_step / per_step_s / 1e9,
        "expert_frac": exp_bytes_per_step / per_step_s / 1e9 / peak,
        "distinct_experts_per_step": distinct,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


class StackSetup:
    """L resident layers (pool, router, Zipf offset each), 4-bit experts."""

    def __init__(self, q, wl, seed, dev, L):
        import torch
        from _util import dev_router, fill_pool
        H, E, K, I = wl["H"], wl["E"], wl["K"], wl["I"]
        self.cfg = q.Cfg(H, E, K, I, 64, EPS32)
        self.pools, self.W, self.off, self.layers = [], [], [], []
        for l in range(L):
            pool = q.ExpertPool(self.cfg, E, wl["bits"], device=dev)
            fill_pool(pool, seed, l)
            W = dev_router(seed, l, E, H, device=dev)
            o = wl_offset(wl, seed, l)
            off = torch.tensor(o, device=dev) if o is not None else None
            self.pools.append(pool)
            self.W.append(W)
            self.off.append(off)
            self.layers.append(q.Layer(W.data_ptr(), off.data_ptr() if off is not None else None, None,
                                       pool.table.data_ptr()))


def run_stack(args, wl, rank, world, local_rank):
    """One step = one token through all L layers (one fused launch per layer,
    residual between layers); CUDA graphs of 8 tokens."""
    import torch
    import quantized_expert_matvec_b200 as q
    from _util import dev_tokens
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H, E, K, I, L = wl["H"], wl["E"], wl["K"], wl["I"], wl["layers"]
    st = StackSetup(q, wl, args.seed, dev, L)
    ws = q.workspace(st.cfg, 1, device=dev)
    n_tok = 256
    x = dev_tokens(args.seed, rank_token_base(20_000_000, rank), n_tok, H, device=dev)
    act = torch.empty((2, 1, H), dtype=torch.float32, device=dev)
    out = torch.empty((n_tok, H), dtype=torch.float32, device=dev)
    idx = torch.empty((n_tok, L, K), dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(device=dev)

    def token(t, stream, xin=None, dst=None, keep_idx=True):
        cur = x[t:t + 1] if xin is None else xin
        for l in range(L):
            o = (dst if dst is not None else out[t:t + 1]) if l == L - 1 else act[l % 2]
            q.moe_layer_step(st.cfg, st.layers[l], cur, o, True, idx[t, l:l + 1] if keep_idx else None, None,
                             ws, stream=stream)
            cur = o

    chunk = 8
    n_graphs = n_tok // chunk
    with torch.cuda.stream(s):
        token(0, s)
        s.synchronize()
        graphs = []
        for c in range(n_graphs):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for i in range(chunk):
                    token(c * chunk + i, s)
            graphs.append(g)
        rem = args.steps % chunk
        rem_graph = None
        if rem:
            rem_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(rem_graph, stream=s):
                for i in range(rem):
                    token(i, s)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for i in range(max(1, args.warmup // chunk)):
            graphs[i % n_graphs].replay()
    s.synchronize()
    if q.qe_workspace_status(ws, s) != q.QE_OK:
        raise RuntimeError("device status after warm-up: " + q.qe_last_error())
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for i in range(args.steps // chunk):
            graphs[i % n_graphs].replay()
        if rem_graph is not None:
            rem_graph.replay()
        ev1.record(s)
    s.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1)
    if q.qe_workspace_status(ws, s) != q.QE_OK:
        raise RuntimeError("device status after timing: " + q.qe_last_error())
    ms_max = sync_max(world, dev, ms)
    ih = idx.cpu().numpy()
    written = min(n_tok, max(args.steps, chunk))
    distinct = float(np.mean([len(np.unique(ih[t, l])) for t in range(written) for l in range(L)])) * L
    hot_share = None
    if wl.get("zipf"):
        import synth
        hots = [synth.hot_set(args.seed, l, E, E // 4) for l in range(L)]
        hot_share = float(np.mean([hots[l][ih[t, l]].mean() for t in range(written) for l in range(L)]))

    # e2e: per token, pinned H2D of x, the L layer steps, D2H of the output
    n_e2e = min(args.steps, 64)
    x_host = x[:n_e2e].cpu().pin_memory()
    out_host = torch.empty((1, H), dtype=torch.float32).pin_memory()
    xin = torch.empty((1, H), dtype=torch.float32, device=dev)
    res = torch.empty((1, H), dtype=torch.float32, device=dev)

    def e2e_step(i):
        xin.copy_(x_host[i % n_e2e:i % n_e2e + 1], non_blocking=True)
        token(0, s, xin=xin, dst=res, keep_idx=False)
        out_host.copy_(res, non_blocking=True)
        s.synchronize()

    with torch.cuda.stream(s):
        for i in range(2):
            e2e_step(i)
    barrier(world)
    t0 = time.perf_counter()
    with torch.cuda.stream(s):
        for i in range(n_e2e):
            e2e_step(i)
    e2e_s = sync_max(world, dev, time.perf_counter() - t0)
    if rank != 0:
        return
    eb = expert_bytes(H, I, 4)
    alg = distinct * eb + L * (E * H * 4 + 2 * H * 4 + E * 4)
    e2e = {"value": world * n_e2e / e2e_s, "unit": UNIT, "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
           "steps": n_e2e, "how": f"per token: pinned H2D of x, {L} moe_layer_step calls, D2H of out, sync"}
    extra = {"layers": L, "tokens_per_step": 1, "tokens_distinct": n_tok,
             "l2": f"inputs larger than L2: {L * E * eb / 1e9:.0f} GB of experts and {L * E * H * 4 / 1e6:.0f} MB "
                   "of routers, read once per token",
             "launch": f"CUDA graphs of {chunk} tokens x {L} layers", "zipf_alpha": 0.40,
             "share_of_selections_in_hottest_25pct": hot_share}
    finish_line(args, wl, world, ms_max, ms, args.steps, alg, distinct * eb, distinct, extra, e2e, clocks,
                args.steps * L, "qe_fused_layer_kernel (one launch per layer)", "whole step (launch gaps included)")


def pinned_host(nbytes):
    """Page-locked host buffer of exactly nbytes (numpy-owned, registered
    with the CUDA driver and mapped into the device's address space; the
    caller unregisters)."""
    import torch
    buf = np.empty(nbytes + 4096, dtype=np.uint8)
    base = (buf.ctypes.data + 4095) // 4096 * 4096
    rc = torch.cuda.cudart().cudaHostRegister(base, nbytes, 2)  # cudaHostRegisterMapped: the device reads it
    if int(rc) != 0:
        raise MemoryError(f"cudaHostRegister of {nbytes} bytes failed ({rc})")
    return buf, base


def mem_available():
    try:
        for ln in open("/proc/meminfo"):
            if ln.startswith("MemAvailable:"):
                return int(ln.split()[1]) * 1024
    except OSError:
        pass
    return 0


def run_gdn(args, wl, rank, world, local_rank):
    """One step = one token through the GatedDeltaNet recurrence of every
    layer: one gdn_decode_step launch per layer on that layer's resident
    state.  CUDA graphs of 32 tokens; the launches overlap their neighbours'
    tails through programmatic dependent launch."""
    import torch
    import quantized_expert_matvec_b200 as q
    import synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    seqs = wl.get("seqs", 1)
    nh, dk, dv, L = wl["heads"] * seqs, wl["dk"], wl["dv"], wl["layers"]
    S = torch.empty((L, nh, dv, dk), dtype=torch.float32, device=dev)
    for l in range(L):
        S[l].copy_(torch.from_numpy(synth.host_gdn_state(args.seed, l, nh, dk, dv)))
    # per (token, layer) one flat fp32 record: q [nh,dk], k [nh,dk], v [nh,dv], alpha [nh], beta [nh]
    oq, ok_, ov, oa, ob = 0, nh * dk, 2 * nh * dk, 2 * nh * dk + nh * dv, 2 * nh * dk + nh * dv + nh
    rec = ob + nh
    chunk = 32 if seqs == 1 else 8
    tok0 = rank_token_base(20_000_000, rank)
    host_in = np.empty((chunk, L, rec), np.float32)
    for t in range(chunk):
        for l in range(L):
            d = synth.host_gdn_token(args.seed, l, tok0 + t, nh, dk, dv)
            host_in[t, l, oq:ok_] = d["q"].ravel()
            host_in[t, l, ok_:ov] = d["k"].ravel()
            host_in[t, l, ov:oa] = d["v"].ravel()
            host_in[t, l, oa:ob] = d["alpha"]
            host_in[t, l, ob:] = d["beta"]
    inp = torch.from_numpy(host_in).to(dev)
    out = torch.empty((chunk, L, nh, dv), dtype=torch.float32, device=dev)
    s = torch.cuda.Stream(device=dev)

    def token(t, src, dst):
        for l in range(L):
            r = src[t, l]
            q.gdn_decode_step(S[l], r[oq:ok_], r[ok_:ov], r[ov:oa], r[oa:ob], r[ob:], dst[t, l], stream=s)

    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        token(0, inp, out)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for t in range(chunk):
                token(t, inp, out)
    torch.cuda.synchronize()
    reps = max(1, args.steps // chunk)
    args.steps = reps * chunk
    with torch.cuda.stream(s):
        for _ in range(max(1, -(-args.warmup // chunk))):
            g.replay()
    s.synchronize()
    barrier(world)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for _ in range(reps):
            g.replay()
        ev1.record(s)
    s.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1)
    ms_max = sync_max(world, dev, ms)
    if not bool(torch.isfinite(S).all().item()):
        raise RuntimeError("non-finite recurrent state after timing")
    del g

    # e2e: per token, the layers' inputs copied from pinned host memory, the
    # 45 launches, the read-outs copied back, one synchronisation
    n_e2e = min(args.steps, 256 if seqs == 1 else 64)
    pin_in = torch.from_numpy(host_in).pin_memory()
    pin_out = torch.empty((1, L, nh, dv), dtype=torch.float32).pin_memory()
    stage_in = torch.empty((1, L, rec), dtype=torch.float32, device=dev)
    stage_out = torch.empty((1, L, nh, dv), dtype=torch.float32, device=dev)

    def e2e_token(i):
        with torch.cuda.stream(s):
            stage_in.copy_(pin_in[i % chunk:i % chunk + 1], non_blocking=True)
            token(0, stage_in, stage_out)
            pin_out.copy_(stage_out, non_blocking=True)
        s.synchronize()

    for i in range(4):
        e2e_token(i)
    barrier(world)
    t0 = time.perf_counter()
    for i in range(n_e2e):
        e2e_token(i)
    e2e_s = sync_max(world, dev, time.perf_counter() - t0)
    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    per_launch_s = (ms / 1000.0) / (args.steps * L)
    alg = 2 * nh * dv * dk * 4 + rec * 4 + nh * dv * 4
    achieved = alg / per_launch_s / 1e9
    cpu = None if args.no_cpu_baseline else gdn_cpu_baseline(wl, args.seed)
    line = {
        "metric": wl["metric"], "value": world * args.steps * seqs / (ms_max / 1000.0), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "tokens_per_step": seqs, "sequences": seqs, "layers": L,
                   "distinct_token_inputs": chunk,
                   "l2": f"inputs larger than L2: {S.numel() * 4 / 2**20:.0f} MiB of recurrent state plus "
                         f"{inp.numel() * 4 / 1e6:.0f} MB of token inputs",
                   "launch": f"CUDA graphs of {chunk} tokens x {L} launches, programmatic dependent launch",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": load_traffic(args.workload), "peak_source": peak_kind,
                     "kernel": "qe_gdn_step_kernel", "algorithmic_bytes_per_launch": alg,
                     "duration": f"whole step / {L} launches (gaps between launches included)",
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "frac_basis": "frac: of the measured copy peak; frac_of_nominal_8tbs: of B200's nominal 8 TB/s"},
        "us_per_layer_step": 1e6 * per_launch_s,
        "cpu_baseline": cpu,
        "e2e": {"value": world * n_e2e * seqs / e2e_s, "unit": UNIT, "h2d_bytes_per_step": L * rec * 4,
                "d2h_bytes_per_step": L * nh * dv * 4, "steps": n_e2e,
                "how": f"per token: pinned H2D of the {L} layers' q, k, v, alpha, beta; {L} gdn_decode_step "
                       f"calls; D2H of the read-outs; stream sync"},
        "gpu_launches": args.steps * L,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_tiered(args, wl, rank, world, local_rank):
    """One step = one token through all tiered layers: per layer the routing
    kernel (router, top-K and the cache resolve on the device), the fill
    kernel (misses copied from mapped host memory into their slots) and the
    single-token kernel with the given routing, residual added; no host
    synchronisation, so tokens run from CUDA graphs."""
    import torch
    import quantized_expert_matvec_b200 as q
    from _util import dev_router, dev_tokens, fill_pool, fill_pool_slots
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H, E, K, I, L, n_hot = wl["H"], wl["E"], wl["K"], wl["I"], wl["layers"], wl["hot"]
    cfg = q.Cfg(H, E, K, I, 64, EPS32)
    cold_b = q.qe_expert_bytes(cfg, 2)
    n_cold = E - n_hot
    need = L * n_cold * cold_b
    avail = mem_available()
    label = None
    if need > 0.6 * avail:
        L_fit = max(1, int(0.6 * avail // (n_cold * cold_b)))
        label = (f"scaled down to {L_fit} of {L} layers: the cold pool needs {need / 1e9:.1f} GB of pinned host "
                 f"memory, {avail / 1e9:.1f} GB available")
        L = L_fit
    import synth
    hot = [synth.hot_set(args.seed, l, E, n_hot) for l in range(L)]
    # cold pool: generated per layer on the device (2-bit, all experts), the
    # cold ones copied to pinned host memory
    stage = q.ExpertPool(cfg, E, 2, device=dev)
    host_bufs, cold_host = [], []
    for l in range(L):
        fill_pool(stage, args.seed, l)
        buf, base = pinned_host(n_cold * cold_b)
        host_bufs.append((buf, base))
        hv = torch.from_numpy(buf[base - buf.ctypes.data: base - buf.ctypes.data + n_cold * cold_b])
        ptrs = [None] * E
        cold_ids = [e for e in range(E) if not hot[l][e]]
        sv = stage.buf[stage.base - stage.buf.data_ptr():]
        for j, e in enumerate(cold_ids):
            hv[j * cold_b:(j + 1) * cold_b].copy_(sv[e * stage.stride:e * stage.stride + cold_b])
            ptrs[e] = base + j * cold_b
        cold_host.append(ptrs)
    del stage, sv
    torch.cuda.synchronize()
    pools, tables, Ws, offs, layers = [], [], [], [], []
    for l in range(L):
        hot_ids = [e for e in range(E) if hot[l][e]]
        pool = q.ExpertPool(cfg, n_hot, 4, device=dev)
        fill_pool_slots(pool, args.seed, l, hot_ids)
        table = (q.Expert * E)()
        for m, e in enumerate(hot_ids):
            table[e] = pool.host_table[m]
        dtab = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).to(dev)
        W = dev_router(args.seed, l, E, H, device=dev)
        off = torch.tensor(wl_offset(wl, args.seed, l), device=dev)
        pools.append(pool)
        tables.append(dtab)
        Ws.append(W)
        offs.append(off)
        layers.append(q.Layer(W.data_ptr(), off.data_ptr(), None, dtab.data_ptr()))
    tier = q.Tier(cfg, cold_host, 2, int(wl["cache_gb"] * 1e9), max_tokens=1)
    ws = q.workspace(cfg, 1, device=dev)
    args.warmup = -(-args.warmup // 8) * 8      # whole graphs of 8 tokens
    args.steps = max(8, -(-args.steps // 8) * 8)
    n_tok = args.warmup + args.steps
    x = dev_tokens(args.seed, rank_token_base(30_000_000, rank), n_tok, H, device=dev)
    act = torch.empty((2, 1, H), dtype=torch.float32, device=dev)
    idx = torch.empty((n_tok, L, K), dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(device=dev)

    def token(t, xin=None, dst=None):
        cur = x[t:t + 1] if xin is None else xin
        for l in range(L):
            o = dst if (dst is not None and l == L - 1) else act[l % 2]
            tier.layer_step(l, layers[l], cur, o, True, idx[t, l:l + 1] if xin is None else None, None, ws,
                            stream=s)
            cur = o

    # no step waits for the host (hits and misses are resolved on the device),
    # so each chunk of tokens is one CUDA graph; every token runs once, in
    # order, and the cache state carries over from graph to graph
    chunk = 8
    n_chunks = -(-n_tok // chunk)
    torch.cuda.synchronize()
    graphs = []
    with torch.cuda.stream(s):
        for c in range(n_chunks):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for t in range(c * chunk, min(n_tok, (c + 1) * chunk)):
                    token(t)
            graphs.append(g)
    torch.cuda.synchronize()
    n_warm_chunks = -(-args.warmup // chunk)
    with torch.cuda.stream(s):
        for c in range(n_warm_chunks):
            graphs[c].replay()
    s.synchronize()
    h0, m0, b0 = tier.stats()
    barrier(world)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for c in range(n_warm_chunks, n_chunks):
            graphs[c].replay()
        ev1.record(s)
    s.synchronize()
    del graphs
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1)
    if q.qe_workspace_status(ws, s) != q.QE_OK:
        raise RuntimeError("device status after timing: " + q.qe_last_error())
    ms_max = sync_max(world, dev, ms)
    h1, m1, b1 = tier.stats()
    ih = idx[args.warmup:].cpu().numpy()
    cold_sel = float(np.mean([[not hot[l][e] for e in ih[t, l]] for t in range(len(ih)) for l in range(L)]))
    distinct = float(np.mean([len(np.unique(ih[t, l])) for t in range(len(ih)) for l in range(L)])) * L

    n_e2e = min(args.steps, 16)
    x_host = x[:n_e2e].cpu().pin_memory()
    out_host = torch.empty((1, H), dtype=torch.float32).pin_memory()
    xin = torch.empty((1, H), dtype=torch.float32, device=dev)
    res = torch.empty((1, H), dtype=torch.float32, device=dev)
    barrier(world)
    t0 = time.perf_counter()
    with torch.cuda.stream(s):
        for i in range(n_e2e):
            xin.copy_(x_host[i:i + 1], non_blocking=True)
            token(0, xin=xin, dst=res)
            out_host.copy_(res, non_blocking=True)
            s.synchronize()
    e2e_s = sync_max(world, dev, time.perf_counter() - t0)
    tier.close()
    for buf, base in host_bufs:
        torch.cuda.cudart().cudaHostUnregister(base)
    if rank != 0:
        return
    per_tok_hbm = L * ((1 - cold_sel) * K * expert_bytes(H, I, 4) + cold_sel * K * expert_bytes(H, I, 2)
                       + E * H * 4 + 2 * H * 4)
    steps_s = ms / 1000.0
    e2e = {"value": world * n_e2e / e2e_s, "unit": UNIT, "h2d_bytes_per_step": H * 4, "d2h_bytes_per_step": H * 4,
           "steps": n_e2e, "how": f"per token: pinned H2D of x, {L} qe_tier_layer_step calls, D2H of out, sync"}
    extra = {"layers": L, "tokens_per_step": 1, "warmup_tokens_excluded": args.warmup,
             "hot_per_layer": n_hot, "cold_per_layer": n_cold, "cache_gb": wl["cache_gb"],
             "cache_slots": int(wl["cache_gb"] * 1e9 // cold_b), "cold_pool_gb": L * n_cold * cold_b / 1e9,
             "cold_share_of_selections": cold_sel,
             "cache_hit_rate": (h1 - h0) / max(1, (h1 - h0) + (m1 - m0)),
             "h2d_gbs": (b1 - b0) / steps_s / 1e9, "misses_per_token": (m1 - m0) / args.steps,
             "l2": "inputs larger than L2",
             "launch": "CUDA graphs of 8 tokens; hits and misses resolved on the device, no host synchronisation"}
    if label:
        extra["scaled"] = label
    finish_line(args, wl, world, ms_max, ms, args.steps, per_tok_hbm, per_tok_hbm - L * (E * H * 4 + 2 * H * 4),
                distinct, extra, e2e, clocks, args.steps * L * 6,
                "per layer: 3 route kernels, tier_resolve_kernel, tier_fill_kernel, qe_fused_layer_kernel with the "
                "given routing", "whole step (launch gaps included)")


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
    defaults = {"c2": (1024, 32), "c3": (224, 32), "gdn": (4096, 32), "gdn8": (1024, 8)}
    if args.steps is None:
        args.steps = defaults.get(args.workload, (32768 if wl["T"] == 1 else 64, 0))[0]
    if args.warmup is None:
        args.warmup = defaults.get(args.workload, (0, 256 if wl["T"] == 1 else 8))[1]
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
        if args.workload == "c2":
            run_stack(args, wl, rank, world, local_rank)
        elif args.workload == "c3":
            run_tiered(args, wl, rank, world, local_rank)
        elif args.workload in ("gdn", "gdn8"):
            run_gdn(args, wl, rank, world, local_rank)
        else:
            run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
