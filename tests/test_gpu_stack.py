"""The 40-layer stack at full size (hidden 4096, 512 experts, top-4,
intermediate 1024, 4-bit, 145 GB of experts in HBM, residual between layers,
Zipf popularity offsets): tokens run through all layers with the fused
single-token kernel, as the benchmark runs them; sampled layer outputs are
compared with the fp64 oracle run on the input that GPU layer received."""
import gc

import numpy as np
import pytest

import oracle
import synth
from _util import TOL, assert_same_routing, dev_router, dev_tokens, fill_pool, normwise_err

pytestmark = pytest.mark.gpu

EPS32 = float(np.float32(1e-6))


def test_stack_40_layers_full_size(cuda):
    import torch
    import quantized_expert_matvec_b200 as q
    gc.collect()
    torch.cuda.empty_cache()
    H, E, K, I, L, seed = 4096, 512, 4, 1024, 40, 0
    cfg = q.Cfg(H, E, K, I, 64, EPS32)
    free, _ = torch.cuda.mem_get_info()
    need = L * (q.qe_expert_bytes(cfg, 4) * E + E * H * 4) + (2 << 30)
    if free < need:
        pytest.skip(f"needs {need / 1e9:.0f} GB of free device memory, {free / 1e9:.0f} GB free")
    pools, Ws, offs, layers = [], [], [], []
    for l in range(L):
        pool = q.ExpertPool(cfg, E, 4)
        fill_pool(pool, seed, l)
        W = dev_router(seed, l, E, H)
        off_h = synth.zipf_logit_offset(seed, l, E)
        off = torch.tensor(off_h, device="cuda")
        pools.append(pool)
        Ws.append(W)
        offs.append(off_h)
        layers.append(q.Layer(W.data_ptr(), off.data_ptr(), None, pool.table.data_ptr()))
        pools.append(off)
    ws = q.workspace(cfg, 1)
    x = dev_tokens(seed, 77_000, 3, H)
    ins, outs, idxs = [], [], []
    for t in range(3):
        cur = x[t:t + 1].clone()
        tin, tout, tidx = [], [], []
        for l in range(L):
            o = torch.empty((1, H), dtype=torch.float32, device="cuda")
            idx = torch.empty((1, K), dtype=torch.int32, device="cuda")
            q.moe_layer_step(cfg, layers[l], cur, o, True, idx, None, ws)
            tin.append(cur)
            tout.append(o)
            tidx.append(idx)
            cur = o
        ins.append(tin)
        outs.append(tout)
        idxs.append(tidx)
    assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    # token 0: every layer; tokens 1, 2: every 7th layer
    checks = [(0, l) for l in range(L)] + [(t, l) for t in (1, 2) for l in range(t, L, 7)]
    hot_hits = 0
    n_ok = 0
    for t, l in checks:
        xin = ins[t][l].cpu().numpy()[0].astype(np.float64)
        W_h = synth.host_router(seed, l, E, H)
        ref = oracle.layer_step(xin, W_h, lambda e: synth.host_expert(seed, l, e, H, I, 4), lambda e: 4, K,
                                eps=EPS32, offset=offs[l], residual=True, nthreads=16)
        got = idxs[t][l].cpu().numpy()[0]
        assert_same_routing(got, ref["idx"], ref["logits"])
        hot_hits += int(synth.hot_set(seed, l, E, E // 4)[got].sum())
        err = normwise_err(outs[t][l].cpu().numpy()[0], ref["out"])
        assert err <= TOL, (t, l, err)
        n_ok += 1
    assert n_ok == len(checks)
    # the Zipf offset concentrates selections on the hottest quarter of experts
    assert hot_hits / (K * len(checks)) > 0.5
    del pools, Ws, layers, ws, ins, outs, idxs
    gc.collect()
    torch.cuda.empty_cache()
