"""Two-tier expert residency through the C ABI: hot 4-bit experts resident in
HBM, cold 2-bit experts in pinned host memory behind a small HBM slot cache.

Tokens run through a stack of layers with a residual and a Zipf logit offset
per layer (hot = the most popular ranks).  Each layer's output is checked
against the fp64 oracle run on the same input the GPU layer received, and the
cache's hits and misses against a model of its replacement policy.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from _util import (TOL, LruModel, assert_same_routing, dev_router, dev_tokens, fill_host_expert, fill_pool_slots,
                   normwise_err)

pytestmark = pytest.mark.gpu

EPS32 = float(np.float32(1e-6))


@pytest.fixture(scope="module")
def q(cuda):
    import quantized_expert_matvec_b200 as q
    return q


class TieredStack:
    def __init__(self, q, cfg, n_layers, n_hot, seed, cache_slots, max_tokens):
        import torch
        E, H, I = cfg.n_experts, cfg.hidden, cfg.inter
        self.q, self.cfg, self.L, self.seed = q, cfg, n_layers, seed
        self.hot = [synth.hot_set(seed, l, E, n_hot) for l in range(n_layers)]
        self.offset = [synth.zipf_logit_offset(seed, l, E) for l in range(n_layers)]
        cold_b = q.qe_expert_bytes(cfg, 2)
        self.keep = []
        cold_host = []
        self.layers = []
        for l in range(n_layers):
            hot_ids = [e for e in range(E) if self.hot[l][e]]
            cold_ids = [e for e in range(E) if not self.hot[l][e]]
            pool = q.ExpertPool(cfg, len(hot_ids), 4)
            fill_pool_slots(pool, seed, l, hot_ids)
            hbuf = torch.empty(cold_b * len(cold_ids) + 256, dtype=torch.uint8).pin_memory()
            base = (hbuf.data_ptr() + 255) // 256 * 256
            _, seg = q.qe_pool_table(cfg, base, 2, 1)
            ptrs = [None] * E
            for j, e in enumerate(cold_ids):
                fill_host_expert(base + j * cold_b, seg, seed, l, e, H, I, 2)
                ptrs[e] = base + j * cold_b
            cold_host.append(ptrs)
            table = (q.Expert * E)()
            for m, e in enumerate(hot_ids):
                table[e] = pool.host_table[m]
            dtab = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).cuda()
            W = dev_router(seed, l, E, H)
            off = torch.tensor(self.offset[l], device="cuda")
            lw = q.Layer(W.data_ptr(), off.data_ptr(), None, dtab.data_ptr())
            self.keep += [pool, hbuf, dtab, W, off]
            self.layers.append(lw)
        self.cold_host = cold_host
        self.tables = [self.keep[5 * l + 2] for l in range(n_layers)]
        self.tier = q.Tier(cfg, cold_host, 2, cache_slots * cold_b, max_tokens=max_tokens)
        self.ws = q.workspace(cfg, max_tokens)
        self.W_host = [synth.host_router(seed, l, E, H) for l in range(n_layers)]
        self.experts = {}

    def bits_of(self, l):
        return lambda e: 4 if self.hot[l][e] else 2

    def host_expert(self, l, e):
        if (l, e) not in self.experts:
            self.experts[(l, e)] = synth.host_expert(self.seed, l, e, self.cfg.hidden, self.cfg.inter,
                                                     self.bits_of(l)(e))
        return self.experts[(l, e)]

    def oracle(self, l, x64):
        return oracle.layer_step(x64, self.W_host[l], lambda e: self.host_expert(l, e), self.bits_of(l),
                                 self.cfg.top_k, eps=EPS32, offset=self.offset[l], residual=True, nthreads=8)


def test_tiered_stack_matches_oracle_and_lru_model(q):
    import torch
    cfg = q.Cfg(1024, 32, 4, 256)
    st = TieredStack(q, cfg, n_layers=3, n_hot=8, seed=3, cache_slots=6, max_tokens=4)
    assert st.tier.slots == 6
    model = LruModel(6)
    K, H, E = cfg.top_k, cfg.hidden, cfg.n_experts
    x = dev_tokens(3, 500, 10, H)
    n_checked = 0
    for t in range(10):
        cur = x[t:t + 1].clone()
        for l in range(3):
            out = torch.empty((1, H), dtype=torch.float32, device="cuda")
            idx = torch.empty((1, K), dtype=torch.int32, device="cuda")
            w = torch.empty((1, K), dtype=torch.float32, device="cuda")
            st.tier.layer_step(l, st.layers[l], cur, out, True, idx, w, st.ws)
            assert q.qe_workspace_status(st.ws) == q.QE_OK, q.qe_last_error()
            idx_h = idx.cpu().numpy()[0]
            model.call([l * E + int(e) for e in idx_h if not st.hot[l][int(e)]])
            ref = st.oracle(l, cur.cpu().numpy()[0].astype(np.float64))
            assert_same_routing(idx_h, ref["idx"], ref["logits"])
            assert np.allclose(w.cpu().numpy()[0], ref["w"], rtol=2e-6, atol=1e-7)
            err = normwise_err(out.cpu().numpy()[0], ref["out"])
            assert err <= TOL, (t, l, err)
            n_checked += 1
            cur = out
    hits, misses, h2d = st.tier.stats()
    assert (hits, misses) == (model.hits, model.misses)
    assert h2d == misses * q.qe_expert_bytes(cfg, 2)
    assert misses > 6 and hits > 0  # evictions happened and reuse happened
    assert n_checked == 30


def test_tiered_batched_call_and_oom(q):
    """Four tokens in one call (grouped experts) against the oracle; a cache
    smaller than one call's cold experts is refused with QE_ERR_OOM."""
    import torch
    cfg = q.Cfg(1024, 32, 4, 256)
    st = TieredStack(q, cfg, n_layers=1, n_hot=8, seed=4, cache_slots=16, max_tokens=4)
    K, H, E = cfg.top_k, cfg.hidden, cfg.n_experts
    x = dev_tokens(4, 900, 4, H)
    out = torch.empty((4, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((4, K), dtype=torch.int32, device="cuda")
    w = torch.empty((4, K), dtype=torch.float32, device="cuda")
    st.tier.layer_step(0, st.layers[0], x, out, True, idx, w, st.ws)
    assert q.qe_workspace_status(st.ws) == q.QE_OK, q.qe_last_error()
    oh, ih, wh = out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    for t in range(4):
        ref = st.oracle(0, x[t].cpu().numpy().astype(np.float64))
        assert_same_routing(ih[t], ref["idx"], ref["logits"])
        assert normwise_err(oh[t], ref["out"]) <= TOL
    n_cold = len({int(e) for e in ih.reshape(-1) if not st.hot[0][int(e)]})
    hits, misses, _ = st.tier.stats()
    assert (hits, misses) == (0, n_cold)

    small = q.Tier(cfg, st.cold_host, 2, q.qe_expert_bytes(cfg, 2), max_tokens=4)
    assert small.slots == 1
    assert n_cold > 1
    with pytest.raises(q.QEError) as ei:
        small.resolve(0, ih.reshape(-1), st.tables[0])
    assert ei.value.code == q.QE_ERR_OOM
    assert small.stats() == (0, 0, 0)
    small.close()


def test_tiered_full_layer_shape(q):
    """The tiered workload's layer shape (hidden 4096, 512 experts: the 128
    most popular 4-bit in HBM, 384 2-bit in pinned host memory), two layers,
    a 48-slot cache, six tokens; every layer output against the oracle."""
    import torch
    cfg = q.Cfg(4096, 512, 4, 1024)
    st = TieredStack(q, cfg, n_layers=2, n_hot=128, seed=0, cache_slots=48, max_tokens=1)
    model = LruModel(48)
    K, H, E = cfg.top_k, cfg.hidden, cfg.n_experts
    x = dev_tokens(0, 123_000, 6, H)
    n_ok = 0
    for t in range(6):
        cur = x[t:t + 1].clone()
        for l in range(2):
            out = torch.empty((1, H), dtype=torch.float32, device="cuda")
            idx = torch.empty((1, K), dtype=torch.int32, device="cuda")
            st.tier.layer_step(l, st.layers[l], cur, out, True, idx, None, st.ws)
            idx_h = idx.cpu().numpy()[0]
            model.call([l * E + int(e) for e in idx_h if not st.hot[l][int(e)]])
            ref = st.oracle(l, cur.cpu().numpy()[0].astype(np.float64))
            assert_same_routing(idx_h, ref["idx"], ref["logits"])
            assert normwise_err(out.cpu().numpy()[0], ref["out"]) <= TOL
            n_ok += 1
            cur = out
    assert q.qe_workspace_status(st.ws) == q.QE_OK, q.qe_last_error()
    hits, misses, _ = st.tier.stats()
    assert (hits, misses) == (model.hits, model.misses)
    assert n_ok == 12
    st.tier.close()


def test_tiered_tokens_captured_in_a_cuda_graph(q):
    """Hits and misses are resolved on the device, so whole tokens through
    the tiered stack capture into one CUDA graph (a host synchronisation
    inside would fail the capture).  Replayed once, the graph gives the same
    routing, outputs and cache counters as the LRU model and the oracle."""
    import torch
    cfg = q.Cfg(1024, 32, 4, 256)
    st = TieredStack(q, cfg, n_layers=3, n_hot=8, seed=5, cache_slots=6, max_tokens=1)
    model = LruModel(6)
    K, H, E, L, NT = cfg.top_k, cfg.hidden, cfg.n_experts, 3, 5
    x = dev_tokens(5, 700, NT, H)
    acts = torch.empty((NT, L, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((NT, L, K), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for t in range(NT):
            cur = x[t:t + 1]
            for l in range(L):
                st.tier.layer_step(l, st.layers[l], cur, acts[t, l:l + 1], True, idx[t, l:l + 1], None, st.ws,
                                   stream=s)
                cur = acts[t, l:l + 1]
    assert st.tier.stats() == (0, 0, 0)  # capturing ran nothing
    g.replay()
    torch.cuda.synchronize()
    assert q.qe_workspace_status(st.ws) == q.QE_OK, q.qe_last_error()
    ih, ah = idx.cpu().numpy(), acts.cpu().numpy()
    for t in range(NT):
        cur = x[t].cpu().numpy().astype(np.float64)
        for l in range(L):
            model.call([l * E + int(e) for e in ih[t, l] if not st.hot[l][int(e)]])
            ref = st.oracle(l, cur)
            assert_same_routing(ih[t, l], ref["idx"], ref["logits"])
            assert normwise_err(ah[t, l], ref["out"]) <= TOL, (t, l)
            cur = ah[t, l].astype(np.float64)
    hits, misses, h2d = st.tier.stats()
    assert (hits, misses) == (model.hits, model.misses)
    assert misses > 6 and hits > 0
    del g
    st.tier.close()


def test_tiered_refusals_before_launch(q):
    """A layer step whose T * top_k cold experts might not fit the cache is
    refused on the host; cold experts in pageable (not page-locked) memory are
    refused at creation, since the device cannot read them."""
    import torch
    cfg = q.Cfg(1024, 32, 4, 256)
    st = TieredStack(q, cfg, n_layers=1, n_hot=8, seed=6, cache_slots=6, max_tokens=2)
    x = dev_tokens(6, 10, 2, cfg.hidden)
    out = torch.empty((2, cfg.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(q.QEError) as ei:
        st.tier.layer_step(0, st.layers[0], x, out, True, None, None, st.ws)  # 2 * 4 > 6 slots
    assert ei.value.code == q.QE_ERR_OOM
    assert st.tier.stats() == (0, 0, 0)
    st.tier.close()
    cold_b = q.qe_expert_bytes(cfg, 2)
    pageable = np.zeros(cold_b + 256, np.uint8)
    base = (pageable.ctypes.data + 255) // 256 * 256
    cold = [[base if e == 0 else None for e in range(cfg.n_experts)]]
    with pytest.raises(q.QEError) as ei:
        q.Tier(cfg, cold, 2, 4 * cold_b, max_tokens=1)
    assert ei.value.code == q.QE_ERR_INVALID_ARG
    assert "page-locked" in str(ei.value)
