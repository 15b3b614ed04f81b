"""Parity of the CUDA library (called through the C ABI) with the fp64 oracle.

Routing must match bit for bit (ties to the lower index; at an oracle
near-tie below 1e-9 relative either expert is accepted); every output must be
within 2e-3 max normwise relative error of the oracle (fp32 accumulation
against fp64).
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from _util import (TOL, HostExperts, assert_same_routing, dev_router, dev_tokens, fill_pool, host_x_f64,
                   normwise_err)

pytestmark = pytest.mark.gpu

EPS32 = float(np.float32(1e-6))


@pytest.fixture(scope="module")
def q(cuda):
    import quantized_expert_matvec_b200 as q
    return q


class DevLayer:
    """One MoE layer on the device (pools, descriptor table, router) and its
    host twin for the oracle, all from the seeded generator."""

    def __init__(self, q, cfg, seed, layer, bits_of=None, offset=None, gamma=None):
        import torch
        self.cfg, self.seed, self.layer = cfg, seed, layer
        E, H, I = cfg.n_experts, cfg.hidden, cfg.inter
        self.bits_of = bits_of or (lambda e: 4)
        need = sorted({self.bits_of(e) for e in range(E)})
        self.pools = {b: q.ExpertPool(cfg, E, b) for b in need}
        for p in self.pools.values():
            fill_pool(p, seed, layer)
        table = (q.Expert * E)()
        for e in range(E):
            table[e] = self.pools[self.bits_of(e)].host_table[e]
        self.table = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).cuda()
        self.W = dev_router(seed, layer, E, H)
        self.W_host = synth.host_router(seed, layer, E, H)
        self.offset = offset
        self.offset_dev = torch.tensor(offset, device="cuda") if offset is not None else None
        self.gamma = gamma
        self.gamma_dev = torch.tensor(gamma, dtype=torch.float32, device="cuda") if gamma is not None else None
        self.layer_struct = q.Layer(self.W.data_ptr(),
                                    self.offset_dev.data_ptr() if offset is not None else None,
                                    self.gamma_dev.data_ptr() if gamma is not None else None,
                                    self.table.data_ptr())
        self.experts = HostExperts(seed, layer, H, I, self.bits_of)

    def oracle(self, x_host, residual=False):
        return oracle.layer_step(x_host, self.W_host, self.experts, self.bits_of, self.cfg.top_k, eps=EPS32,
                                 gamma=None if self.gamma is None else np.asarray(self.gamma, np.float64),
                                 offset=self.offset, residual=residual, nthreads=8)


def run_fused(q, dl, x, residual=False, ws=None):
    import torch
    T = x.shape[0]
    K, H = dl.cfg.top_k, dl.cfg.hidden
    ws = ws if ws is not None else q.workspace(dl.cfg, 1)
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    for t in range(T):
        q.moe_layer_step(dl.cfg, dl.layer_struct, x[t:t + 1], out[t:t + 1], residual, idx[t:t + 1], w[t:t + 1], ws)
    assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    return out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def check(dl, out, idx, w, ref, tol=TOL):
    """Routing bit-exact (no token excused as a near-tie), softmax weights
    to fp32 rounding, the output within the normwise tolerance."""
    assert_same_routing(idx, ref["idx"], ref["logits"])
    assert np.allclose(w, ref["w"], rtol=2e-6, atol=1e-7), (w, ref["w"])
    err = normwise_err(out, ref["out"])
    assert err <= tol, err
    return err


# ---------------------------------------------------------------- fused, T = 1

@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("residual", [False, True])
def test_fused_tiny_layer(q, bits, residual):
    """hidden 256, 16 experts, top-2, intermediate 64 (the tiny workload)."""
    cfg = q.Cfg(256, 16, 2, 64)
    dl = DevLayer(q, cfg, seed=0, layer=0, bits_of=lambda e: bits)
    x = dev_tokens(0, 0, 16, 256)
    out, idx, w = run_fused(q, dl, x, residual)
    errs = []
    for t in range(16):
        ref = dl.oracle(host_x_f64(0, t, 256), residual)
        errs.append(check(dl, out[t], idx[t], w[t], ref))
    assert max(errs) < 1e-5


@pytest.mark.parametrize("H", [768, 320])
def test_ragged_mixed_bits_gamma_offset(q, H):
    """Odd sizes (intermediate 192, 37 experts, top-3): rows do not divide
    evenly over the CTAs; half the experts are 2-bit; random gamma and a Zipf
    logit offset.  At hidden 320 and 768 one warp covers a whole gate/up row,
    with 10 and 24 of its 32 lanes holding a 32-column chunk."""
    cfg = q.Cfg(H, 37, 3, 192)
    gamma = np.random.default_rng(1).uniform(0.5, 1.5, H).astype(np.float32)
    off = synth.zipf_logit_offset(5, 1, 37)
    dl = DevLayer(q, cfg, seed=5, layer=1, bits_of=lambda e: 4 if e % 2 == 0 else 2, offset=off, gamma=gamma)
    x = dev_tokens(5, 100, 12, H)
    out, idx, w = run_fused(q, dl, x, residual=True)
    for t in range(12):
        ref = dl.oracle(host_x_f64(5, 100 + t, H), residual=True)
        check(dl, out[t], idx[t], w[t], ref)


def test_fused_k_equals_e_and_k1(q):
    for (E, K) in ((8, 8), (16, 1)):
        cfg = q.Cfg(256, E, K, 64)
        dl = DevLayer(q, cfg, seed=2, layer=0)
        x = dev_tokens(2, 0, 4, 256)
        out, idx, w = run_fused(q, dl, x)
        for t in range(4):
            check(dl, out[t], idx[t], w[t], dl.oracle(host_x_f64(2, t, 256)))


def test_fused_one_hot_router(q):
    """A +1000 logit offset on expert e gives weights exactly (1, 0) and the
    layer output equals expert e's output."""
    cfg = q.Cfg(256, 16, 2, 64)
    for e in (3, 15):
        off = np.zeros(16, np.float32)
        off[e] = 1000.0
        dl = DevLayer(q, cfg, seed=4, layer=0, offset=off)
        x = dev_tokens(4, 0, 2, 256)
        out, idx, w = run_fused(q, dl, x)
        for t in range(2):
            assert idx[t][0] == e and w[t][0] == 1.0 and w[t][1] == 0.0
            ye = oracle.expert_ffn(dl.experts(e), 4, oracle.rmsnorm(host_x_f64(4, t, 256), None, EPS32))
            assert normwise_err(out[t], ye) < 1e-5


def test_fused_bf16_input(q):
    cfg = q.Cfg(256, 16, 2, 64)
    dl = DevLayer(q, cfg, seed=6, layer=0)
    x = dev_tokens(6, 0, 4, 256, bf16=True)
    out, idx, w = run_fused(q, dl, x, residual=True)
    for t in range(4):
        check(dl, out[t], idx[t], w[t], dl.oracle(host_x_f64(6, t, 256, bf16=True), residual=True))


def test_fused_large_hidden_many_experts(q):
    """hidden 8192 (the largest supported), top-16 of 32 experts."""
    cfg = q.Cfg(8192, 32, 16, 256)
    dl = DevLayer(q, cfg, seed=8, layer=0)
    x = dev_tokens(8, 0, 2, 8192)
    out, idx, w = run_fused(q, dl, x)
    for t in range(2):
        check(dl, out[t], idx[t], w[t], dl.oracle(host_x_f64(8, t, 8192)))


# ---------------------------------------------------- C1: bench configuration

@pytest.fixture(scope="module")
def c1_layer(q):
    """One decode layer shaped like the pages' model: hidden 4096, 512
    experts, top-4, intermediate 1024, all 4-bit experts resident in HBM."""
    cfg = q.Cfg(4096, 512, 4, 1024)
    return DevLayer(q, cfg, seed=0, layer=0)


def test_c1_graph_stream_sampled(q, c1_layer):
    """The launch configuration the benchmark times: a CUDA graph of
    single-token layer steps over distinct tokens; sampled tokens are checked
    against the oracle."""
    import torch
    dl = c1_layer
    n = 48
    x = dev_tokens(0, 0, n, 4096)
    out = torch.zeros((n, 4096), dtype=torch.float32, device="cuda")
    idx = torch.zeros((n, 4), dtype=torch.int32, device="cuda")
    w = torch.zeros((n, 4), dtype=torch.float32, device="cuda")
    ws = q.workspace(dl.cfg, 1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q.moe_layer_step(dl.cfg, dl.layer_struct, x[0:1], out[0:1], False, idx[0:1], w[0:1], ws, stream=s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for t in range(n):
                q.moe_layer_step(dl.cfg, dl.layer_struct, x[t:t + 1], out[t:t + 1], False, idx[t:t + 1],
                                 w[t:t + 1], ws, stream=s)
        out.zero_()
        g.replay()
        g.replay()
        s.synchronize()
    assert q.qe_workspace_status(ws, s) == q.QE_OK
    out_h, idx_h, w_h = out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    for t in (0, 1, 17, 30, 46, 47):
        ref = dl.oracle(host_x_f64(0, t, 4096))
        check(dl, out_h[t], idx_h[t], w_h[t], ref)


def test_c1_standalone_calls(q, c1_layer):
    """moe_route, moe_expert_ffn_q4 and moe_combine on 3 tokens of the C1 layer."""
    import torch
    dl = c1_layer
    cfg = dl.cfg
    T = 3
    x = dev_tokens(0, 500, T, 4096)
    xn = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    y = torch.empty((T, 4, 4096), dtype=torch.float32, device="cuda")
    out = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, T)
    q.moe_route(cfg, x, None, dl.W, None, xn, idx, w, ws)
    q.moe_expert_ffn_q4(cfg, dl.table, xn, idx, y, ws)
    q.moe_combine(y, w, x, out)
    assert q.qe_workspace_status(ws) == q.QE_OK
    xn_h, idx_h, w_h, y_h, out_h = (a.cpu().numpy() for a in (xn, idx, w, y, out))
    for t in range(T):
        xh = host_x_f64(0, 500 + t, 4096)
        ref = dl.oracle(xh, residual=True)
        assert np.max(np.abs(xn_h[t] - ref["xn"])) <= 1e-6 * np.max(np.abs(ref["xn"]))
        assert list(idx_h[t]) == list(ref["idx"])
        for k in range(4):
            assert normwise_err(y_h[t, k], ref["y"][k]) <= TOL
        assert normwise_err(out_h[t], ref["out"]) <= TOL


@pytest.mark.parametrize("mode", ["q2", "mixed"])
def test_standalone_ffn_q2_and_mixed(q, mode):
    import torch
    cfg = q.Cfg(512, 16, 4, 128)
    bits_of = (lambda e: 2) if mode == "q2" else (lambda e: 4 if e < 8 else 2)
    dl = DevLayer(q, cfg, seed=9, layer=3, bits_of=bits_of)
    T = 5
    x = dev_tokens(9, 0, T, 512)
    xn = torch.empty((T, 512), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    y = torch.empty((T, 4, 512), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, T)
    q.moe_route(cfg, x, None, dl.W, None, xn, idx, w, ws)
    (q.moe_expert_ffn_q2 if mode == "q2" else q.moe_expert_ffn_mixed)(cfg, dl.table, xn, idx, y, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK
    for t in range(T):
        ref = dl.oracle(host_x_f64(9, t, 512))
        assert list(idx[t].cpu().numpy()) == list(ref["idx"])
        for k in range(4):
            assert normwise_err(y[t, k].cpu().numpy(), ref["y"][k]) <= TOL


def test_ffn_q4_rejects_2bit_descriptor(q):
    import torch
    cfg = q.Cfg(256, 16, 2, 64)
    dl = DevLayer(q, cfg, seed=1, layer=0, bits_of=lambda e: 2)
    xn = torch.ones((1, 256), dtype=torch.float32, device="cuda")
    idx = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    y = torch.zeros((1, 2, 256), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, 1)
    q.moe_expert_ffn_q4(cfg, dl.table, xn, idx, y, ws)
    assert q.qe_workspace_status(ws) == q.QE_ERR_INVALID_ARG
    assert q.qe_workspace_status(ws) == q.QE_OK  # cleared


# ------------------------------------------------------------- batched, T > 1

@pytest.mark.parametrize("bf16", [False, True])
def test_batched_layer_step_tiny(q, bf16):
    import torch
    cfg = q.Cfg(256, 16, 2, 64)
    dl = DevLayer(q, cfg, seed=11, layer=0)
    T = 24
    x = dev_tokens(11, 0, T, 256, bf16=bf16)
    out = torch.empty((T, 256), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 2), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, T)
    q.moe_layer_step(cfg, dl.layer_struct, x, out, False, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK
    out_h, idx_h, w_h = out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    for t in range(T):
        check(dl, out_h[t], idx_h[t], w_h[t], dl.oracle(host_x_f64(11, t, 256, bf16=bf16)))


def test_batched_c1_bf16_sampled(q, c1_layer):
    """Batched decode of the C1 layer: 64 bf16 tokens in one step; sampled
    tokens checked."""
    import torch
    dl = c1_layer
    T = 64
    x = dev_tokens(0, 1000, T, 4096, bf16=True)
    out = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    ws = q.workspace(dl.cfg, T)
    q.moe_layer_step(dl.cfg, dl.layer_struct, x, out, False, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK
    out_h, idx_h, w_h = out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    for t in (0, 13, 63):
        check(dl, out_h[t], idx_h[t], w_h[t], dl.oracle(host_x_f64(0, 1000 + t, 4096, bf16=True)))


# ---------------------------------------------------------- failure handling

def test_bounded_wait_times_out_and_recovers(q):
    """A CTA that never arrives at the routing barrier makes every other
    CTA's bounded wait give up: the workspace reports QE_ERR_TIMEOUT, and
    after re-initialising it the next step is correct."""
    import torch
    cfg = q.Cfg(256, 16, 2, 64)
    dl = DevLayer(q, cfg, seed=0, layer=0)
    x = dev_tokens(0, 0, 1, 256)
    ws = q.workspace(cfg, 1)
    out = torch.zeros((1, 256), dtype=torch.float32, device="cuda")
    q.qe_set_wait_budget_ns(20_000_000)
    q.qe_test_skip_arrival(5)
    try:
        q.moe_layer_step(cfg, dl.layer_struct, x, out, False, None, None, ws)
        assert q.qe_workspace_status(ws) == q.QE_ERR_TIMEOUT
    finally:
        q.qe_test_skip_arrival(-1)
        q.qe_set_wait_budget_ns(200_000_000)
    q.qe_workspace_init(ws)
    o, i, w = run_fused(q, dl, x, ws=ws)
    check(dl, o[0], i[0], w[0], dl.oracle(host_x_f64(0, 0, 256)))


def test_c1_fused_matches_multikernel_path_on_many_tokens(q, c1_layer):
    """256 tokens through the fused kernel (a CUDA graph of single-token
    steps) against the separate route / expert-FFN / combine kernels on the
    same tokens.  Both are fp32 GPU paths, so they agree far inside the oracle
    tolerance; a missed barrier inside the fused kernel would read
    unfinished partial sums and show up here."""
    import torch
    dl = c1_layer
    cfg = dl.cfg
    n = 256
    x = dev_tokens(0, 20000, n, 4096)
    out = torch.zeros((n, 4096), dtype=torch.float32, device="cuda")
    idx = torch.zeros((n, 4), dtype=torch.int32, device="cuda")
    ws = q.workspace(cfg, 1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q.moe_layer_step(cfg, dl.layer_struct, x[0:1], out[0:1], True, idx[0:1], None, ws, stream=s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for t in range(n):
                q.moe_layer_step(cfg, dl.layer_struct, x[t:t + 1], out[t:t + 1], True, idx[t:t + 1], None, ws,
                                 stream=s)
        g.replay()
        s.synchronize()
    assert q.qe_workspace_status(ws, s) == q.QE_OK
    xn = torch.empty((n, 4096), dtype=torch.float32, device="cuda")
    idx2 = torch.empty((n, 4), dtype=torch.int32, device="cuda")
    w2 = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    y2 = torch.empty((n, 4, 4096), dtype=torch.float32, device="cuda")
    out2 = torch.empty((n, 4096), dtype=torch.float32, device="cuda")
    ws2 = q.workspace(cfg, n)
    q.moe_route(cfg, x, None, dl.W, None, xn, idx2, w2, ws2)
    q.moe_expert_ffn_q4(cfg, dl.table, xn, idx2, y2, ws2)
    q.moe_combine(y2, w2, x, out2)
    assert q.qe_workspace_status(ws2) == q.QE_OK
    same = (idx == idx2).all(dim=1)
    assert int(same.sum()) >= n - 2
    a, b = out[same].double(), out2[same].double()
    err = ((a - b).abs().amax(dim=1) / b.abs().amax(dim=1)).max().item()
    assert err < 2e-5, err


def test_batched_skewed_routing_many_tokens_per_expert(q):
    """Every token's top expert is the same (a +8 logit offset), so one
    expert serves all 40 tokens: several token tiles over its weights."""
    import torch
    cfg = q.Cfg(512, 32, 2, 128)
    off = np.zeros(32, np.float32)
    off[7] = 8.0
    dl = DevLayer(q, cfg, seed=12, layer=0, offset=off)
    T = 40
    x = dev_tokens(12, 0, T, 512)
    out = torch.empty((T, 512), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 2), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, T)
    q.moe_layer_step(cfg, dl.layer_struct, x, out, True, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK
    idx_h = idx.cpu().numpy()
    assert (idx_h[:, 0] == 7).all()
    out_h, w_h = out.cpu().numpy(), w.cpu().numpy()
    for t in range(0, T, 3):
        check(dl, out_h[t], idx_h[t], w_h[t], dl.oracle(host_x_f64(12, t, 512), residual=True))


def test_batched_c4_full_step_sampled(q, c1_layer):
    """The batched workload at full size: 256 bf16 tokens, top-4 of 512,
    grouped experts; sampled tokens against the oracle."""
    import torch
    dl = c1_layer
    T = 256
    x = dev_tokens(0, 50000, T, 4096, bf16=True)
    out = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    ws = q.workspace(dl.cfg, T)
    for _ in range(2):  # the second step reuses the workspace
        q.moe_layer_step(dl.cfg, dl.layer_struct, x, out, False, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK
    out_h, idx_h, w_h = out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    for t in (0, 100, 255):
        check(dl, out_h[t], idx_h[t], w_h[t], dl.oracle(host_x_f64(0, 50000 + t, 4096, bf16=True)))


def test_batched_tensor_core_groups_full_shape(q):
    """Hidden 4096, intermediate 1024: a +8 logit offset on four experts (two
    4-bit, two 2-bit) sends all 150 tokens to them: groups far above the
    8-token pass of the grouped kernels; sampled tokens against the oracle."""
    import torch
    cfg = q.Cfg(4096, 64, 4, 1024)
    off = np.zeros(64, np.float32)
    hot = [3, 10, 21, 40]
    off[hot] = 8.0
    dl = DevLayer(q, cfg, seed=31, layer=0, bits_of=lambda e: 2 if e % 2 else 4, offset=off)
    T = 150
    x = dev_tokens(31, 7000, T, 4096, bf16=True)
    ws = q.workspace(cfg, T)
    out = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    q.moe_layer_step(cfg, dl.layer_struct, x, out, True, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    ih = idx.cpu().numpy()
    assert all(sorted(r) == hot for r in ih.tolist())
    oh = out.cpu().numpy()
    xb = x.cpu().view(torch.int16).numpy().astype(np.uint16)
    for t in (0, 77, 128, 149):
        x64 = (xb[t].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ref = dl.oracle(x64, residual=True)
        assert list(ih[t]) == list(ref["idx"])
        err = normwise_err(oh[t], ref["out"])
        assert err <= TOL, (t, err)


def test_layer_step_on_host_buffers(q, c1_layer):
    """moe_layer_step_host (host buffers in and out) gives exactly what
    moe_layer_step gives on device buffers, for one token (fused kernel) and
    for five (batched path)."""
    import torch
    dl = c1_layer
    for T, bf16 in ((1, False), (5, True)):
        x = dev_tokens(0, 9100 + T, T, 4096, bf16=bf16)
        ws = q.workspace(dl.cfg, T)
        ref = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
        q.moe_layer_step(dl.cfg, dl.layer_struct, x, ref, True, None, None, ws)
        assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
        xh = x.cpu().pin_memory()
        oh = torch.empty((T, 4096), dtype=torch.float32).pin_memory()
        q.moe_layer_step_host(dl.cfg, dl.layer_struct, xh, oh, True, ws)
        assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
        assert torch.equal(oh, ref.cpu())


def test_hidden_2048_mixed_bits_single_and_batched(q):
    """Hidden 2048 (two warps per gate/up row), 64 experts,
    top-4, intermediate 512, every third expert 2-bit, Zipf offset, residual:
    one token at a time through the fused kernel and six tokens through the
    batched path, all against the oracle."""
    import torch
    cfg = q.Cfg(2048, 64, 4, 512)
    off = synth.zipf_logit_offset(8, 2, 64)
    dl = DevLayer(q, cfg, seed=8, layer=2, bits_of=lambda e: 2 if e % 3 == 0 else 4, offset=off)
    x = dev_tokens(8, 300, 6, 2048)
    out, idx, w = run_fused(q, dl, x, residual=True)
    for t in range(6):
        check(dl, out[t], idx[t], w[t], dl.oracle(host_x_f64(8, 300 + t, 2048), residual=True))
    ws = q.workspace(cfg, 6)
    ob = torch.empty((6, 2048), dtype=torch.float32, device="cuda")
    ib = torch.empty((6, 4), dtype=torch.int32, device="cuda")
    wb = torch.empty((6, 4), dtype=torch.float32, device="cuda")
    q.moe_layer_step(cfg, dl.layer_struct, x, ob, True, ib, wb, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    ob, ib, wb = ob.cpu().numpy(), ib.cpu().numpy(), wb.cpu().numpy()
    for t in range(6):
        check(dl, ob[t], ib[t], wb[t], dl.oracle(host_x_f64(8, 300 + t, 2048), residual=True))
