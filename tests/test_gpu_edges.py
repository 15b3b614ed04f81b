"""Edge cases of the layer step, each run through the three ways a token can
take (the single-token kernel, the batched path, the two-tier store) and
compared with the fp64 oracle: routing bit for bit with no token excused
as a near-tie, outputs within the normwise tolerance.

The cases:
* exact logit ties: router weights all zero, so every logit is its expert's
  offset, drawn from a few repeated values (and all zero: no offset at all);
  equal logits go to the lower expert index, at every level of the top-K;
* all-zero and all-ones quantised words (q = 0 and q = 2^bits - 1 in every
  field), 4-bit and 2-bit;
* one-hot activations;
* activations and gamma at the ends of the fp32 range, and one token whose
  entries span 60 decades;
* one selected expert whose SwiGLU output is up to a million times the
  others', with a router weight 1e4 times smaller, so that its contribution
  to the output is of the same size as theirs.

Expert tensors are the seeded generator's, then edited on the host; the
device copies are written from those host arrays, so the oracle and the
library see the same bytes.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from _util import TOL, assert_same_routing, normwise_err

pytestmark = pytest.mark.gpu

EPS32 = float(np.float32(1e-6))
# qe_pool_table's segment order
SEG_KEYS = ["gate_wq", "up_wq", "down_wq", "gate_s", "gate_b", "up_s", "up_b", "down_s", "down_b"]


@pytest.fixture(scope="module")
def q(cuda):
    import quantized_expert_matvec_b200 as q
    return q


def _expert_bytes(ex):
    return [np.ascontiguousarray(ex[k]).view(np.uint8).reshape(-1) for k in SEG_KEYS]


class ArbLayer:
    """A layer from arbitrary host tensors: experts[e] in the host_expert
    layout at bits_of(e), router W [E, H] fp32, optional offset [E] and
    gamma [H].  Device copies for the resident paths (every expert in HBM)
    and, for the two-tier path, hot experts (bits 4) in HBM and cold ones
    (bits 2) in pinned host memory."""

    def __init__(self, q, cfg, experts, bits_of, W, offset=None, gamma=None):
        import torch
        self.q, self.cfg, self.experts, self.bits_of = q, cfg, experts, bits_of
        E = cfg.n_experts
        self.W = np.ascontiguousarray(W, np.float32)
        self.offset = None if offset is None else np.ascontiguousarray(offset, np.float32)
        self.gamma = None if gamma is None else np.ascontiguousarray(gamma, np.float32)
        self.keep = []
        self.W_dev = torch.from_numpy(self.W).cuda()
        self.off_dev = torch.from_numpy(self.offset).cuda() if offset is not None else None
        self.gamma_dev = torch.from_numpy(self.gamma).cuda() if gamma is not None else None
        # every expert resident, one pool per bit width
        table = (q.Expert * E)()
        for b in sorted({bits_of(e) for e in range(E)}):
            ids = [e for e in range(E) if bits_of(e) == b]
            pool = q.ExpertPool(cfg, len(ids), b)
            host = np.zeros(pool.stride * len(ids), np.uint8)
            for m, e in enumerate(ids):
                for s, arr in enumerate(_expert_bytes(experts[e])):
                    o = m * pool.stride + pool.seg[s]
                    host[o:o + arr.size] = arr
            off = pool.base - pool.buf.data_ptr()
            pool.buf[off:off + host.size].copy_(torch.from_numpy(host))
            for m, e in enumerate(ids):
                table[e] = pool.host_table[m]
            self.keep.append(pool)
        self.table = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).cuda()
        self.layer = q.Layer(self.W_dev.data_ptr(), self.off_dev.data_ptr() if offset is not None else None,
                             self.gamma_dev.data_ptr() if gamma is not None else None, self.table.data_ptr())
        torch.cuda.synchronize()

    def tiered(self):
        """(tier, layer struct) with 4-bit experts in HBM and 2-bit experts
        in pinned host memory behind a slot cache."""
        import torch
        q, cfg, E = self.q, self.cfg, self.cfg.n_experts
        hot = [e for e in range(E) if self.bits_of(e) == 4]
        cold = [e for e in range(E) if self.bits_of(e) == 2]
        table = (q.Expert * E)()
        if hot:
            pool = q.ExpertPool(cfg, len(hot), 4)
            host = np.zeros(pool.stride * len(hot), np.uint8)
            for m, e in enumerate(hot):
                for s, arr in enumerate(_expert_bytes(self.experts[e])):
                    o = m * pool.stride + pool.seg[s]
                    host[o:o + arr.size] = arr
            off = pool.base - pool.buf.data_ptr()
            pool.buf[off:off + host.size].copy_(torch.from_numpy(host))
            for m, e in enumerate(hot):
                table[e] = pool.host_table[m]
            self.keep.append(pool)
        cold_b = q.qe_expert_bytes(cfg, 2)
        hbuf = torch.empty(cold_b * max(len(cold), 1) + 256, dtype=torch.uint8).pin_memory()
        base = (hbuf.data_ptr() + 255) // 256 * 256
        _, seg = q.qe_pool_table(cfg, base, 2, 1)
        ptrs = [None] * E
        for j, e in enumerate(cold):
            for s, arr in enumerate(_expert_bytes(self.experts[e])):
                ctypes.memmove(base + j * cold_b + seg[s], arr.ctypes.data, arr.size)
            ptrs[e] = base + j * cold_b
        dtab = torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).cuda()
        lw = q.Layer(self.W_dev.data_ptr(), self.off_dev.data_ptr() if self.offset is not None else None,
                     self.gamma_dev.data_ptr() if self.gamma is not None else None, dtab.data_ptr())
        tier = q.Tier(cfg, [ptrs], 2, 8 * cold_b, max_tokens=8)
        self.keep += [hbuf, dtab]
        return tier, lw

    def oracle(self, x64, residual=False):
        return oracle.layer_step(x64, self.W.astype(np.float64), lambda e: self.experts[e], self.bits_of,
                                 self.cfg.top_k, eps=EPS32,
                                 gamma=None if self.gamma is None else self.gamma.astype(np.float64),
                                 offset=None if self.offset is None else self.offset.astype(np.float64),
                                 residual=residual, nthreads=8)


def run_paths(q, al, x_host, residual=False, paths=("fused", "batched", "tier")):
    """Run every token of x_host [T, H] (fp32) through each path; returns
    {path: (out [T,H], idx [T,K], w [T,K])}."""
    import torch
    cfg = al.cfg
    T, H, K = x_host.shape[0], cfg.hidden, cfg.top_k
    x = torch.from_numpy(np.ascontiguousarray(x_host, np.float32)).cuda()
    res = {}
    for path in paths:
        out = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, K), float("nan"), dtype=torch.float32, device="cuda")
        if path == "fused":
            ws = q.workspace(cfg, 1)
            for t in range(T):
                q.moe_layer_step(cfg, al.layer, x[t:t + 1], out[t:t + 1], residual, idx[t:t + 1], w[t:t + 1], ws)
        elif path == "batched":
            ws = q.workspace(cfg, T)
            q.moe_layer_step(cfg, al.layer, x, out, residual, idx, w, ws)
        else:
            tier, lw = al.tiered()
            ws = q.workspace(cfg, T)
            for t in range(T):
                tier.layer_step(0, lw, x[t:t + 1], out[t:t + 1], residual, idx[t:t + 1], w[t:t + 1], ws)
        assert q.qe_workspace_status(ws) == q.QE_OK, (path, q.qe_last_error())
        res[path] = (out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())
        if path == "tier":
            tier.close()
    return res


def check_all(al, x_host, res, residual=False, tol=TOL):
    """Every path, every token: routing bit for bit (no near-tie excused),
    weights to fp32 rounding, output within the normwise tolerance."""
    n = 0
    for t in range(x_host.shape[0]):
        ref = al.oracle(x_host[t].astype(np.float64), residual)
        for path, (out, idx, w) in res.items():
            assert_same_routing(idx[t], ref["idx"], ref["logits"])
            assert np.allclose(w[t], ref["w"], rtol=2e-6, atol=1e-7), (path, t, w[t], ref["w"])
            err = normwise_err(out[t], ref["out"])
            assert err <= tol, (path, t, err)
            n += 1
    return n


def gen_experts(cfg, seed, bits_of):
    return {e: synth.host_expert(seed, 0, e, cfg.hidden, cfg.inter, bits_of(e)) for e in range(cfg.n_experts)}


def gen_x(seed, T, H):
    return np.stack([synth.host_tokens(seed, t, 1, H)[0] for t in range(T)]).astype(np.float32)


def mixed_bits(e):
    return 4 if e % 2 == 0 else 2


# ------------------------------------------------------------ exact ties

@pytest.mark.parametrize("shape", [(512, 64, 4, 128), (256, 512, 4, 64)], ids=["64experts", "512experts"])
def test_exact_logit_ties_lower_index_wins(q, shape):
    """Router weights zero: every logit is its expert's offset, taken from
    five values, so many experts tie exactly; each path must pick the
    lowest indices among the tied largest (and equal weights)."""
    cfg = q.Cfg(*shape)
    E, H = cfg.n_experts, cfg.hidden
    off = ((np.arange(E) * 7) % 5).astype(np.float32) * 0.5
    al = ArbLayer(q, cfg, gen_experts(cfg, 11, mixed_bits), mixed_bits, np.zeros((E, H), np.float32), offset=off)
    x = gen_x(11, 5, H)
    res = run_paths(q, al, x)
    assert check_all(al, x, res) == 15
    want = [e for e in range(E) if off[e] == off.max()][:cfg.top_k]
    for _, (_, idx, w) in res.items():
        assert (idx == np.array(want)).all()
        assert np.all(w == np.float32(1.0 / cfg.top_k))


def test_all_logits_zero_takes_first_experts(q):
    """No offset and zero router weights (and one all-zero token): every
    logit is 0; the first K experts are taken, in index order."""
    cfg = q.Cfg(256, 512, 4, 64)
    E, H = cfg.n_experts, cfg.hidden
    al = ArbLayer(q, cfg, gen_experts(cfg, 12, mixed_bits), mixed_bits, np.zeros((E, H), np.float32))
    x = gen_x(12, 3, H)
    x[1] = 0.0
    res = run_paths(q, al, x)
    check_all(al, x, res)
    for _, (_, idx, _) in res.items():
        assert (idx == np.arange(cfg.top_k)).all()


# ------------------------------------------------------ extreme q words

@pytest.mark.parametrize("fill", ["zeros", "ones", "alternate"])
def test_extreme_quantised_words(q, fill):
    """Every quantised field 0 (w = bias), every field 2^bits - 1 (w = the
    largest level times the scale plus the bias), or the two alternating by
    expert; 4-bit and 2-bit experts."""
    cfg = q.Cfg(512, 64, 4, 128)
    ex = gen_experts(cfg, 13, mixed_bits)
    for e, d in ex.items():
        v = {"zeros": 0, "ones": 0xFFFFFFFF, "alternate": 0xFFFFFFFF if (e // 2) % 2 else 0}[fill]
        for m in ("gate", "up", "down"):
            d[m + "_wq"] = np.full_like(d[m + "_wq"], v)
    W = synth.host_router(13, 0, cfg.n_experts, cfg.hidden)
    al = ArbLayer(q, cfg, ex, mixed_bits, W)
    x = gen_x(13, 4, cfg.hidden)
    res = run_paths(q, al, x)
    assert check_all(al, x, res) == 12


# ------------------------------------------------------ activation edges

def test_one_hot_activations(q):
    """x = c e_j at the first, a middle and the last column (after the
    RMSNorm: sqrt(H) at j, zeros elsewhere)."""
    cfg = q.Cfg(512, 64, 4, 128)
    H = cfg.hidden
    W = synth.host_router(14, 0, cfg.n_experts, H)
    al = ArbLayer(q, cfg, gen_experts(cfg, 14, mixed_bits), mixed_bits, W)
    x = np.zeros((3, H), np.float32)
    for t, j in enumerate((0, H // 2 + 1, H - 1)):
        x[t, j] = 3.0 if t != 1 else -7.5
    res = run_paths(q, al, x, residual=True)
    assert check_all(al, x, res, residual=True) == 9


@pytest.mark.parametrize("case", ["x_1e30", "x_1e-15", "span_60_decades", "gamma_1e-12", "gamma_1e8"])
def test_range_extremes(q, case):
    """Activations near the top of the fp32 range (the RMSNorm sum of
    squares is taken in fp64) and tiny ones (eps then dominates the RMSNorm
    and xn is about 1e-12), a token whose entries run from 1e-30 to 1e30,
    and gamma tiny or large (the fixed-point exponents of xn and of h follow
    the vector's own magnitude).  Each case keeps the layer's output within
    fp32's normal range: the SwiGLU is quadratic in xn, so xn near 1e-27
    would give outputs near 1e-53, which no fp32 result can hold."""
    cfg = q.Cfg(512, 64, 4, 128)
    H = cfg.hidden
    rng = np.random.default_rng(15)
    x = gen_x(15, 3, H)
    gamma = None
    if case == "x_1e30":
        x = x * np.float32(1e30)
    elif case == "x_1e-15":
        x = x * np.float32(1e-15)
    elif case == "span_60_decades":
        x = (np.sign(x) * 10.0 ** rng.uniform(-30, 30, x.shape)).astype(np.float32)
    elif case == "gamma_1e-12":
        gamma = (rng.uniform(0.5, 1.5, H) * 1e-12).astype(np.float32)
    else:
        gamma = (rng.uniform(0.5, 1.5, H) * 1e8).astype(np.float32)
    W = synth.host_router(15, 0, cfg.n_experts, H)
    al = ArbLayer(q, cfg, gen_experts(cfg, 15, mixed_bits), mixed_bits, W, gamma=gamma)
    res = run_paths(q, al, x)
    assert check_all(al, x, res) == 9


# ------------------------------------------------ one expert much larger

def test_one_expert_with_a_much_larger_h(q):
    """Experts 0..2 at logit 0, expert 3 at -ln(1e4), the rest at -100 (zero
    router weights): expert 3 takes a weight 1e4 times smaller.  Its gate and
    up scales are 1000 times larger, so its SwiGLU output is up to 1e6 times
    the others' (silu keeps the large positive gate values and nearly zeroes
    the large negative ones), and its weighted contribution to the output is
    of the others' size; an error in either shows in the output."""
    cfg = q.Cfg(512, 64, 4, 128)
    E, H = cfg.n_experts, cfg.hidden
    ex = gen_experts(cfg, 16, mixed_bits)
    for m in ("gate", "up"):
        s = oracle.bf16_value(ex[3][m + "_s"]).astype(np.float32) * np.float32(1000.0)
        ex[3][m + "_s"] = (s.view(np.uint32) >> 16).astype(np.uint16)  # truncated back to bf16
    off = np.full(E, -100.0, np.float32)
    off[:3] = 0.0
    off[3] = -np.log(1e4)
    al = ArbLayer(q, cfg, ex, mixed_bits, np.zeros((E, H), np.float32), offset=off)
    x = gen_x(16, 4, H)
    res = run_paths(q, al, x)
    assert check_all(al, x, res) == 12
    ref = al.oracle(x[0].astype(np.float64))
    contrib = np.abs(ref["w"][:, None] * ref["y"]).max(axis=1)
    assert contrib[3] > 0.05 * contrib[:3].max() and contrib[3] < 20 * contrib[:3].max()
