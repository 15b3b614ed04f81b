"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against something fixed independently of its own
code: a closed form, an exact special case, brute force on tiny inputs with an
independent unpacking route, a library routine, an invariant, or the sizes the
Flash-MoE pages print.  A dropped term, a wrong sign, a swapped index or a
transposed operand anywhere in the oracle breaks at least one of them.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def pack_rows(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack a [rows, cols] matrix of q values with the layout convention under
    test: field j of a uint32 word holds column (word*32/bits + j) at bits
    [bits*j, bits*j + bits)."""
    rows, cols = q.shape
    per = 32 // bits
    out = np.zeros((rows, cols // per), np.uint64)
    for j in range(per):
        out |= q[:, j::per].astype(np.uint64) << np.uint64(bits * j)
    return out.astype(np.uint32)


def unpack_bytes(wq: np.ndarray, cols: int, bits: int) -> np.ndarray:
    """Independent unpack through numpy's bit unpacking of the little-endian
    byte stream (no shifts or masks on words)."""
    rows = wq.shape[0]
    b = np.ascontiguousarray(wq.astype("<u4")).view(np.uint8).reshape(rows, -1)
    bitstream = np.unpackbits(b, axis=1, bitorder="little").reshape(rows, cols, bits)
    weights = (1 << np.arange(bits)).astype(np.int64)
    return (bitstream.astype(np.int64) * weights).sum(axis=2)


def rand_sb(rng, rows, cols):
    s = rng.uniform(0.005, 0.02, size=(rows, cols // 64)).astype(np.float32)
    b = rng.normal(0, 0.01, size=(rows, cols // 64)).astype(np.float32)
    to_bf16 = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)  # truncation is fine for a fixture
    return to_bf16(s), to_bf16(b)


# ---------------------------------------------------------------- unpack / dequant

@pytest.mark.parametrize("bits", [4, 2])
def test_one_hot_column_recovers_q_scale_bias(bits):
    """x = e_c makes y_r = q_rc * s_r,g(c) + b_r,g(c) exactly: pins the field
    order inside a word, the word order along a row and the group index."""
    rng = np.random.default_rng(1)
    rows, cols = 5, 192
    q = rng.integers(0, 1 << bits, size=(rows, cols))
    s, b = rand_sb(rng, rows, cols)
    wq = pack_rows(q, bits)
    sv, bv = oracle.bf16_value(s), oracle.bf16_value(b)
    for c in range(cols):
        x = np.zeros(cols)
        x[c] = 1.0
        y = oracle.qmatvec(wq, s, b, bits, x)
        expect = q[:, c] * sv[:, c // 64] + bv[:, c // 64]
        assert np.array_equal(y, expect), (c, y, expect)


@pytest.mark.parametrize("bits", [4, 2])
def test_all_levels_round_trip(bits):
    """Every group holds every q level; dequant recovers q exactly."""
    levels = 1 << bits
    rows, cols = 3, 128
    q = np.tile(np.arange(cols) % levels, (rows, 1))
    q[1] = q[1][::-1]
    rng = np.random.default_rng(2)
    s, b = rand_sb(rng, rows, cols)
    wq = pack_rows(q, bits)
    for r in range(rows):
        for c in range(cols):
            assert oracle.q_value(wq, cols, bits, r, c) == q[r, c]
            w = oracle.dequant(wq, s, b, bits, cols, r, c)
            g = c // 64
            sv, bv = oracle.bf16_value(s[r, g]), oracle.bf16_value(b[r, g])
            assert (w - bv) / sv == q[r, c]


def test_bf16_values():
    """bf16 decoding against fp32 values known exactly."""
    cases = {0x3F80: 1.0, 0xBF80: -1.0, 0x4000: 2.0, 0x3C00: 2.0 ** -7, 0x3F81: 1.0 + 2.0 ** -7, 0x0000: 0.0}
    for bits16, v in cases.items():
        assert oracle.bf16_value(np.uint16(bits16)) == v


@pytest.mark.parametrize("bits", [4, 2])
def test_all_zero_q_closed_form(bits):
    """q = 0 everywhere: y_r = sum_g b_rg * sum_{c in g} x_c."""
    rng = np.random.default_rng(3)
    rows, cols = 7, 256
    wq = np.zeros((rows, cols * bits // 32), np.uint32)
    s, b = rand_sb(rng, rows, cols)
    x = rng.normal(size=cols)
    y = oracle.qmatvec(wq, s, b, bits, x)
    gx = x.reshape(-1, 64).sum(axis=1)
    expect = oracle.bf16_value(b) @ gx
    assert np.allclose(y, expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("shape", [(1, 64), (9, 128), (64, 128), (33, 320)])
def test_matvec_vs_dense_brute_force(bits, shape):
    """Explicitly dequantised dense fp64 matrix (independent byte-level
    unpack) times x with numpy's matmul equals the oracle to 1e-12."""
    rows, cols = shape
    rng = np.random.default_rng(rows * 1000 + cols + bits)
    q = rng.integers(0, 1 << bits, size=(rows, cols))
    s, b = rand_sb(rng, rows, cols)
    wq = pack_rows(q, bits)
    assert np.array_equal(unpack_bytes(wq, cols, bits), q)
    dense = unpack_bytes(wq, cols, bits) * np.repeat(oracle.bf16_value(s), 64, axis=1) \
        + np.repeat(oracle.bf16_value(b), 64, axis=1)
    x = rng.normal(size=cols)
    y = oracle.qmatvec(wq, s, b, bits, x)
    ref = dense @ x
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("bits", [4, 2])
def test_fma_rewrite_identity(bits):
    """The pages' FMA rewrite fma(q, s*x, b*x) and (q*s+b)*x agree, and both
    equal the group-factored form s*sum(q x) + b*sum(x)."""
    rng = np.random.default_rng(4)
    rows, cols = 16, 512
    q = rng.integers(0, 1 << bits, size=(rows, cols))
    s, b = rand_sb(rng, rows, cols)
    wq = pack_rows(q, bits)
    x = rng.normal(size=cols)
    y1 = oracle.qmatvec(wq, s, b, bits, x)
    y2 = oracle.qmatvec_fma_form(wq, s, b, bits, x)
    qx = (q * x).reshape(rows, -1, 64).sum(axis=2)
    gx = x.reshape(-1, 64).sum(axis=1)
    y3 = (oracle.bf16_value(s) * qx).sum(axis=1) + oracle.bf16_value(b) @ gx
    scale = np.max(np.abs(y1))
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * scale
    assert np.max(np.abs(y1 - y3)) <= 1e-12 * scale


def test_matvec_on_synthetic_expert_tensors():
    """The generator's expert tensors, dequantised by the independent byte
    unpack, give the same product as the oracle (C0-sized gate matrix)."""
    ex = synth.host_expert(0, 0, 3, 256, 64, 4)
    x = np.random.default_rng(5).normal(size=256)
    dense = unpack_bytes(ex["gate_wq"], 256, 4) * np.repeat(oracle.bf16_value(ex["gate_s"]), 64, axis=1) \
        + np.repeat(oracle.bf16_value(ex["gate_b"]), 64, axis=1)
    y = oracle.qmatvec(ex["gate_wq"], ex["gate_s"], ex["gate_b"], 4, x)
    assert np.max(np.abs(y - dense @ x)) <= 1e-12 * np.max(np.abs(y))


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_unit_mean_square():
    x = np.random.default_rng(6).normal(size=4096) * 3.7
    xn = oracle.rmsnorm(x, None, 0.0)
    assert abs(np.mean(xn * xn) - 1.0) < 1e-12
    # with eps: mean(xn^2) = ms / (ms + eps), closed form
    eps = 1e-2
    xn = oracle.rmsnorm(x, None, eps)
    ms = np.mean(x * x)
    assert abs(np.mean(xn * xn) - ms / (ms + eps)) < 1e-12


def test_rmsnorm_constant_and_gamma():
    c, eps = 0.3, 1e-6
    xn = oracle.rmsnorm(np.full(64, c), None, eps)
    assert np.allclose(xn, c / math.sqrt(c * c + eps), rtol=1e-15)
    x = np.random.default_rng(7).normal(size=128)
    g = np.random.default_rng(8).uniform(0.5, 2.0, size=128)
    assert np.allclose(oracle.rmsnorm(x, g, eps), oracle.rmsnorm(x, None, eps) * g, rtol=1e-14)
    # scale invariance with eps = 0
    assert np.allclose(oracle.rmsnorm(5.0 * x, None, 0.0), oracle.rmsnorm(x, None, 0.0), rtol=1e-14)


# ---------------------------------------------------------------- router / top-K

def test_router_is_matvec():
    rng = np.random.default_rng(9)
    W = rng.normal(0, 0.02, size=(16, 256)).astype(np.float32)
    xn = rng.normal(size=256)
    off = rng.normal(size=16).astype(np.float32)
    ref = W.astype(np.float64) @ xn + off.astype(np.float64)
    assert np.allclose(oracle.router(W, xn, off), ref, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("E,K", [(16, 2), (512, 4), (64, 64), (5, 1)])
def test_topk_brute_force(E, K):
    rng = np.random.default_rng(E + K)
    lg = rng.normal(size=E)
    idx, w = oracle.topk(lg, K)
    brute = sorted(range(E), key=lambda e: (-lg[e], e))[:K]
    assert list(idx) == brute
    assert abs(w.sum() - 1.0) < 1e-15
    p = oracle.softmax(lg)
    assert np.allclose(w, p[idx] / p[idx].sum(), rtol=1e-13)


def test_topk_ties_lower_index_wins():
    lg = np.array([0.5, 2.0, 1.0, 2.0, 1.0, 2.0, -1.0])
    idx, w = oracle.topk(lg, 4)
    assert list(idx) == [1, 3, 5, 2]
    assert np.allclose(w[:3], w[0]) and w[3] < w[0]


def test_softmax_known_values():
    p = oracle.softmax(np.array([0.0, math.log(3.0)]))
    assert np.allclose(p, [0.25, 0.75], rtol=1e-15)


# ---------------------------------------------------------------- SwiGLU

def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    for v in [0.1, 1.0, 3.5, 20.0]:
        assert abs((oracle.silu(v) - oracle.silu(-v)) - v) <= 4e-16 * max(1.0, v)


def test_silu_high_precision():
    getcontext().prec = 50
    for v in [-7.25, -1.0, -0.3, 0.01, 0.7, 2.0, 9.0]:
        exact = Decimal(v) / (1 + (-Decimal(v)).exp())
        assert abs(Decimal(oracle.silu(v)) - exact) <= Decimal(4e-16) * abs(exact)


def test_swiglu_is_silu_gate_times_up():
    g = np.array([-2.0, 0.0, 1.5])
    u = np.array([3.0, 5.0, -2.0])
    h = oracle.swiglu(g, u)
    assert h[1] == 0.0
    assert np.allclose(h, g / (1 + np.exp(-g)) * u, rtol=1e-15)


# ---------------------------------------------------------------- expert / layer

def _tiny_layer(seed=0, H=256, E=16, I=64, bits=4):
    experts = {e: synth.host_expert(seed, 0, e, H, I, bits) for e in range(E)}
    W = synth.host_router(seed, 0, E, H)
    x = synth.host_tokens(seed, 0, 1, H)[0].astype(np.float64)
    return experts, W, x


def test_expert_ffn_composition_brute_force():
    """Expert FFN equals dense brute force: Wd (silu(Wg xn) * (Wu xn))."""
    ex = synth.host_expert(0, 0, 1, 256, 64, 4)
    xn = oracle.rmsnorm(np.random.default_rng(10).normal(size=256))

    def dense(m, rows, cols):
        return unpack_bytes(ex[m + "_wq"], cols, 4) * np.repeat(oracle.bf16_value(ex[m + "_s"]), 64, axis=1) \
            + np.repeat(oracle.bf16_value(ex[m + "_b"]), 64, axis=1)

    g = dense("gate", 64, 256) @ xn
    u = dense("up", 64, 256) @ xn
    h = g / (1.0 + np.exp(-g)) * u
    ref = dense("down", 256, 64) @ h
    y = oracle.expert_ffn(ex, 4, xn)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_one_hot_router_reproduces_single_expert():
    """An offset of +1000 on expert e makes its weight exactly 1 and every
    other weight exactly 0, so the layer output is expert e's output, bit for
    bit."""
    experts, W, x = _tiny_layer()
    for e in (0, 7, 15):
        off = np.zeros(16, np.float32)
        off[e] = 1000.0
        r = oracle.layer_step(x, W, lambda i: experts[i], lambda i: 4, K=2, offset=off)
        assert r["idx"][0] == e and r["w"][0] == 1.0 and r["w"][1] == 0.0
        ye = oracle.expert_ffn(experts[e], 4, r["xn"])
        assert np.array_equal(r["out"], ye)


def test_k_equals_e_is_full_softmax_mixture():
    experts, W, x = _tiny_layer(E=8)
    r = oracle.layer_step(x, W[:8], lambda i: experts[i], lambda i: 4, K=8)
    p = oracle.softmax(r["logits"])
    ys = np.stack([oracle.expert_ffn(experts[e], 4, r["xn"]) for e in range(8)])
    ref = (p[:, None] * ys).sum(axis=0)
    assert np.max(np.abs(r["out"] - ref)) <= 1e-13 * np.max(np.abs(ref))


def test_residual_with_zero_experts_is_identity():
    """All-zero weights (q = 0, bias = 0) make every expert output 0, so the
    residual layer returns x."""
    H, I = 128, 64
    zero = {}
    for m, (rows, cols) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items():
        zero[m + "_wq"] = np.zeros((rows, cols // 8), np.uint32)
        zero[m + "_s"] = np.full((rows, cols // 64), 0x3F80, np.uint16)
        zero[m + "_b"] = np.zeros((rows, cols // 64), np.uint16)
    W = np.random.default_rng(11).normal(size=(4, H)).astype(np.float32)
    x = np.random.default_rng(12).normal(size=H)
    r = oracle.layer_step(x, W, lambda i: zero, lambda i: 4, K=2, residual=True)
    assert np.array_equal(r["out"], x)


def test_combine_weighted_sum():
    y = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0]])
    w = np.array([0.5, 0.25, 0.25])
    assert np.array_equal(oracle.combine(y, w), [28.0, 56.0])
    assert np.array_equal(oracle.combine(y, w, np.array([1.0, -1.0])), [29.0, 55.0])


# ---------------------------------------------------------------- sizes on the pages

def expert_bytes(H, I, bits, group=64, sb_bytes=2):
    n = 3 * H * I
    return n * bits // 8 + 2 * sb_bytes * n // group


def test_expert_size_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "page_sizes.json")))
    b4 = expert_bytes(4096, 1024, 4)
    assert b4 == 7_077_888
    assert b4 / 2 ** 20 == g["expert_mib_4bit"]
    assert g["top_k"] * b4 / 2 ** 20 == g["token_layer_mb_4bit"]
    assert g["layers"] * g["top_k"] * b4 / 2 ** 20 / 1000 == pytest.approx(g["experts_gb_per_token_4bit"], rel=1e-9)
    total4 = g["layers"] * g["n_experts"] * b4 / 2 ** 30 + g["non_expert_gb"]
    total2 = g["layers"] * g["n_experts"] * expert_bytes(4096, 1024, 2) / 2 ** 30 + g["non_expert_gb"]
    assert total4 == pytest.approx(g["model_gb_4bit"], rel=0.02)
    assert total2 == pytest.approx(g["model_gb_2bit"], rel=0.02)
    # a 32-bit scale/bias or group 32 would break the 6.75 MiB figure
    assert expert_bytes(4096, 1024, 4, sb_bytes=4) / 2 ** 20 != g["expert_mib_4bit"]
    assert expert_bytes(4096, 1024, 4, group=32) / 2 ** 20 != g["expert_mib_4bit"]
