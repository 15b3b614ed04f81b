"""The seeded input generator: determinism, counter access, distributions.

The device fill is checked against the host fill bit for bit in
test_gpu_synth.py; here everything runs on the CPU.
"""
import math

import numpy as np
import pytest

import synth


def test_counter_access_matches_sequential():
    full = synth.host_fill(1000, synth.K_U32, 7, 1, 2, synth.T_GATE_WQ)
    part = synth.host_fill(100, synth.K_U32, 7, 1, 2, synth.T_GATE_WQ, i0=450)
    assert np.array_equal(full[450:550], part)


def test_streams_differ_and_repeat():
    a = synth.host_fill(64, synth.K_U32, 0, 0, 1, synth.T_GATE_WQ)
    b = synth.host_fill(64, synth.K_U32, 0, 0, 2, synth.T_GATE_WQ)
    c = synth.host_fill(64, synth.K_U32, 0, 0, 1, synth.T_UP_WQ)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    assert np.array_equal(a, synth.host_fill(64, synth.K_U32, 0, 0, 1, synth.T_GATE_WQ))


def test_splitmix64_reference_values():
    """splitmix64 from state 0: the first outputs of the published generator."""
    L = synth._host_lib()
    # draw(key=0, i) is splitmix64's output i from seed 0
    assert L.sy_host_draw(0, 0) == 0xE220A8397B1DCDAF
    assert L.sy_host_draw(0, 1) == 0x6E789E6AA1B965F4
    assert L.sy_host_draw(0, 2) == 0x06C45D188009454F


def test_series_ln_and_cos_accuracy():
    L = synth._host_lib()
    for u in np.concatenate([np.logspace(-16, -0.0001, 200), [0.5, 0.70710678, 0.9999999]]):
        assert abs(L.sy_host_ln(float(u)) - math.log(u)) <= 4e-16 * max(1.0, abs(math.log(u)))
    for v in np.linspace(1e-6, 1 - 1e-6, 501):
        assert abs(L.sy_host_cos2pi(float(v)) - math.cos(2 * math.pi * v)) <= 2e-15


def test_distributions():
    n = 200_000
    q = synth.host_fill(n, synth.K_U32, 0, 0, 0, synth.T_GATE_WQ)
    nib = ((q[:, None] >> (4 * np.arange(8, dtype=np.uint32))) & 15).ravel()
    counts = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(counts - 1 / 16) < 0.002)
    s = synth.host_fill(n, synth.K_BF16_UNIFORM, 0, 0, 0, synth.T_GATE_S, synth.SCALE_LO, synth.SCALE_HI)
    sv = (s.astype(np.uint32) << 16).view(np.float32)
    assert sv.min() >= 0.005 * (1 - 2 ** -8) and sv.max() <= 0.02 * (1 + 2 ** -8)
    assert abs(sv.mean() - 0.0125) < 1e-4
    z = synth.host_fill(n, synth.K_F32_NORMAL, 0, 0, 0, synth.T_X, 1.0)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert abs(((z - z.mean()) ** 4).mean() - 3.0) < 0.1
    b = synth.host_fill(n, synth.K_BF16_NORMAL, 0, 0, 0, synth.T_GATE_B, synth.BIAS_STD)
    bv = (b.astype(np.uint32) << 16).view(np.float32)
    assert abs(bv.std() - 0.01) < 2e-4


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1 + 2^-7: ties to even (1.0);
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: ties to even (1 + 2^-6).
    z = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    u = z.view(np.uint32)
    rne = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert list(rne) == [0x3F80, 0x3F82, 0x3F81]


def test_zipf_offset_hot_share():
    """The Zipf(1.1) offset with alpha 0.40 sends about 70% of top-4
    selections to the 128 most popular experts (simulated routing on random
    logits of the router's spread)."""
    off = synth.zipf_logit_offset(0, 3, 512)
    hot = synth.hot_set(0, 3, 512, 128)
    assert hot.sum() == 128
    rng = np.random.default_rng(0)
    hits = 0
    trials = 2000
    for _ in range(trials):
        lg = rng.normal(0, math.sqrt(4096) * 0.02, size=512) + off
        top = np.argsort(-lg, kind="stable")[:4]
        hits += hot[top].sum()
    share = hits / (4 * trials)
    assert 0.6 < share < 0.8, share


def test_host_expert_shapes():
    ex = synth.host_expert(0, 0, 0, 256, 64, 4)
    assert ex["gate_wq"].shape == (64, 32) and ex["gate_s"].shape == (64, 4)
    assert ex["down_wq"].shape == (256, 8) and ex["down_b"].shape == (256, 1)
    ex2 = synth.host_expert(0, 0, 0, 256, 64, 2)
    assert ex2["gate_wq"].shape == (64, 16) and ex2["down_wq"].shape == (256, 4)
