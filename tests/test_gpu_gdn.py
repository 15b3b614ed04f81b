"""GatedDeltaNet decode step on the GPU against the fp64 oracle.

The kernel (``gdn_decode_step``) computes in fp32; the oracle runs the same
step in fp64 from the same fp32 inputs.  Every element of the new state and of
the read-out is compared against a bound derived from the kernel's fp32
arithmetic (``step_bounds``), not a fixed tolerance:

* scal:  x1 = fl(alpha x), one rounding;
* recall: u = sum_j x1_j k_j with 4V sequential fmas per lane (V = dk/128
  rounded up) and a 5-level shuffle tree, so |error| <= gamma_(4V+5) A with
  A = sum_j |alpha x_j k_j|;
* c = fl(beta fl(v - u)): two roundings plus beta times the recall error;
* ger:  x2_j = fma(c, k_j, x1_j), one rounding plus |k_j| times the error of c
  and the error of x1;
* read-out: o = sum_j x2_j q_j, again gamma_(4V+5) relative to
  sum_j |x2_j q_j|, plus the state errors weighted by |q_j|.
Both bounds carry a factor 2 of slack.  Over several tokens the bound adds up
per row (with unit keys and beta in [0, 1] the step is non-expansive in each
row's 2-norm), which the recurrence test uses.

Shapes: the pages' layer (64 heads x 128 x 128), batched sequences (512
heads), and ragged ones (dk not a multiple of 128, dv not a multiple of the
rows per warp, a single row, the largest dk).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def q(cuda):
    import quantized_expert_matvec_b200 as q
    return q


def step_bounds(S0, tok, S1, o1):
    """Elementwise bounds on |kernel - exact| for one step from fp32 state S0
    (exact values S1, o1 from the oracle)."""
    S0 = S0.astype(np.float64)
    k = tok["k"].astype(np.float64)[:, None, :]
    qv = tok["q"].astype(np.float64)[:, None, :]
    al = tok["alpha"].astype(np.float64)[:, None, None]
    be = tok["beta"].astype(np.float64)[:, None, None]
    v = tok["v"].astype(np.float64)[:, :, None]
    dk = S0.shape[2]
    n = 4 * ((dk // 4 + 31) // 32) + 5
    ax = np.abs(al * S0)
    A = (ax * np.abs(k)).sum(axis=2, keepdims=True)
    tol_s = 2 * U32 * (np.abs(S1) + ax + np.abs(be) * np.abs(k) * (np.abs(v) + (n + 3) * A))
    tol_o = 2 * (n * U32 * (np.abs(S1) * np.abs(qv)).sum(axis=2) + (tol_s * np.abs(qv)).sum(axis=2))
    return tol_s, tol_o


def to_dev(tok, dev):
    import torch
    return {name: torch.from_numpy(np.ascontiguousarray(a)).to(dev) for name, a in tok.items()}


def gpu_step(q, S_dev, tok_dev, out=None):
    import torch
    nh, dv, _ = S_dev.shape
    if out is None:
        out = torch.empty((nh, dv), dtype=torch.float32, device=S_dev.device)
    q.gdn_decode_step(S_dev, tok_dev["q"], tok_dev["k"], tok_dev["v"], tok_dev["alpha"], tok_dev["beta"], out)
    return out


# one row per warp with the L2 prefetch (up to 64 warps' rows per SM), four
# rows per warp with it (up to four times that) and without it (beyond)
SHAPES = [(64, 128, 128), (128, 128, 128), (512, 128, 128), (100, 100, 130), (3, 36, 7), (5, 100, 130),
          (2, 512, 9), (1, 4, 1), (7, 260, 33), (4, 384, 64), (40, 512, 300)]


@pytest.mark.parametrize("nh,dk,dv", SHAPES, ids=[f"{a}h_dk{b}_dv{c}" for a, b, c in SHAPES])
def test_one_step_matches_oracle(q, cuda, nh, dk, dv):
    import torch
    S0 = synth.host_gdn_state(21, 0, nh, dk, dv)
    tok = synth.host_gdn_token(21, 0, 0, nh, dk, dv)
    S_dev = torch.from_numpy(S0.copy()).to(cuda)
    o_dev = gpu_step(q, S_dev, to_dev(tok, cuda))
    torch.cuda.synchronize()
    S1, o1 = oracle.gdn_step(S0, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
    tol_s, tol_o = step_bounds(S0, tok, S1, o1)
    dS = np.abs(S_dev.cpu().numpy().astype(np.float64) - S1)
    dO = np.abs(o_dev.cpu().numpy().astype(np.float64) - o1)
    assert np.all(dS <= tol_s), f"state: worst excess {np.max(dS - tol_s):.3g} at {np.unravel_index(np.argmax(dS - tol_s), dS.shape)}"
    assert np.all(dO <= tol_o), f"read-out: worst excess {np.max(dO - tol_o):.3g}"
    # the bound is not vacuous: it stays near fp32 resolution of the values
    assert np.max(tol_s) < 1e-4 * max(1.0, np.abs(S1).max())


def test_special_cases_exact_on_the_gpu(q, cuda):
    # beta = 0 and alpha = 1: the state is unchanged bit for bit and o = S q;
    # alpha = 0: the state becomes beta v k^T (one rounding of a product)
    import torch
    nh, dk, dv = 8, 128, 128
    S0 = synth.host_gdn_state(22, 0, nh, dk, dv)
    tok = synth.host_gdn_token(22, 0, 0, nh, dk, dv)
    t1 = dict(tok, alpha=np.ones(nh, np.float32), beta=np.zeros(nh, np.float32))
    S_dev = torch.from_numpy(S0.copy()).to(cuda)
    o_dev = gpu_step(q, S_dev, to_dev(t1, cuda))
    torch.cuda.synchronize()
    assert np.array_equal(S_dev.cpu().numpy(), S0)
    _, o1 = oracle.gdn_step(S0, t1["q"], t1["k"], t1["v"], t1["alpha"], t1["beta"])
    assert np.allclose(o_dev.cpu().numpy(), o1, rtol=0, atol=20 * U32 * np.abs(S0).sum(axis=2).max())
    t0 = dict(tok, alpha=np.zeros(nh, np.float32))
    S_dev = torch.from_numpy(S0.copy()).to(cuda)
    gpu_step(q, S_dev, to_dev(t0, cuda))
    torch.cuda.synchronize()
    # fma(c, k, 0) with c = fl(beta * fl(v - 0)) = fl(beta v): exactly fl(fl(beta v) k)
    c = (t0["beta"][:, None] * t0["v"]).astype(np.float32)
    expect = (c[:, :, None] * t0["k"][:, None, :]).astype(np.float32)
    assert np.array_equal(S_dev.cpu().numpy(), expect)


def test_recurrence_over_tokens(q, cuda):
    # 16 tokens launched back to back on one state with no synchronisation in
    # between (each launch may start while the previous one drains: it must
    # still read the state that one wrote), against the fp64 recurrence
    import torch
    nh, dk, dv, T = 64, 128, 128, 16
    S0 = synth.host_gdn_state(23, 3, nh, dk, dv)
    toks = [synth.host_gdn_token(23, 3, t, nh, dk, dv) for t in range(T)]
    S_dev = torch.from_numpy(S0.copy()).to(cuda)
    outs = torch.empty((T, nh, dv), dtype=torch.float32, device=cuda)
    devs = [to_dev(t, cuda) for t in toks]
    torch.cuda.synchronize()
    for t in range(T):
        gpu_step(q, S_dev, devs[t], outs[t])
    torch.cuda.synchronize()
    S = S0.astype(np.float64)
    acc = np.zeros((nh, dv))            # accumulated per-row 2-norm bound
    for t in range(T):
        Sn, o = oracle.gdn_step(S, toks[t]["q"], toks[t]["k"], toks[t]["v"], toks[t]["alpha"], toks[t]["beta"])
        tol_s, tol_o = step_bounds(S.astype(np.float32), toks[t], Sn, o)
        # the read-out sees the state error so far (times |q| = 1) plus its own
        got_o = outs[t].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got_o - o) <= 1.01 * (acc + np.sqrt((tol_s ** 2).sum(axis=2))) + tol_o), t
        acc = 1.01 * acc + np.sqrt((tol_s ** 2).sum(axis=2))
        S = Sn
    err_rows = np.sqrt(((S_dev.cpu().numpy().astype(np.float64) - S) ** 2).sum(axis=2))
    assert np.all(err_rows <= acc)


def test_graph_replay_is_bit_identical_to_eager(q, cuda):
    import torch
    nh, dk, dv, T = 64, 128, 128, 4
    S0 = synth.host_gdn_state(24, 0, nh, dk, dv)
    devs = [to_dev(synth.host_gdn_token(24, 0, t, nh, dk, dv), cuda) for t in range(T)]
    S_e = torch.from_numpy(S0.copy()).to(cuda)
    o_e = torch.empty((T, nh, dv), dtype=torch.float32, device=cuda)
    for t in range(T):
        gpu_step(q, S_e, devs[t], o_e[t])
    S_g = torch.from_numpy(S0.copy()).to(cuda)
    o_g = torch.empty_like(o_e)
    s = torch.cuda.Stream(device=cuda)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for t in range(T):
            gpu_step(q, S_g, devs[t], o_g[t])
    S_g.copy_(torch.from_numpy(S0))       # capture ran nothing; start from S0
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(S_g, S_e) and torch.equal(o_g, o_e)
    del g


def test_zero_heads_is_a_no_op(q, cuda):
    import torch
    e = torch.empty((0, 8, 16), dtype=torch.float32, device=cuda)
    z = torch.empty(0, dtype=torch.float32, device=cuda)
    q.gdn_decode_step(e, z, z, z, z, z, z)
    torch.cuda.synchronize()
