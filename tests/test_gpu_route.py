"""Router of the batched path (more than 4 tokens): clustered fp64 tiles.

Checked against the oracle's RMSNorm, router and top-K at shapes that leave
ragged expert and token tiles and give some CTAs of a cluster one column
chunk or none, and for run-to-run and batch-position independence (the
partial tiles are added in a fixed order).
"""
import numpy as np
import pytest

import oracle
import synth
from _util import assert_same_routing, dev_router, dev_tokens, host_x_f64

pytestmark = pytest.mark.gpu

EPS32 = float(np.float32(1e-6))


@pytest.fixture(scope="module")
def q(cuda):
    import quantized_expert_matvec_b200 as q
    return q


def _route(q, cfg, x, W, gamma=None, offset=None):
    import torch
    T, H, K = x.shape[0], cfg.hidden, cfg.top_k
    xn = torch.empty((T, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = q.workspace(cfg, T)
    q.moe_route(cfg, x, gamma, W, offset, xn, idx, w, ws)
    assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    return xn.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("H,E,K,T", [(320, 96, 6, 70), (64, 130, 3, 9), (2048, 512, 8, 129)])
def test_route_ragged_tiles_match_oracle(q, H, E, K, T):
    """Expert and token counts that are not multiples of the 64 x 64 tile;
    hidden 320 and 64 give 10 and 2 column chunks to the 8 CTAs of a cluster
    (several own none); gamma and a per-expert logit offset are applied."""
    import torch
    cfg = q.Cfg(H, E, K, 64)
    seed = 41
    W = dev_router(seed, 0, E, H)
    W_host = synth.host_router(seed, 0, E, H)
    rng = np.random.default_rng(7)
    gamma = (1.0 + 0.25 * rng.standard_normal(H)).astype(np.float32)
    offset = (0.5 * rng.standard_normal(E)).astype(np.float32)
    x = dev_tokens(seed, 100, T, H)
    xn, idx, w = _route(q, cfg, x, W, torch.tensor(gamma, device="cuda"), torch.tensor(offset, device="cuda"))
    for t in range(T):
        xh = host_x_f64(seed, 100 + t, H)
        xn_ref = oracle.rmsnorm(xh, gamma.astype(np.float64), EPS32)
        lg = oracle.router(W_host, xn_ref, offset)
        idx_ref, w_ref = oracle.topk(lg, K)
        assert np.max(np.abs(xn[t] - xn_ref)) <= 1e-6 * np.max(np.abs(xn_ref))
        assert_same_routing(idx[t], idx_ref, lg)
        assert np.max(np.abs(w[t] - w_ref)) <= 1e-6


def test_route_deterministic_and_independent_of_batch_position(q):
    """The same token routed twice in a batch of 256, and again at another
    position of a batch of 70, gets bit-identical experts and weights."""
    H, E, K = 4096, 512, 4
    cfg = q.Cfg(H, E, K, 1024)
    W = dev_router(3, 0, E, H)
    xa = dev_tokens(3, 0, 256, H, bf16=True)
    _, ia1, wa1 = _route(q, cfg, xa, W)
    _, ia2, wa2 = _route(q, cfg, xa, W)
    assert np.array_equal(ia1, ia2) and np.array_equal(wa1.view(np.uint32), wa2.view(np.uint32))
    xb = dev_tokens(3, 150, 70, H, bf16=True)  # tokens 150..219 at positions 0..69
    _, ib, wb = _route(q, cfg, xb, W)
    assert np.array_equal(ib, ia1[150:220])
    assert np.array_equal(wb.view(np.uint32), wa1[150:220].view(np.uint32))
