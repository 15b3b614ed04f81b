"""moe_layer_step_noalloc (the single-token step with the library's built-in
scratch) against moe_layer_step with a caller workspace, through the C ABI.

Kept in a file of its own so that it also runs after every other GPU test
(pytest collects this file last), where earlier launches have left state in
the library, and alone in a fresh process, where its first call does the
per-device set-up.
"""
import numpy as np
import pytest

import synth
from _util import TOL, dev_router, dev_tokens, fill_pool, normwise_err

pytestmark = pytest.mark.gpu


def _layer(q, cfg, seed, layer):
    """Device layer with mixed 4/2-bit experts, random gamma and a Zipf logit
    offset, from the seeded generator."""
    import torch
    E, H = cfg.n_experts, cfg.hidden
    bits_of = (lambda e: 4 if e % 3 else 2)
    pools = {b: q.ExpertPool(cfg, E, b) for b in (4, 2)}
    for p in pools.values():
        fill_pool(p, seed, layer)
    table = (q.Expert * E)()
    for e in range(E):
        table[e] = pools[bits_of(e)].host_table[e]
    keep = {
        "pools": pools,
        "table": torch.frombuffer(bytearray(bytes(table)), dtype=torch.uint8).cuda(),
        "W": dev_router(seed, layer, E, H),
        "gamma": torch.tensor(np.random.default_rng(seed).uniform(0.5, 1.5, H), dtype=torch.float32,
                              device="cuda"),
        "offset": torch.tensor(synth.zipf_logit_offset(seed, layer, E), device="cuda"),
    }
    keep["struct"] = q.Layer(keep["W"].data_ptr(), keep["offset"].data_ptr(), keep["gamma"].data_ptr(),
                             keep["table"].data_ptr())
    return keep


def _step(q, cfg, L, x, residual, noalloc, ws=None):
    import torch
    K, H = cfg.top_k, cfg.hidden
    out = torch.full((1, H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((1, K), -1, dtype=torch.int32, device="cuda")
    w = torch.full((1, K), float("nan"), dtype=torch.float32, device="cuda")
    if noalloc:
        status = torch.full((1,), -99, dtype=torch.int32, device="cuda")
        q.moe_layer_step_noalloc(cfg, L["struct"], x, out, residual, idx, w, status)
        torch.cuda.synchronize()
        assert int(status.item()) == q.QE_OK
    else:
        q.moe_layer_step(cfg, L["struct"], x, out, residual, idx, w, ws)
        assert q.qe_workspace_status(ws) == q.QE_OK, q.qe_last_error()
    return out.cpu().numpy()[0], idx.cpu().numpy()[0], w.cpu().numpy()[0]


def test_noalloc_matches_workspace_step_two_calls(cuda):
    """Two calls in a row on different tokens (the second with a residual and
    bf16 input) agree with the workspace entry point: same experts, same
    weights, outputs within the parity tolerance."""
    import quantized_expert_matvec_b200 as q
    cfg = q.Cfg(1024, 64, 4, 512)
    L = _layer(q, cfg, seed=21, layer=3)
    ws = q.workspace(cfg, 1)
    cases = [(dev_tokens(21, 0, 1, cfg.hidden), False),
             (dev_tokens(21, 1, 1, cfg.hidden, bf16=True), True)]
    for x, residual in cases:
        got = _step(q, cfg, L, x, residual, noalloc=True)
        ref = _step(q, cfg, L, x, residual, noalloc=False, ws=ws)
        assert list(got[1]) == list(ref[1]), (got[1], ref[1])
        assert np.allclose(got[2], ref[2], rtol=2e-6, atol=1e-7), (got[2], ref[2])
        assert np.all(np.isfinite(got[0]))
        err = normwise_err(got[0].astype(np.float64), ref[0].astype(np.float64))
        assert err <= TOL, err


def test_noalloc_rejects_oversized_scratch(cuda):
    """top_k * inter above the built-in limit fails on the host with a clear
    message, before anything is launched."""
    import torch
    import quantized_expert_matvec_b200 as q
    cfg = q.Cfg(256, 16, 8, 8192)
    dummy = torch.zeros(4096, dtype=torch.float32, device="cuda")
    layer = q.Layer(dummy.data_ptr(), None, None, dummy.data_ptr())
    x = torch.zeros((1, 256), dtype=torch.float32, device="cuda")
    out = torch.empty((1, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(q.QEError) as ei:
        q.moe_layer_step_noalloc(cfg, layer, x, out)
    assert ei.value.code == q.QE_ERR_INVALID_ARG
    assert "scratch limit" in str(ei.value)


def test_noalloc_at_the_scratch_limit(cuda):
    """top_k * inter exactly at the built-in limit (16 x 1024): the SwiGLU
    records fill their part of the scratch array; the result matches the
    workspace entry point."""
    import quantized_expert_matvec_b200 as q
    cfg = q.Cfg(256, 32, 16, 1024)
    L = _layer(q, cfg, seed=23, layer=0)
    ws = q.workspace(cfg, 1)
    x = dev_tokens(23, 5, 1, cfg.hidden)
    got = _step(q, cfg, L, x, True, noalloc=True)
    ref = _step(q, cfg, L, x, True, noalloc=False, ws=ws)
    assert list(got[1]) == list(ref[1])
    assert np.allclose(got[2], ref[2], rtol=2e-6, atol=1e-7)
    assert normwise_err(got[0].astype(np.float64), ref[0].astype(np.float64)) <= TOL


def test_noalloc_call_after_a_timed_out_call(cuda):
    """A call whose bounded waits give up (one CTA withholds its router
    logits, a 20 ms budget) reports QE_ERR_TIMEOUT in dev_status; the next
    call needs no re-initialisation and matches the workspace entry point."""
    import torch
    import quantized_expert_matvec_b200 as q
    cfg = q.Cfg(1024, 64, 4, 512)
    L = _layer(q, cfg, seed=22, layer=1)
    ws = q.workspace(cfg, 1)
    x = dev_tokens(22, 9, 1, cfg.hidden)
    out = torch.zeros((1, cfg.hidden), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    q.qe_set_wait_budget_ns(20_000_000)
    q.qe_test_skip_arrival(3)
    try:
        q.moe_layer_step_noalloc(cfg, L["struct"], x, out, False, None, None, status)
        torch.cuda.synchronize()
        assert int(status.item()) == q.QE_ERR_TIMEOUT
    finally:
        q.qe_test_skip_arrival(-1)
        q.qe_set_wait_budget_ns(200_000_000)
    got = _step(q, cfg, L, x, False, noalloc=True)
    ref = _step(q, cfg, L, x, False, noalloc=False, ws=ws)
    assert list(got[1]) == list(ref[1])
    assert normwise_err(got[0].astype(np.float64), ref[0].astype(np.float64)) <= TOL
