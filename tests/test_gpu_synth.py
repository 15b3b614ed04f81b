"""The device fill of the input generator writes exactly the host fill's
bits (so the oracle, fed from the host, sees the GPU's inputs)."""
import numpy as np
import pytest

import synth
from _util import dev_router, dev_tokens, fill_pool

pytestmark = pytest.mark.gpu


def test_device_fill_matches_host_fill(cuda):
    import torch
    import quantized_expert_matvec_b200 as q
    cfg = q.Cfg(256, 16, 2, 64)
    for bits in (4, 2):
        pool = q.ExpertPool(cfg, 16, bits)
        fill_pool(pool, seed=3, layer=2)
        torch.cuda.synchronize()
        raw = pool.buf.cpu().numpy()
        off0 = pool.base - pool.buf.data_ptr()
        for e in (0, 5, 15):
            ex = synth.host_expert(3, 2, e, 256, 64, bits)
            for seg, key in enumerate(["gate_wq", "up_wq", "down_wq", "gate_s", "gate_b", "up_s", "up_b",
                                       "down_s", "down_b"]):
                a = ex[key]
                start = off0 + e * pool.stride + pool.seg[seg]
                got = raw[start:start + a.nbytes].view(a.dtype).reshape(a.shape)
                assert np.array_equal(got, a), (bits, e, key)
    W = dev_router(7, 1, 32, 512).cpu().numpy()
    assert np.array_equal(W.view(np.uint32), synth.host_router(7, 1, 32, 512).view(np.uint32))
    x = dev_tokens(7, 10, 5, 512).cpu().numpy()
    assert np.array_equal(x.view(np.uint32), synth.host_tokens(7, 10, 5, 512).view(np.uint32))
    xb = dev_tokens(7, 10, 5, 512, bf16=True).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(xb, synth.host_tokens(7, 10, 5, 512, bf16=True))
