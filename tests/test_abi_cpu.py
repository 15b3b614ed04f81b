"""The C-ABI library without a GPU: it loads, exports every symbol that
include/qexpert.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^QE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M))
    return names


@pytest.fixture(scope="module")
def q():
    import quantized_expert_matvec_b200 as q
    return q


def test_library_exports_every_declared_symbol(q):
    names = declared_symbols()
    assert {"moe_route", "moe_expert_ffn_q4", "moe_expert_ffn_q2", "moe_combine", "moe_layer_step"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", q.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = names - exported
    assert not missing, missing
    lib = ctypes.CDLL(q.LIB_PATH)
    for n in names:
        getattr(lib, n)


def test_sizes_and_pool_table(q):
    c = q.Cfg(4096, 512, 4, 1024)
    assert q.qe_expert_bytes(c, 4) == 7_077_888
    assert q.qe_expert_bytes(c, 2) == 3_932_160
    table, seg = q.qe_pool_table(c, 1 << 24, 4, 3)
    stride = q.qe_expert_bytes(c, 4)
    assert table[2].gate.wq == (1 << 24) + 2 * stride + seg[0]
    assert table[1].down.biases == (1 << 24) + stride + seg[8]
    assert all(t.bits == 4 for e in range(3) for t in (table[e].gate, table[e].up, table[e].down))
    assert seg == sorted(seg) and all(s % 256 == 0 for s in seg)
    assert q.qe_workspace_bytes(c, 1) > 0 and q.qe_workspace_bytes(c, 256) > q.qe_workspace_bytes(c, 1)


@pytest.mark.parametrize("cfg,msg", [
    ((4096, 512, 4, 1000), "inter"),
    ((4100, 512, 4, 1024), "hidden"),
    ((4096, 512, 0, 1024), "top_k"),
    ((4096, 4, 8, 1024), "top_k"),
    ((4096, 2048, 4, 1024), "n_experts"),
])
def test_invalid_shapes_rejected_before_launch(q, cfg, msg):
    c = q.Cfg(*cfg)
    layer = q.Layer(16, 0, 0, 16)
    rc = q.lib.moe_layer_step(ctypes.byref(c), ctypes.byref(layer), 16, 0, 1, 32, 0, None, None, 256, 1 << 20, None)
    assert rc == q.QE_ERR_INVALID_ARG
    assert msg in q.qe_last_error()
    assert q.qe_expert_bytes(c, 4) == 0


def test_null_and_misaligned_pointers_rejected(q):
    c = q.Cfg(256, 16, 2, 64)
    ws_bytes = q.qe_workspace_bytes(c, 1)
    layer = q.Layer(0, 0, 0, 4096)
    rc = q.lib.moe_layer_step(ctypes.byref(c), ctypes.byref(layer), 4096, 0, 1, 8192, 0, None, None, 1 << 20,
                              ws_bytes, None)
    assert rc == q.QE_ERR_INVALID_ARG and "router_w" in q.qe_last_error()
    layer = q.Layer(4096 + 4, 0, 0, 4096)
    rc = q.lib.moe_layer_step(ctypes.byref(c), ctypes.byref(layer), 4096, 0, 1, 8192, 0, None, None, 1 << 20,
                              ws_bytes, None)
    assert rc == q.QE_ERR_INVALID_ARG and "router_w is not 16-byte aligned" in q.qe_last_error()
    layer = q.Layer(4096, 0, 0, 4096)
    rc = q.lib.moe_layer_step(ctypes.byref(c), ctypes.byref(layer), 4096, 0, 1, 8192, 0, None, None, 1 << 20,
                              ws_bytes - 256, None)
    assert rc == q.QE_ERR_INVALID_ARG and "workspace too small" in q.qe_last_error()
    rc = q.lib.moe_combine(16, 16, None, 1, 0, 64, 32, None)
    assert rc == q.QE_ERR_INVALID_ARG


def test_empty_batches_are_noops(q):
    c = q.Cfg(256, 16, 2, 64)
    layer = q.Layer(4096, 0, 0, 4096)
    assert q.lib.moe_layer_step(ctypes.byref(c), ctypes.byref(layer), 4096, 0, 0, 8192, 0, None, None, None, 0,
                                None) == q.QE_OK
    assert q.lib.moe_combine(None, None, None, 0, 2, 64, None, None) == q.QE_OK


def test_tier_arguments_checked_before_any_cuda_call(q):
    lib = q.lib
    h = ctypes.c_void_p()
    assert lib.qe_tier_create(None, ctypes.byref(h)) == q.QE_ERR_INVALID_ARG
    cfg = q.Cfg(256, 16, 2, 64)
    arr = (ctypes.c_void_p * 16)()
    ptr = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    for bits, layers, toks, cache, msg in [(3, 1, 1, 1 << 20, "cold_bits"), (2, 0, 1, 1 << 20, "n_layers"),
                                           (2, 1, 0, 1 << 20, "max_tokens"), (2, 1, 1, 100, "cache_bytes")]:
        d = q.TierDesc(cfg, layers, bits, toks, 0, ptr, cache)
        assert lib.qe_tier_create(ctypes.byref(d), ctypes.byref(h)) == q.QE_ERR_INVALID_ARG
        assert msg in q.qe_last_error()
        assert not h.value
    assert lib.qe_tier_slots(None) == 0
    assert lib.qe_tier_stats(None, None, None, None) == q.QE_ERR_INVALID_ARG
    assert lib.qe_tier_resolve(None, 0, None, 0, None, None) == q.QE_ERR_INVALID_ARG
    lib.qe_tier_destroy(None)


def test_host_buffer_step_arguments_checked_first(q):
    """moe_layer_step_host rejects bad arguments before any CUDA call."""
    lib = q.lib
    cfg = q.Cfg(256, 16, 2, 64)
    layer = q.Layer(None, None, None, None)
    buf = (ctypes.c_float * 256)()
    assert lib.moe_layer_step_host(ctypes.byref(cfg), ctypes.byref(layer), None, 0, 1, buf, 0, None, 0,
                                   None) == q.QE_ERR_INVALID_ARG
    assert lib.moe_layer_step_host(ctypes.byref(cfg), ctypes.byref(layer), buf, 5, 1, buf, 0, None, 0,
                                   None) == q.QE_ERR_INVALID_ARG
    assert "x_dtype" in q.qe_last_error()
    assert lib.moe_layer_step_host(ctypes.byref(cfg), ctypes.byref(layer), buf, 0, 1, buf, 0, None, 0,
                                   None) == q.QE_ERR_INVALID_ARG
    assert "workspace" in q.qe_last_error()
    assert lib.moe_layer_step_host(ctypes.byref(cfg), ctypes.byref(layer), buf, 0, 0, buf, 0, None, 0, None) == q.QE_OK


def test_build_script_loads_without_the_library():
    """A fresh checkout has no libqexpert.so, and importing the package needs
    it: the build entry point must reach the build script without importing
    the package."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, __graft_entry__ as g; b = g._library_builder(); "
            "assert callable(b.build) and b.sources(), 'no build()'; "
            "assert 'quantized_expert_matvec_b200' not in sys.modules, 'package imported'; print('ok')")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


@pytest.mark.parametrize("nh,dk,dv,what", [
    (-1, 128, 128, "n_heads"), (4, 6, 8, "dk"), (4, 516, 8, "dk"), (4, 0, 8, "dk"), (4, 128, 0, "dv"),
])
def test_gdn_bad_shapes_rejected_before_launch(q, nh, dk, dv, what):
    rc = q.lib.gdn_decode_step(nh, dk, dv, 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20, 6 << 20, 7 << 20, None)
    assert rc == q.QE_ERR_INVALID_ARG
    assert "gdn_decode_step" in q.qe_last_error()


def test_gdn_bad_pointers_rejected_before_launch(q):
    L = q.lib
    M = 1 << 20
    # NULL, misaligned state / k (16 bytes needed), misaligned v (4 bytes)
    assert L.gdn_decode_step(2, 128, 8, None, 2 * M, 3 * M, 4 * M, 5 * M, 6 * M, 7 * M, None) == q.QE_ERR_INVALID_ARG
    assert L.gdn_decode_step(2, 128, 8, M + 8, 2 * M, 3 * M, 4 * M, 5 * M, 6 * M, 7 * M, None) == q.QE_ERR_INVALID_ARG
    assert "16-byte" in q.qe_last_error()
    assert L.gdn_decode_step(2, 128, 8, M, 2 * M, 3 * M + 4, 4 * M, 5 * M, 6 * M, 7 * M, None) == q.QE_ERR_INVALID_ARG
    assert L.gdn_decode_step(2, 128, 8, M, 2 * M, 3 * M, 4 * M + 2, 5 * M, 6 * M, 7 * M, None) == q.QE_ERR_INVALID_ARG
    assert "4-byte" in q.qe_last_error()
    # out inside the state, and out overlapping v by one element
    assert L.gdn_decode_step(2, 128, 8, M, 2 * M, 3 * M, 4 * M, 5 * M, 6 * M, M + 4096, None) == q.QE_ERR_INVALID_ARG
    assert "overlaps" in q.qe_last_error()
    assert L.gdn_decode_step(2, 128, 8, M, 2 * M, 3 * M, 4 * M + 60, 5 * M, 6 * M, 4 * M, None) == q.QE_ERR_INVALID_ARG
    # no heads: nothing to do, no pointer looked at
    assert L.gdn_decode_step(0, 128, 8, None, None, None, None, None, None, None, None) == q.QE_OK


def test_gdn_binding_checks_dtypes_and_sizes_first(q):
    import torch
    S = torch.zeros((2, 8, 16), dtype=torch.float32)
    f = lambda n, dt=torch.float32: torch.zeros(n, dtype=dt)  # noqa: E731
    with pytest.raises(ValueError, match="float32"):
        q.gdn_decode_step(S, f(32, torch.float64), f(32), f(16), f(2), f(2), f(16))
    with pytest.raises(ValueError, match="elements"):
        q.gdn_decode_step(S, f(32), f(31), f(16), f(2), f(2), f(16))
    with pytest.raises(ValueError, match="CUDA"):
        q.gdn_decode_step(S, f(32), f(32), f(16), f(2), f(2), f(16))  # host tensors never reach the library
