"""ctypes binding of libqexpert.so: same entry-point names as the C ABI.

Only argument marshalling happens here; every step of the expert path runs in
the library's CUDA kernels.  Tensors must be CUDA tensors (contiguous);
``stream`` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqexpert.so")

QE_OK = 0
QE_ERR_INVALID_ARG = -1
QE_ERR_UNSUPPORTED = -2
QE_ERR_CUDA = -3
QE_ERR_TIMEOUT = -4
QE_ERR_OOM = -5
QE_F32 = 0
QE_BF16 = 1

__all__ = [
    "LIB_PATH", "lib", "QEError", "Cfg", "QMat", "Expert", "Layer", "ExpertPool",
    "QE_OK", "QE_ERR_INVALID_ARG", "QE_ERR_UNSUPPORTED", "QE_ERR_CUDA", "QE_ERR_TIMEOUT", "QE_ERR_OOM",
    "QE_F32", "QE_BF16",
    "qe_last_error", "qe_version", "qe_expert_bytes", "qe_pool_table", "qe_workspace_bytes",
    "qe_workspace_init", "qe_workspace_status", "qe_set_wait_budget_ns", "qe_test_skip_arrival", "qe_trace_fused",
    "moe_route", "moe_expert_ffn_q4", "moe_expert_ffn_q2", "moe_expert_ffn_mixed", "moe_combine",
    "moe_layer_step", "moe_layer_step_noalloc", "moe_layer_step_host", "workspace", "Tier", "TierDesc",
    "gdn_decode_step",
]


class QEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("group", ctypes.c_int32), ("eps", ctypes.c_float)]

    def __init__(self, hidden, n_experts, top_k, inter, group=64, eps=1e-6):
        super().__init__(hidden, n_experts, top_k, inter, group, eps)


class QMat(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
                ("bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class Expert(ctypes.Structure):
    _fields_ = [("gate", QMat), ("up", QMat), ("down", QMat)]


class Layer(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("logit_offset", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("experts", ctypes.c_void_p)]


class TierDesc(ctypes.Structure):
    _fields_ = [("cfg", Cfg), ("n_layers", ctypes.c_int32), ("cold_bits", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("cold_host", ctypes.POINTER(ctypes.c_void_p)), ("cache_bytes", ctypes.c_size_t)]


assert ctypes.sizeof(TierDesc) == 56


assert ctypes.sizeof(Expert) == 96


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with quantized_expert_matvec_b200/build.py "
                          "(or __graft_entry__.build()); there is no CPU fallback")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    P = ctypes.POINTER
    sigs = {
        "qe_last_error": (ctypes.c_char_p, []),
        "qe_version": (ctypes.c_char_p, []),
        "qe_expert_bytes": (sz, [P(Cfg), i32]),
        "qe_pool_table": (i32, [P(Cfg), vp, i32, i32, P(Expert), P(ctypes.c_size_t)]),
        "qe_workspace_bytes": (sz, [P(Cfg), i32]),
        "qe_workspace_init": (i32, [vp, sz, vp]),
        "qe_workspace_status": (i32, [vp, vp]),
        "qe_set_wait_budget_ns": (None, [ctypes.c_uint64]),
        "qe_test_skip_arrival": (None, [i32]),
        "qe_trace_fused": (None, [vp]),
        "moe_route": (i32, [P(Cfg), vp, i32, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]),
        "moe_expert_ffn_q4": (i32, [P(Cfg), vp, vp, vp, i32, vp, vp, sz, vp]),
        "moe_expert_ffn_q2": (i32, [P(Cfg), vp, vp, vp, i32, vp, vp, sz, vp]),
        "moe_expert_ffn_mixed": (i32, [P(Cfg), vp, vp, vp, i32, vp, vp, sz, vp]),
        "moe_combine": (i32, [vp, vp, vp, i32, i32, i32, vp, vp]),
        "moe_layer_step": (i32, [P(Cfg), P(Layer), vp, i32, i32, vp, i32, vp, vp, vp, sz, vp]),
        "moe_layer_step_noalloc": (i32, [P(Cfg), P(Layer), vp, i32, vp, i32, vp, vp, vp, vp]),
        "moe_layer_step_host": (i32, [P(Cfg), P(Layer), vp, i32, i32, vp, i32, vp, sz, vp]),
        "qe_tier_create": (i32, [P(TierDesc), P(vp)]),
        "qe_tier_resolve": (i32, [vp, i32, P(ctypes.c_int32), i32, vp, vp]),
        "qe_tier_layer_step": (i32, [vp, i32, P(Layer), vp, i32, i32, vp, i32, vp, vp, vp, sz, vp]),
        "qe_tier_stats": (i32, [vp, P(ctypes.c_uint64), P(ctypes.c_uint64), P(ctypes.c_uint64)]),
        "qe_tier_slots": (i32, [vp]),
        "qe_tier_destroy": (None, [vp]),
        "gdn_decode_step": (i32, [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != QE_OK:
        raise QEError(rc, lib.qe_last_error().decode())
    return rc


def qe_last_error() -> str:
    return lib.qe_last_error().decode()


def qe_version() -> str:
    return lib.qe_version().decode()


def qe_expert_bytes(cfg: Cfg, bits: int) -> int:
    return int(lib.qe_expert_bytes(ctypes.byref(cfg), bits))


def qe_pool_table(cfg: Cfg, base_ptr: int, bits: int, n: int):
    """Descriptors (ctypes array of Expert) and segment offsets of n experts
    stored back to back from base_ptr in the standard layout."""
    table = (Expert * max(n, 1))()
    seg = (ctypes.c_size_t * 9)()
    _check(lib.qe_pool_table(ctypes.byref(cfg), base_ptr, bits, n, table, seg))
    return table, list(seg)


def qe_workspace_bytes(cfg: Cfg, T: int) -> int:
    return int(lib.qe_workspace_bytes(ctypes.byref(cfg), T))


def qe_workspace_init(ws, stream=None):
    _check(lib.qe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def qe_workspace_status(ws, stream=None) -> int:
    """Synchronise and return the device status (0, or a negative QE_ERR_*)."""
    return int(lib.qe_workspace_status(_ptr(ws), _stream(stream)))


def qe_set_wait_budget_ns(ns: int):
    lib.qe_set_wait_budget_ns(int(ns))


def qe_test_skip_arrival(cta: int):
    lib.qe_test_skip_arrival(int(cta))


def qe_trace_fused(buf):
    """Record per-CTA phase timestamps of fused launches into buf (uint64
    CUDA tensor [SMs, 64]); None disables."""
    lib.qe_trace_fused(_ptr(buf) if buf is not None else None)


def workspace(cfg: Cfg, T: int, device="cuda"):
    """Allocate (through torch) and zero a workspace for T tokens."""
    import torch
    n = qe_workspace_bytes(cfg, T)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    qe_workspace_init(ws)
    return ws


def _nbytes(t):
    return t.numel() * t.element_size()


def moe_route(cfg, x, gamma, router_w, logit_offset, xn, topk_idx, topk_w, ws, stream=None):
    import torch
    T = x.shape[0]
    dt = QE_BF16 if x.dtype == torch.bfloat16 else QE_F32
    _check(lib.moe_route(ctypes.byref(cfg), _ptr(x), dt, _ptr(gamma), _ptr(router_w), _ptr(logit_offset), T,
                         _ptr(xn), _ptr(topk_idx), _ptr(topk_w), _ptr(ws), _nbytes(ws), _stream(stream)))


def _ffn(fn, cfg, experts, xn, topk_idx, y, ws, stream):
    T = xn.shape[0]
    _check(fn(ctypes.byref(cfg), _ptr(experts), _ptr(xn), _ptr(topk_idx), T, _ptr(y), _ptr(ws), _nbytes(ws),
              _stream(stream)))


def moe_expert_ffn_q4(cfg, experts, xn, topk_idx, y, ws, stream=None):
    _ffn(lib.moe_expert_ffn_q4, cfg, experts, xn, topk_idx, y, ws, stream)


def moe_expert_ffn_q2(cfg, experts, xn, topk_idx, y, ws, stream=None):
    _ffn(lib.moe_expert_ffn_q2, cfg, experts, xn, topk_idx, y, ws, stream)


def moe_expert_ffn_mixed(cfg, experts, xn, topk_idx, y, ws, stream=None):
    _ffn(lib.moe_expert_ffn_mixed, cfg, experts, xn, topk_idx, y, ws, stream)


def moe_combine(y, w, residual, out, stream=None):
    T, K, H = y.shape
    _check(lib.moe_combine(_ptr(y), _ptr(w), _ptr(residual), T, K, H, _ptr(out), _stream(stream)))


def moe_layer_step(cfg, layer: Layer, x, out, add_residual=False, topk_idx=None, topk_w=None, ws=None,
                   stream=None):
    import torch
    T = x.shape[0]
    dt = QE_BF16 if x.dtype == torch.bfloat16 else QE_F32
    _check(lib.moe_layer_step(ctypes.byref(cfg), ctypes.byref(layer), _ptr(x), dt, T, _ptr(out),
                              1 if add_residual else 0, _ptr(topk_idx), _ptr(topk_w), _ptr(ws), _nbytes(ws),
                              _stream(stream)))


def moe_layer_step_noalloc(cfg, layer: Layer, x, out, add_residual=False, topk_idx=None, topk_w=None,
                           status=None, stream=None):
    """One token through the layer with the library's built-in scratch
    (no workspace, no allocation); `status` is an optional int32 device
    tensor that receives the call's device-side status."""
    import torch
    if x.shape[0] != 1:
        raise ValueError("moe_layer_step_noalloc takes exactly one token")
    dt = QE_BF16 if x.dtype == torch.bfloat16 else QE_F32
    _check(lib.moe_layer_step_noalloc(ctypes.byref(cfg), ctypes.byref(layer), _ptr(x), dt, _ptr(out),
                                      1 if add_residual else 0, _ptr(topk_idx), _ptr(topk_w), _ptr(status),
                                      _stream(stream)))


class Tier:
    """A two-tier expert store (qe_tier_*): cold_host[l][e] is the host
    address of cold expert (l, e) in the standard pool layout at cold_bits,
    or None for a hot expert.  Owns the native tier until close()."""

    def __init__(self, cfg: Cfg, cold_host, cold_bits: int, cache_bytes: int, max_tokens: int = 1):
        L = len(cold_host)
        E = cfg.n_experts
        arr = (ctypes.c_void_p * (L * E))()
        for l in range(L):
            for e in range(E):
                arr[l * E + e] = cold_host[l][e]
        self._arr = arr
        d = TierDesc(cfg, L, cold_bits, max_tokens, 0, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)),
                     int(cache_bytes))
        h = ctypes.c_void_p()
        _check(lib.qe_tier_create(ctypes.byref(d), ctypes.byref(h)))
        self.handle = h
        self.cfg = cfg

    @property
    def slots(self) -> int:
        return lib.qe_tier_slots(self.handle)

    def stats(self):
        """(hits, misses, h2d_bytes) since creation."""
        a, b, c = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib.qe_tier_stats(self.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
        return a.value, b.value, c.value

    def resolve(self, layer: int, idx, dev_table, stream=None):
        idx = [int(i) for i in idx]
        arr = (ctypes.c_int32 * len(idx))(*idx)
        _check(lib.qe_tier_resolve(self.handle, layer, arr, len(idx), _ptr(dev_table), _stream(stream)))

    def layer_step(self, layer: int, layer_w: Layer, x, out, add_residual=False, topk_idx=None, topk_w=None,
                   ws=None, stream=None):
        import torch
        T = x.shape[0]
        dt = QE_BF16 if x.dtype == torch.bfloat16 else QE_F32
        _check(lib.qe_tier_layer_step(self.handle, layer, ctypes.byref(layer_w), _ptr(x), dt, T, _ptr(out),
                                      1 if add_residual else 0, _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                      _nbytes(ws), _stream(stream)))

    def close(self):
        if self.handle:
            lib.qe_tier_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_layer_step_host(cfg, layer: Layer, x_host, out_host, add_residual=False, ws=None, stream=None):
    """The layer step on host tensors (pinned for asynchronous copies):
    copy in, step, copy out, synchronise."""
    import torch
    if x_host.is_cuda or out_host.is_cuda:
        raise ValueError("moe_layer_step_host takes host tensors")
    if not (x_host.is_contiguous() and out_host.is_contiguous()):
        raise ValueError("expected contiguous tensors")
    T = x_host.shape[0]
    dt = QE_BF16 if x_host.dtype == torch.bfloat16 else QE_F32
    _check(lib.moe_layer_step_host(ctypes.byref(cfg), ctypes.byref(layer), x_host.data_ptr(), dt, T,
                                   out_host.data_ptr(), 1 if add_residual else 0, _ptr(ws), _nbytes(ws),
                                   _stream(stream)))


class ExpertPool:
    """n experts of one bit width, back to back in one device buffer
    (standard layout of qe_pool_table), plus the device descriptor table."""

    def __init__(self, cfg: Cfg, n: int, bits: int, device="cuda"):
        import torch
        self.cfg, self.n, self.bits = cfg, n, bits
        self.stride = qe_expert_bytes(cfg, bits)
        if self.stride == 0:
            raise QEError(QE_ERR_INVALID_ARG, qe_last_error())
        self.buf = torch.empty(self.stride * n + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.base = (base + 255) // 256 * 256
        self.host_table, self.seg = qe_pool_table(cfg, self.base, bits, n)
        raw = bytes(self.host_table)[: ctypes.sizeof(Expert) * n]
        self.table = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)

    def seg_ptr(self, seg: int, expert: int = 0) -> int:
        """Device address of segment `seg` (0..8, qe_pool_table order) of an expert."""
        return self.base + expert * self.stride + self.seg[seg]


def gdn_decode_step(state, q, k, v, alpha, beta, out, stream=None):
    """One GatedDeltaNet decode step for every head, in place on ``state``
    (fp32 CUDA tensors: state [n_heads, dv, dk], q and k [n_heads, dk], v and
    out [n_heads, dv], alpha and beta [n_heads])."""
    import torch
    if state.dim() != 3:
        raise ValueError("state must be [n_heads, dv, dk]")
    nh, dv, dk = (int(d) for d in state.shape)
    for name, t, n in (("state", state, nh * dv * dk), ("q", q, nh * dk), ("k", k, nh * dk), ("v", v, nh * dv),
                       ("alpha", alpha, nh), ("beta", beta, nh), ("out", out, nh * dv)):
        if t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32, got {t.dtype}")
        if t.numel() != n:
            raise ValueError(f"{name} has {t.numel()} elements, expected {n}")
    _check(lib.gdn_decode_step(nh, dk, dv, _ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                               _ptr(out), _stream(stream)))
