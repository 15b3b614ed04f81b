"""fp64 CPU oracle of the quantized MoE expert step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and this
package never imports the CUDA library: the two share no code.  Inputs come
from the ``synth`` generator (or from a test), never from the GPU path.

The arithmetic lives in ``oracle.c`` (plain C, double precision, sums in index
order); this module only marshals numpy arrays and sequences the steps of one
layer as the Flash-MoE pages order them (lilting.ch article on Flash-MoE,
sections "Model architecture" and "Metal Compute Shaders"): RMSNorm, router,
softmax + top-K, per-expert gate/up dequant-matvec, SwiGLU, down
dequant-matvec, weighted combine.  ``gdn_step`` is the GatedDeltaNet decode
step of the same model (lilting.ch article, section "GatedDeltaNet
acceleration"), stated in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")

_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_I32 = ctypes.POINTER(ctypes.c_int32)


class _QMat(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("bits", ctypes.c_int32)]


def build(verbose: bool = False) -> None:
    """Compile liboracle.so with gcc (OpenMP over independent rows only)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-o", _SO, os.path.join(_HERE, "oracle.c"), "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


_lib = None


def _L():
    global _lib
    if _lib is None:
        if not os.path.exists(_SO):
            build()
        lib = ctypes.CDLL(_SO)
        lib.or_bf16.restype = ctypes.c_double
        lib.or_bf16.argtypes = [ctypes.c_uint16]
        lib.or_q.restype = ctypes.c_uint
        lib.or_q.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.or_dequant.restype = ctypes.c_double
        lib.or_dequant.argtypes = [ctypes.POINTER(_QMat), ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.or_qmatvec.restype = None
        lib.or_qmatvec.argtypes = [ctypes.POINTER(_QMat), ctypes.c_int, ctypes.c_int, _D, _D, ctypes.c_int]
        lib.or_qmatvec_fma_form.restype = None
        lib.or_qmatvec_fma_form.argtypes = [ctypes.POINTER(_QMat), ctypes.c_int, ctypes.c_int, _D, _D]
        lib.or_rmsnorm.restype = None
        lib.or_rmsnorm.argtypes = [_D, _D, ctypes.c_int, ctypes.c_double, _D]
        lib.or_router.restype = None
        lib.or_router.argtypes = [_F, _D, _F, ctypes.c_int, ctypes.c_int, _D, ctypes.c_int]
        lib.or_softmax.restype = None
        lib.or_softmax.argtypes = [_D, ctypes.c_int, _D]
        lib.or_topk.restype = None
        lib.or_topk.argtypes = [_D, ctypes.c_int, ctypes.c_int, _I32, _D]
        lib.or_silu.restype = ctypes.c_double
        lib.or_silu.argtypes = [ctypes.c_double]
        lib.or_swiglu.restype = None
        lib.or_swiglu.argtypes = [_D, _D, ctypes.c_int, _D]
        lib.or_expert_ffn.restype = None
        lib.or_expert_ffn.argtypes = [ctypes.POINTER(_QMat)] * 3 + [ctypes.c_int, ctypes.c_int, _D, _D, _D,
                                                                    ctypes.c_int]
        lib.or_gdn_step.restype = None
        lib.or_gdn_step.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _D, _D, _D, _D, _D, _D, _D]
        lib.or_combine.restype = None
        lib.or_combine.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, _D, _D]
        _lib = lib
    return _lib


def _d(a):
    return a.ctypes.data_as(_D)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _qmat(wq, s, b, bits):
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    b = np.ascontiguousarray(b, dtype=np.uint16)
    m = _QMat(wq.ctypes.data, s.ctypes.data, b.ctypes.data, int(bits))
    return m, (wq, s, b)  # keep the arrays alive with the struct


def bf16_value(bits16) -> np.ndarray:
    """Exact values of bf16 bit patterns (uint16 array) as float64."""
    b = np.asarray(bits16, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def q_value(wq, cols: int, bits: int, r: int, c: int) -> int:
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    return int(_L().or_q(wq.ctypes.data, cols, bits, r, c))


def dequant(wq, s, b, bits: int, cols: int, r: int, c: int) -> float:
    m, keep = _qmat(wq, s, b, bits)
    return float(_L().or_dequant(ctypes.byref(m), cols, r, c))


def qmatvec(wq, s, b, bits: int, x, nthreads: int = 1) -> np.ndarray:
    """y = deq(W) x for a packed [rows, cols] matrix; x has cols entries."""
    x = _f64(x)
    rows = np.asarray(wq).shape[0]
    cols = x.shape[0]
    y = np.empty(rows, np.float64)
    m, keep = _qmat(wq, s, b, bits)
    _L().or_qmatvec(ctypes.byref(m), rows, cols, _d(x), _d(y), int(nthreads))
    return y


def qmatvec_fma_form(wq, s, b, bits: int, x) -> np.ndarray:
    x = _f64(x)
    rows = np.asarray(wq).shape[0]
    y = np.empty(rows, np.float64)
    m, keep = _qmat(wq, s, b, bits)
    _L().or_qmatvec_fma_form(ctypes.byref(m), rows, x.shape[0], _d(x), _d(y))
    return y


def rmsnorm(x, gamma=None, eps: float = 1e-6) -> np.ndarray:
    x = _f64(x)
    xn = np.empty_like(x)
    g = _f64(gamma) if gamma is not None else None
    _L().or_rmsnorm(_d(x), _d(g) if g is not None else None, x.shape[0], float(eps), _d(xn))
    return xn


def router(W, xn, offset=None, nthreads: int = 1) -> np.ndarray:
    W = np.ascontiguousarray(W, dtype=np.float32)
    xn = _f64(xn)
    E, H = W.shape
    off = np.ascontiguousarray(offset, dtype=np.float32) if offset is not None else None
    out = np.empty(E, np.float64)
    _L().or_router(W.ctypes.data_as(_F), _d(xn), off.ctypes.data_as(_F) if off is not None else None,
                   E, H, _d(out), int(nthreads))
    return out


def softmax(logits) -> np.ndarray:
    lg = _f64(logits)
    p = np.empty_like(lg)
    _L().or_softmax(_d(lg), lg.shape[0], _d(p))
    return p


def topk(logits, K: int):
    lg = _f64(logits)
    idx = np.empty(K, np.int32)
    w = np.empty(K, np.float64)
    _L().or_topk(_d(lg), lg.shape[0], int(K), idx.ctypes.data_as(_I32), _d(w))
    return idx, w


def silu(g: float) -> float:
    return float(_L().or_silu(float(g)))


def swiglu(g, u) -> np.ndarray:
    g, u = _f64(g), _f64(u)
    h = np.empty_like(g)
    _L().or_swiglu(_d(g), _d(u), g.shape[0], _d(h))
    return h


def expert_ffn(expert: dict, bits: int, xn, nthreads: int = 1, return_h: bool = False):
    """y = Wd (silu(Wg xn) * (Wu xn)) for one expert given as the dict of
    packed tensors produced by ``synth.host_expert``."""
    xn = _f64(xn)
    H = xn.shape[0]
    I = np.asarray(expert["gate_wq"]).shape[0]
    mg, k1 = _qmat(expert["gate_wq"], expert["gate_s"], expert["gate_b"], bits)
    mu, k2 = _qmat(expert["up_wq"], expert["up_s"], expert["up_b"], bits)
    md, k3 = _qmat(expert["down_wq"], expert["down_s"], expert["down_b"], bits)
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float64)
    _L().or_expert_ffn(ctypes.byref(mg), ctypes.byref(mu), ctypes.byref(md), H, I, _d(xn), _d(y), _d(h),
                       int(nthreads))
    return (y, h) if return_h else y


def combine(y, w, residual=None) -> np.ndarray:
    y = _f64(y)
    K, H = y.shape
    w = _f64(w)
    res = _f64(residual) if residual is not None else None
    out = np.empty(H, np.float64)
    _L().or_combine(_d(y), _d(w), K, H, _d(res) if res is not None else None, _d(out))
    return out


def layer_step(x, router_w, experts, bits_of, K: int, eps: float = 1e-6, gamma=None, offset=None,
               residual: bool = False, nthreads: int = 1) -> dict:
    """One token through one MoE layer.

    ``experts(e)`` returns expert e's packed tensors (``synth.host_expert``
    layout) and ``bits_of(e)`` its bit width; only the K selected experts are
    requested.  Returns xn, logits, idx, w, y [K, H] and out.
    """
    x = _f64(x)
    xn = rmsnorm(x, gamma, eps)
    logits = router(router_w, xn, offset, nthreads)
    idx, w = topk(logits, K)
    y = np.stack([expert_ffn(experts(int(e)), bits_of(int(e)), xn, nthreads) for e in idx])
    out = combine(y, w, x if residual else None)
    return {"xn": xn, "logits": logits, "idx": idx, "w": w, "y": y, "out": out}


def gdn_step(S, q, k, v, alpha, beta):
    """One gated-delta-rule decode step (scal, gemv, ger, gemv per head).

    S [n_heads, dv, dk], q and k [n_heads, dk], v [n_heads, dv], alpha and
    beta [n_heads].  Returns (S', o) as new float64 arrays; S is not changed."""
    S2 = np.array(S, dtype=np.float64, copy=True, order="C")
    nh, dv, dk = S2.shape
    q, k, v = _f64(q).reshape(nh, dk), _f64(k).reshape(nh, dk), _f64(v).reshape(nh, dv)
    a, b = _f64(alpha).reshape(nh), _f64(beta).reshape(nh)
    o = np.empty((nh, dv), np.float64)
    _L().or_gdn_step(nh, dk, dv, _d(S2), _d(q), _d(k), _d(v), _d(a), _d(b), _d(o))
    return S2, o
