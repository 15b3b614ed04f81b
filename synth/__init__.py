"""Seeded synthetic inputs for the quantized MoE expert step.

This module is the one piece shared by the fp64 oracle and the GPU path: it
draws the inputs (packed q words, bf16 scales/biases, fp32 activations and
router weights, Zipf popularity offsets) and nothing else.  It holds none of
the step's arithmetic.

Value distributions follow the workload shapes of the Flash-MoE pages
(512 experts, top-4, 4-bit MLX-style affine group quantisation, group 64):

* q words: 32 uniform random bits per uint32 word, so every 4-bit (or 2-bit)
  field is U{0..15} (U{0..3});
* scales: bf16(U(0.005, 0.02)); biases: bf16(N(0, 0.01));
* x: N(0, 1) fp32 (bf16 for the batched workload); router W: N(0, 0.02) fp32;
* Zipf(s=1.1) expert popularity enters the router as a per-layer logit offset;
* GatedDeltaNet decode step (64 heads x 128x128 state per layer): state
  N(0, 0.1) fp32, q and k uniform on the unit sphere (normalised N(0,1) draws,
  rounded to fp32), v N(0, 1) fp32, decay alpha bf16(U(0.9, 1)) and write
  strength beta bf16(U(0, 1)), both as fp32.

Host fills (numpy) come from ``libsynth_host.so`` and device fills (torch
CUDA tensors) from ``libsynth_dev.so``; both evaluate the same counter-based
splitmix64 streams with IEEE-exact double arithmetic, so they agree bit for bit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_DEV_SO = os.path.join(_HERE, "libsynth_dev.so")

# tensor ids (must match synth_core.h)
T_GATE_WQ, T_GATE_S, T_GATE_B = 1, 2, 3
T_UP_WQ, T_UP_S, T_UP_B = 4, 5, 6
T_DOWN_WQ, T_DOWN_S, T_DOWN_B = 7, 8, 9
T_ROUTER, T_X, T_PERM = 10, 11, 12
T_GDN_S, T_GDN_Q, T_GDN_K, T_GDN_V, T_GDN_ALPHA, T_GDN_BETA = 13, 14, 15, 16, 17, 18

# value kinds
K_U32, K_BF16_UNIFORM, K_BF16_NORMAL, K_F32_NORMAL = 0, 1, 2, 3

SCALE_LO, SCALE_HI = 0.005, 0.02
BIAS_STD = 0.01
ROUTER_STD = 0.02
X_STD = 1.0
GROUP = 64

# a (layer-like) id used for token streams, so token inputs never share a
# stream with weights
TOKEN_STREAM = 0xFFFFF

# recipe of each expert tensor: (tensor id, kind, p0, p1)
_WQ = {"gate": T_GATE_WQ, "up": T_UP_WQ, "down": T_DOWN_WQ}
_SC = {"gate": T_GATE_S, "up": T_UP_S, "down": T_DOWN_S}
_BI = {"gate": T_GATE_B, "up": T_UP_B, "down": T_DOWN_B}


def build(verbose: bool = False) -> None:
    """Compile the host (gcc) and device (nvcc, sm_100a) generator libraries."""
    host_cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                "-o", _HOST_SO, os.path.join(_HERE, "synth_host.c")]
    dev_cmd = ["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "--fmad=false",
               "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_SO,
               os.path.join(_HERE, "synth_dev.cu")]
    for cmd in (host_cmd, dev_cmd):
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_SO):
            build()
        lib = ctypes.CDLL(_HOST_SO)
        lib.sy_host_fill.restype = ctypes.c_int
        lib.sy_host_fill.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                     ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                     ctypes.c_double, ctypes.c_double]
        lib.sy_host_key.restype = ctypes.c_uint64
        lib.sy_host_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        lib.sy_host_draw.restype = ctypes.c_uint64
        lib.sy_host_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        for fn in ("sy_host_normal",):
            getattr(lib, fn).restype = ctypes.c_double
            getattr(lib, fn).argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.sy_host_ln.restype = ctypes.c_double
        lib.sy_host_ln.argtypes = [ctypes.c_double]
        lib.sy_host_cos2pi.restype = ctypes.c_double
        lib.sy_host_cos2pi.argtypes = [ctypes.c_double]
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError(f"{_DEV_SO} is missing: run synth.build() (or __graft_entry__.build())")
        lib = ctypes.CDLL(_DEV_SO)
        lib.sy_dev_fill_family.restype = ctypes.c_int
        lib.sy_dev_fill_family.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                           ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                           ctypes.c_uint32, ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
        _dev = lib
    return _dev


def _dtype(kind: int):
    return np.uint16 if kind in (K_BF16_UNIFORM, K_BF16_NORMAL) else (
        np.float32 if kind == K_F32_NORMAL else np.uint32)


def host_fill(n: int, kind: int, seed: int, a: int, b: int, tensor: int,
              p0: float = 0.0, p1: float = 0.0, i0: int = 0) -> np.ndarray:
    """Elements [i0, i0+n) of stream (seed, a, b, tensor) as a numpy array."""
    out = np.empty(int(n), dtype=_dtype(kind))
    rc = _host_lib().sy_host_fill(out.ctypes.data, int(i0), int(n), int(kind), int(seed),
                                  int(a), int(b), int(tensor), float(p0), float(p1))
    if rc != 0:
        raise RuntimeError(f"sy_host_fill failed ({rc})")
    return out


def host_fill_into(dst_ptr: int, n: int, kind: int, seed: int, a: int, b: int, tensor: int,
                   p0: float = 0.0, p1: float = 0.0, i0: int = 0) -> None:
    """Write elements [i0, i0+n) of stream (seed, a, b, tensor) to host memory
    at dst_ptr (for pinned buffers that numpy does not own)."""
    rc = _host_lib().sy_host_fill(ctypes.c_void_p(dst_ptr), int(i0), int(n), int(kind), int(seed),
                                  int(a), int(b), int(tensor), float(p0), float(p1))
    if rc != 0:
        raise RuntimeError(f"sy_host_fill failed ({rc})")


def dev_fill_family(base_ptr: int, stride_bytes: int, n_per: int, n_members: int, kind: int,
                    seed: int, a: int, b0: int, tensor: int, p0: float = 0.0, p1: float = 0.0,
                    stream: int = 0) -> None:
    """Fill a run of device tensors: member m at base_ptr + m*stride_bytes gets
    n_per elements of stream (seed, a, b0+m, tensor)."""
    rc = _dev_lib().sy_dev_fill_family(ctypes.c_void_p(base_ptr), int(stride_bytes), int(n_per),
                                       int(n_members), int(kind), int(seed), int(a), int(b0),
                                       int(tensor), float(p0), float(p1), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"sy_dev_fill_family failed ({rc})")


# --------------------------------------------------------------------------
# recipes: which stream and distribution each input tensor uses
# --------------------------------------------------------------------------

def wq_recipe(mat: str):
    return _WQ[mat], K_U32, 0.0, 0.0


def scale_recipe(mat: str):
    return _SC[mat], K_BF16_UNIFORM, SCALE_LO, SCALE_HI


def bias_recipe(mat: str):
    return _BI[mat], K_BF16_NORMAL, BIAS_STD, 0.0


def matrix_shape(mat: str, hidden: int, inter: int):
    """(rows, cols) of an expert matrix: gate/up [I, H], down [H, I]."""
    return (inter, hidden) if mat in ("gate", "up") else (hidden, inter)


def host_expert(seed: int, layer: int, expert: int, hidden: int, inter: int, bits: int) -> dict:
    """One expert's packed tensors on the host: for m in gate/up/down,
    '<m>_wq' uint32 [rows, cols*bits/32], '<m>_s' and '<m>_b' bf16 bits
    (uint16) [rows, cols/64]."""
    out = {}
    for mat in ("gate", "up", "down"):
        rows, cols = matrix_shape(mat, hidden, inter)
        nw = rows * cols * bits // 32
        ng = rows * cols // GROUP
        t, k, p0, p1 = wq_recipe(mat)
        out[mat + "_wq"] = host_fill(nw, k, seed, layer, expert, t, p0, p1).reshape(rows, cols * bits // 32)
        t, k, p0, p1 = scale_recipe(mat)
        out[mat + "_s"] = host_fill(ng, k, seed, layer, expert, t, p0, p1).reshape(rows, cols // GROUP)
        t, k, p0, p1 = bias_recipe(mat)
        out[mat + "_b"] = host_fill(ng, k, seed, layer, expert, t, p0, p1).reshape(rows, cols // GROUP)
    return out


def host_router(seed: int, layer: int, n_experts: int, hidden: int) -> np.ndarray:
    """Router weights W_r fp32 [E, H] ~ N(0, 0.02)."""
    return host_fill(n_experts * hidden, K_F32_NORMAL, seed, layer, 0, T_ROUTER,
                     ROUTER_STD).reshape(n_experts, hidden)


def host_tokens(seed: int, t0: int, n_tokens: int, hidden: int, bf16: bool = False) -> np.ndarray:
    """Token activations x [n, H] ~ N(0,1): fp32, or bf16 bits (uint16) if bf16."""
    rows = []
    for t in range(t0, t0 + n_tokens):
        kind = K_BF16_NORMAL if bf16 else K_F32_NORMAL
        rows.append(host_fill(hidden, kind, seed, TOKEN_STREAM, t, T_X, X_STD))
    return np.stack(rows) if rows else np.empty((0, hidden), np.uint16 if bf16 else np.float32)


def expert_permutation(seed: int, layer: int, n_experts: int) -> np.ndarray:
    """Seeded permutation pi of the experts: pi[e] = popularity rank (0-based)
    of expert e.  Experts are ranked by one random 64-bit draw each."""
    key = _host_lib().sy_host_key(int(seed), int(layer), 0, T_PERM)
    draws = np.array([_host_lib().sy_host_draw(key, e) for e in range(n_experts)], dtype=np.uint64)
    order = np.argsort(draws, kind="stable")          # order[r] = expert with rank r
    rank = np.empty(n_experts, dtype=np.int64)
    rank[order] = np.arange(n_experts)
    return rank


def zipf_logit_offset(seed: int, layer: int, n_experts: int, s: float = 1.1,
                      alpha: float = 0.40) -> np.ndarray:
    """Per-layer router logit offset alpha*ln(p_rank(e)), p_r proportional to
    r^-s over ranks r = 1..E (Zipf popularity).  Returned as fp32 [E]."""
    rank = expert_permutation(seed, layer, n_experts)
    r = np.arange(1, n_experts + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return (alpha * np.log(p[rank])).astype(np.float32)


def hot_set(seed: int, layer: int, n_experts: int, n_hot: int) -> np.ndarray:
    """Boolean mask of the n_hot most popular experts of a layer (ranks < n_hot)."""
    return expert_permutation(seed, layer, n_experts) < n_hot


GDN_STATE_STD = 0.1
GDN_ALPHA_LO, GDN_ALPHA_HI = 0.9, 1.0


def _unit_rows(z: np.ndarray) -> np.ndarray:
    """Rows of z scaled to unit length in float64, then rounded to fp32 (a
    sample from the uniform distribution on the sphere)."""
    z = z.astype(np.float64)
    n = np.sqrt((z * z).sum(axis=1, keepdims=True))
    return (z / np.where(n > 0, n, 1.0)).astype(np.float32)


def host_gdn_state(seed: int, layer: int, n_heads: int, dk: int, dv: int) -> np.ndarray:
    """Initial recurrent state S fp32 [n_heads, dv, dk] ~ N(0, 0.1)."""
    return host_fill(n_heads * dv * dk, K_F32_NORMAL, seed, layer, 0, T_GDN_S,
                     GDN_STATE_STD).reshape(n_heads, dv, dk)


def host_gdn_token(seed: int, layer: int, t: int, n_heads: int, dk: int, dv: int) -> dict:
    """Inputs of one decode step of one layer: q, k [n_heads, dk] unit rows,
    v [n_heads, dv] ~ N(0,1), alpha, beta [n_heads] (fp32)."""
    def bf16_uniform(tensor, lo, hi):
        b = host_fill(n_heads, K_BF16_UNIFORM, seed, layer, t, tensor, lo, hi)
        return (b.astype(np.uint32) << 16).view(np.float32).copy()
    return {
        "q": _unit_rows(host_fill(n_heads * dk, K_F32_NORMAL, seed, layer, t, T_GDN_Q, 1.0).reshape(n_heads, dk)),
        "k": _unit_rows(host_fill(n_heads * dk, K_F32_NORMAL, seed, layer, t, T_GDN_K, 1.0).reshape(n_heads, dk)),
        "v": host_fill(n_heads * dv, K_F32_NORMAL, seed, layer, t, T_GDN_V, 1.0).reshape(n_heads, dv),
        "alpha": bf16_uniform(T_GDN_ALPHA, GDN_ALPHA_LO, GDN_ALPHA_HI),
        "beta": bf16_uniform(T_GDN_BETA, 0.0, 1.0),
    }
