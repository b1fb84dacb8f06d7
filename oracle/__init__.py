"""CPU oracle for the dropless sparse MoE feed-forward block (ctypes wrapper).

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline leg may import this package.  The CUDA implementation never does.
The arithmetic lives in moe_oracle.c, which carries the definitions and the
passages of the pages each step follows; this file only marshals arguments.
`oracle.mxfp4` (numpy) decodes MXFP4 expert weights and feeds them to the
same expert arithmetic.

Functions accept torch CPU tensors (float32, or bfloat16 for activations and
expert weights) or numpy arrays, and return numpy arrays (float64 results).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class OracleShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("I_shared", ctypes.c_int32), ("routed_scale", ctypes.c_double),
                ("act_bf16", ctypes.c_int32), ("w_bf16", ctypes.c_int32)]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-Wall", "-shared", "-fPIC", "-o", _LIB,
                               _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        S = ctypes.POINTER(OracleShape)
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        _lib.oracle_router.argtypes = [S, P, P, P, P, i64, P]
        _lib.oracle_topk_softmax.argtypes = [i64, i32, i32, P, P, P]
        _lib.oracle_permute.argtypes = [i64, i32, i32, P, P, P, P, P]
        _lib.oracle_expert.argtypes = [i32, i32, P, P, i32, P, P]
        _lib.oracle_moe_block.argtypes = [S, P, P, P, P, P, P, P, P, i64, P, P, P]
        _lib.oracle_moe_dense.argtypes = [S, P, P, P, P, P, P, P, P]
        _lib.oracle_threads.argtypes = []
        for f in ("oracle_router", "oracle_topk_softmax", "oracle_permute", "oracle_expert",
                  "oracle_moe_block", "oracle_moe_dense", "oracle_threads"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def _buf(t):
    """(keep-alive object, pointer, is_bf16) for a tensor/array, or (None, None, 0)."""
    if t is None:
        return None, None, 0
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu").contiguous()
        if t.dtype == torch.bfloat16:
            a = t.view(torch.int16).numpy()
            return a, a.ctypes.data, 1
        a = t.numpy()
    else:
        a = np.ascontiguousarray(t)
    if a.dtype == np.float64:
        return a, a.ctypes.data, 0
    if a.dtype != np.float32 and a.dtype != np.int32 and a.dtype != np.int64:
        a = a.astype(np.float32)
    a = np.ascontiguousarray(a)
    return a, a.ctypes.data, 0


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _shape(T, H, I, E, k, n_shared=0, I_shared=0, routed_scale=1.0, act_bf16=0, w_bf16=0):
    return OracleShape(int(T), int(H), int(I), int(E), int(k), int(n_shared), int(I_shared),
                       float(routed_scale), int(act_bf16), int(w_bf16))


def threads() -> int:
    return _load().oracle_threads()


def router(x, w_router, bias=None, tokens=None) -> np.ndarray:
    """Router logits [n, E] (float64) for the given token rows (all rows if None)."""
    lib = _load()
    kx, px, xb = _buf(x)
    kw, pw, _ = _buf(w_router.float() if isinstance(w_router, torch.Tensor) else w_router)
    kb, pb, _ = _buf(bias)
    T, H = x.shape
    E = w_router.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tok is None else len(tok)
    out = np.zeros((n, E), dtype=np.float64)
    s = _shape(T, H, 1, E, 1, act_bf16=xb)
    _check(lib.oracle_router(ctypes.byref(s), px, pw, pb,
                             None if tok is None else tok.ctypes.data, n, out.ctypes.data),
           "router")
    return out


def topk_softmax(logits: np.ndarray, k: int):
    """(idx [n,k] int32, w [n,k] float64) from float64 logits [n, E]."""
    lib = _load()
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    n, E = lg.shape
    idx = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    _check(lib.oracle_topk_softmax(n, E, k, lg.ctypes.data, idx.ctypes.data, w.ctypes.data),
           "topk_softmax")
    return idx, w


def permute(topk_idx: np.ndarray, E: int):
    """(counts [E], offsets [E+1], perm [T*k], inv [T*k]) int32 from topk_idx [T, k]."""
    lib = _load()
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    perm = np.zeros(T * k, dtype=np.int32)
    inv = np.zeros(T * k, dtype=np.int32)
    _check(lib.oracle_permute(T, E, k, idx.ctypes.data, counts.ctypes.data, offsets.ctypes.data,
                              perm.ctypes.data, inv.ctypes.data), "permute")
    return counts, offsets, perm, inv


def expert(gate_up_e, down_e, x_vec) -> np.ndarray:
    """One SwiGLU expert on a float64 hidden vector: gate_up_e [2I,H], down_e [H,I]."""
    lib = _load()
    k1, p1, b1 = _buf(gate_up_e)
    k2, p2, b2 = _buf(down_e)
    assert b1 == b2
    xv = np.ascontiguousarray(x_vec, dtype=np.float64)
    H = down_e.shape[0]
    I = down_e.shape[1]
    out = np.zeros(H, dtype=np.float64)
    _check(lib.oracle_expert(H, I, p1, p2, b1, xv.ctypes.data, out.ctypes.data), "expert")
    return out


def _block_args(inp, routed_scale):
    x = inp["x"]
    gu, dn = inp["gate_up"], inp["down"]
    shgu, shdn = inp.get("sh_gate_up"), inp.get("sh_down")
    T, H = x.shape
    E, twoI, _ = gu.shape
    S = 0 if shgu is None else shgu.shape[0]
    Is = 0 if shgu is None else shgu.shape[1] // 2
    bufs = [_buf(t) for t in (x, inp["w_router"], inp.get("router_bias"), gu, dn, shgu, shdn)]
    return T, H, twoI // 2, E, S, Is, bufs


def moe_block(inp: dict, k: int, routed_scale: float = 1.0, tokens=None):
    """The sparse block for the listed tokens (all if None).

    Returns (y [n,H] float64, idx [n,k] int32, w [n,k] float64)."""
    lib = _load()
    T, H, I, E, S, Is, bufs = _block_args(inp, routed_scale)
    (kx, px, xb), (kw, pw, _), (kb, pb, _), (k1, p1, wb), (k2, p2, _), (k3, p3, _), \
        (k4, p4, _) = bufs
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tok is None else len(tok)
    y = np.zeros((n, H), dtype=np.float64)
    idx = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    s = _shape(T, H, I, E, k, S, Is, routed_scale, xb, wb)
    _check(lib.oracle_moe_block(ctypes.byref(s), px, pw, pb, p1, p2, p3, p4,
                                None if tok is None else tok.ctypes.data, n, y.ctypes.data,
                                idx.ctypes.data, w.ctypes.data), "moe_block")
    return y, idx, w


def moe_dense(inp: dict, k: int, routed_scale: float = 1.0) -> np.ndarray:
    """Brute-force dense block over all tokens: y [T, H] float64."""
    lib = _load()
    T, H, I, E, S, Is, bufs = _block_args(inp, routed_scale)
    (kx, px, xb), (kw, pw, _), (kb, pb, _), (k1, p1, wb), (k2, p2, _), (k3, p3, _), \
        (k4, p4, _) = bufs
    y = np.zeros((T, H), dtype=np.float64)
    s = _shape(T, H, I, E, k, S, Is, routed_scale, xb, wb)
    _check(lib.oracle_moe_dense(ctypes.byref(s), px, pw, pb, p1, p2, p3, p4, y.ctypes.data),
           "moe_dense")
    return y
