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
from typing import Optional

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
        _lib.oracle_route_noaux_tc.argtypes = [i64, i32, i32, i32, i32, P, P, P, P]
        _lib.oracle_moe_backward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                             P, P]
        _lib.oracle_aux_loss.argtypes = [i64, i32, i32, P, P, ctypes.c_double, P, P]
        _lib.oracle_moe_block_routed.argtypes = [S, P, P, P, P, P, P, i64, P, P, P]
        for f in ("oracle_router", "oracle_topk_softmax", "oracle_permute", "oracle_expert",
                  "oracle_moe_block", "oracle_moe_dense", "oracle_threads",
                  "oracle_route_noaux_tc", "oracle_moe_block_routed", "oracle_moe_backward",
                  "oracle_aux_loss"):
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


def moe_block_experts(inp: dict, k: int, routed_scale: float = 1.0, e_begin: int = 0,
                      e_end: Optional[int] = None, with_shared: bool = True, tokens=None):
    """One expert-parallel rank's partial output, for the listed tokens.

    "Mixture of Experts in Transformers", section "expert parallelism": each
    rank keeps a slice of the experts, masks the experts it does not hold, and
    the ranks' partial outputs are summed by an all-reduce.  The partial of
    the rank holding routed experts [e_begin, e_end) is
        y_t = routed_scale * sum over j with e_begin <= idx_tj < e_end of w_tj * FFN_idx_tj(x_t)
              (+ the shared experts' FFNs when with_shared),
    with the routing (idx, w) of the whole block.  Plain loops over tokens
    and their k slots; the expert arithmetic is oracle.expert.
    Returns y [n, H] float64."""
    x = inp["x"]
    T, H = x.shape
    E = inp["gate_up"].shape[0]
    e_end = E if e_end is None else e_end
    lg = router(x, inp["w_router"], inp.get("router_bias"), tokens=tokens)
    idx, w = topk_softmax(lg, k)
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    xs = x.float().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, dtype=np.float64)
    y = np.zeros((len(toks), H), dtype=np.float64)
    for n, t in enumerate(toks):
        xt = xs[t].astype(np.float64)
        for j in range(k):
            e = int(idx[n, j])
            if e_begin <= e < e_end:
                y[n] += routed_scale * w[n, j] * expert(inp["gate_up"][e], inp["down"][e], xt)
        if with_shared and inp.get("sh_gate_up") is not None:
            for s in range(inp["sh_gate_up"].shape[0]):
                y[n] += expert(inp["sh_gate_up"][s], inp["sh_down"][s], xt)
    return y


def route_noaux_tc(logits: np.ndarray, bias, k: int, n_group: int = 1, topk_group: int = 1):
    """DeepSeek-V3 ("noaux_tc") selection and weights from bias-free float64
    logits [n, E] and the selection-only bias [E] (or None): (idx [n,k] int32,
    w [n,k] float64).  See noaux_one in moe_oracle.c for the steps."""
    lib = _load()
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    n, E = lg.shape
    kb, pb, _ = _buf(bias.float() if isinstance(bias, torch.Tensor) else bias)
    idx = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    _check(lib.oracle_route_noaux_tc(n, E, k, n_group, topk_group, lg.ctypes.data, pb,
                                     idx.ctypes.data, w.ctypes.data), "route_noaux_tc")
    return idx, w


def moe_block_routed(inp: dict, idx: np.ndarray, w: np.ndarray, routed_scale: float = 1.0,
                     tokens=None) -> np.ndarray:
    """The block for the listed tokens (all if None) given each listed token's
    routing idx [n, k] and weights w [n, k]: y [n, H] float64."""
    lib = _load()
    T, H, I, E, S, Is, bufs = _block_args(inp, routed_scale)
    (kx, px, xb), _, _, (k1, p1, wb), (k2, p2, _), (k3, p3, _), (k4, p4, _) = bufs
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tok is None else len(tok)
    ii = np.ascontiguousarray(idx, dtype=np.int32)
    ww = np.ascontiguousarray(w, dtype=np.float64)
    k = ii.shape[1]
    y = np.zeros((n, H), dtype=np.float64)
    s = _shape(T, H, I, E, k, S, Is, routed_scale, xb, wb)
    _check(lib.oracle_moe_block_routed(ctypes.byref(s), px, p1, p2, p3, p4,
                                       None if tok is None else tok.ctypes.data, n,
                                       ii.ctypes.data, ww.ctypes.data, y.ctypes.data),
           "moe_block_routed")
    return y


def moe_block_noaux(inp: dict, k: int, routed_scale: float = 1.0, n_group: int = 1,
                    topk_group: int = 1, tokens=None):
    """The block with DeepSeek-V3 ("noaux_tc") routing: the router is bias-free
    and `router_bias` is the selection-only correction bias.
    Returns (y [n,H] float64, idx [n,k] int32, w [n,k] float64)."""
    lg = router(inp["x"], inp["w_router"], None, tokens=tokens)
    idx, w = route_noaux_tc(lg, inp.get("router_bias"), k, n_group, topk_group)
    return moe_block_routed(inp, idx, w, routed_scale, tokens=tokens), idx, w


def moe_backward(inp: dict, k: int, dy, routed_scale: float = 1.0) -> dict:
    """Gradients of the block (softmax top-k routing) for the upstream gradient
    dy [T, H], all in float64: x, gate_up, down, w_router, router_bias,
    sh_gate_up, sh_down (None without shared experts), dw [T,k] (routing
    weights) and dl [T,E] (logits).  See oracle_moe_backward for the steps."""
    lib = _load()
    T, H, I, E, S, Is, bufs = _block_args(inp, routed_scale)
    (kx, px, xb), (kw, pw, _), (kb, pb, _), (k1, p1, wb), (k2, p2, _), (k3, p3, _), \
        (k4, p4, _) = bufs
    dyv = np.ascontiguousarray(dy.double().numpy() if isinstance(dy, torch.Tensor) else dy,
                               dtype=np.float64)
    out = {
        "x": np.zeros((T, H)), "gate_up": np.zeros((E, 2 * I, H)), "down": np.zeros((E, H, I)),
        "w_router": np.zeros((E, H)), "router_bias": np.zeros(E),
        "sh_gate_up": np.zeros((S, 2 * Is, H)) if S else None,
        "sh_down": np.zeros((S, H, Is)) if S else None,
        "dw": np.zeros((T, k)), "dl": np.zeros((T, E)),
    }
    s = _shape(T, H, I, E, k, S, Is, routed_scale, xb, wb)

    def ptr(a):
        return None if a is None else a.ctypes.data
    _check(lib.oracle_moe_backward(ctypes.byref(s), px, pw, pb, p1, p2, p3, p4, dyv.ctypes.data,
                                   ptr(out["x"]), ptr(out["gate_up"]), ptr(out["down"]),
                                   ptr(out["w_router"]), ptr(out["router_bias"]),
                                   ptr(out["sh_gate_up"]), ptr(out["sh_down"]), ptr(out["dw"]),
                                   ptr(out["dl"])), "moe_backward")
    return out


def aux_loss(logits: np.ndarray, idx: np.ndarray, E: int, coef: float = 1.0):
    """(loss, dl [T, E]) of the load-balancing auxiliary loss (Switch
    Transformer eqs. 4-6 as the PhiMoE page uses it, times coef)."""
    lib = _load()
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    ii = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = ii.shape
    loss = ctypes.c_double(0.0)
    dl = np.zeros((T, E), dtype=np.float64)
    _check(lib.oracle_aux_loss(T, E, k, lg.ctypes.data, ii.ctypes.data, float(coef),
                               ctypes.byref(loss), dl.ctypes.data), "aux_loss")
    return loss.value, dl
